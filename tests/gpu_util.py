"""Helpers for the GPU parity tests: storage arrays <-> device tensors, oracle sampling."""
from __future__ import annotations

import numpy as np

from linear_recurrent_lm_b200 import inputs as I


def to_dev(x, dev="cuda"):
    import torch
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
    return torch.from_numpy(x).to(dev)


def f64(t) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def inputs_dev(d, dev="cuda"):
    return [to_dev(d[n], dev) for n in I.NAMES]


def inputs_f64(d):
    return [I.to_f64(d[n]) for n in I.NAMES]


def sample_units(B, H, k, seed=0):
    """k distinct (b, h) units, always including the first and the last."""
    rng = np.random.default_rng(seed)
    units = {(0, 0), (B - 1, H - 1)}
    while len(units) < min(k, B * H):
        units.add((int(rng.integers(B)), int(rng.integers(H))))
    return sorted(units)
