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


def checkpoint_states(ws, B, H, n_ck) -> np.ndarray:
    """Checkpoints of a forward workspace as [B, H, n_ck, 64, 64] fp64 states.

    Inside one checkpoint, element (i, j) sits at the documented tiled offset
    (i//16)*1024 + (j//8)*128 + (4*(i%8) + (j%8)//2)*4 + 2*((i//8)%2) + j%2."""
    import torch
    raw = ws[: B * H * n_ck * 64 * 64 * 4].view(torch.float32).view(B, H, n_ck, 4096)
    raw = raw.double().cpu().numpy()
    i = np.arange(64)[:, None]
    j = np.arange(64)[None, :]
    off = (i // 16) * 1024 + (j // 8) * 128 + (4 * (i % 8) + (j % 8) // 2) * 4 + 2 * ((i // 8) % 2) + j % 2
    assert len(np.unique(off)) == 4096
    return raw[..., off]

