"""GPU parity of the log-space decay input (WKV7_FLAG_LOG_DECAY): the w tensor holds x, the kernels use
w = exp(-exp(x)), and the backward writes dL/dx into dw -- against the oracle run the same way.

Every form (scan, fused chunked, split chunked; forward, backward, decode step) on ragged lengths with resets, s0 and dS_T, and the packed full-size batch on all units; the
bounds are those of the input dtype (err_rms_excess; cosine >= 0.999 for the gradients).
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from linear_recurrent_lm_b200 import inputs as I
from tests.gpu_util import f64, inputs_dev, inputs_f64, to_dev
from tests.metrics import cosine, err_rms, err_rms_excess

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2, "f16": 5e-3}
GRADS = ("dr", "dw", "dk", "dv", "da", "db")


@pytest.fixture(scope="module")
def W():
    import torch
    from linear_recurrent_lm_b200 import wkv7
    torch.cuda.set_device(0)
    return wkv7


def _case(B, T, H, dtype, seed):
    rng = np.random.default_rng(seed)
    d = I.draw_inputs(rng, (B, T, H, 64), dtype, log_decay=True)
    dy = I.to_storage(rng.standard_normal((B, T, H, 64)), dtype)
    s0 = rng.standard_normal((B, H, 64, 64)).astype(np.float32)
    dsT = rng.standard_normal((B, H, 64, 64)).astype(np.float32)
    reset = np.zeros((B, T), np.uint8)
    if T > 6:
        reset[0, T // 3] = 1
    if B > 1:
        reset[1, 0] = 1
    return d, dy, s0, dsT, reset


def _check(W, d, dy, s0, dsT, reset, algo, dtype):
    xs = inputs_dev(d)
    y, s, ws = W.forward(*xs, s0=to_dev(s0), reset=to_dev(reset), algo=algo, log_decay=True)
    g = W.backward(*xs, to_dev(dy), ws, s0=to_dev(s0), reset=to_dev(reset), dsT=to_dev(dsT), algo=algo,
                   log_decay=True)
    args = inputs_f64(d)
    yo, so, _ = oracle.forward(*args, s0=s0, reset=reset, log_decay=True)
    go, _ = oracle.backward(*args, I.to_f64(dy), s0=s0, reset=reset, dsT=dsT, log_decay=True)
    tol = TOL[dtype]
    errs = {"y": err_rms_excess(f64(y), yo, dtype), "s_out": err_rms(f64(s), so)}
    for n in GRADS:
        errs[n] = err_rms_excess(f64(g[n]), go[n], dtype)
        assert cosine(f64(g[n]), go[n]) >= 0.999, (algo, dtype, n)
    errs["ds0"] = err_rms(f64(g["ds0"]), go["ds0"])
    bad = {k: v for k, v in errs.items() if v > tol}
    assert not bad, (algo, dtype, bad)
    return errs


def _cases():
    return [(a, dt) for a in ("scan", "chunked_fused", "chunked_split") for dt in ("f32", "bf16", "f16")
            if not (dt == "f32" and a != "scan")]


@pytest.mark.parametrize("algo,dtype", _cases())
@pytest.mark.parametrize("T", [1, 17, 40, 100])
def test_log_decay_ragged_with_resets(W, algo, dtype, T):
    d, dy, s0, dsT, reset = _case(2, T, 3, dtype, 500 + T)
    _check(W, d, dy, s0, dsT, reset, algo, dtype)


@pytest.mark.parametrize("algo", ("chunked_fused", "chunked_split", "scan"))
def test_log_decay_packed_batch_all_units(W, algo):
    """The packed training batch (B=8, T=4096, H=32, documents with resets) with x in place of w,
    every (b,h) unit, forward and backward."""
    wl = I.make_workload(3, log_decay=True)
    xs = inputs_dev(wl.inputs)
    y, s, ws = W.forward(*xs, reset=to_dev(wl.reset), algo=algo, log_decay=True)
    g = W.backward(*xs, to_dev(wl.dy), ws, reset=to_dev(wl.reset), algo=algo, log_decay=True)
    args = inputs_f64(wl.inputs)
    yo, so, _ = oracle.forward(*args, reset=wl.reset, log_decay=True)
    go, _ = oracle.backward(*args, I.to_f64(wl.dy), reset=wl.reset, log_decay=True)
    errs = {"y": err_rms_excess(f64(y), yo, "bf16"), "s_out": err_rms(f64(s), so)}
    for n in GRADS:
        errs[n] = err_rms_excess(f64(g[n]), go[n], "bf16")
        assert cosine(f64(g[n]), go[n]) >= 0.999, n
    print(f"log-decay config3 {algo}: " + ", ".join(f"{k} {v:.4f}" for k, v in errs.items()))
    assert max(errs.values()) <= 2e-2, errs


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_log_decay_decode_steps(W, dtype):
    """Ragged decode steps with x inputs against the oracle stepped alongside."""
    rng = np.random.default_rng(77)
    B, H, steps = 24, 4, 12
    state = rng.normal(0.0, 0.1, (B, H, 64, 64)).astype(np.float32)
    st_d = to_dev(state)
    st_o = state.astype(np.float64)
    lengths = rng.integers(1, steps + 1, B)
    for s in range(steps):
        d = I.draw_inputs(rng, (B, 1, H, 64), dtype, log_decay=True)
        act = (lengths > s).astype(np.uint8)
        y = W.step(*(to_dev(d[n][:, 0]) for n in I.NAMES), st_d, to_dev(act), log_decay=True)
        yo, st_o = oracle.step(*(I.to_f64(d[n][:, 0]) for n in I.NAMES), st_o, act, log_decay=True)
        assert err_rms_excess(f64(y), yo, dtype) <= TOL[dtype], s
    assert err_rms(f64(st_d), st_o) <= TOL[dtype]
