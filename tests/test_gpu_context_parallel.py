"""GPU parity of context parallelism (the tokens of every row split into consecutive segments)
on one device: every rank's phases run in turn through the library's kernels (the forward and
backward of each segment and ``wkv7_state_compose``), the gathers replaced by lists, and the
result held to the oracle's single run over the whole sequence -- y of every segment, the final
state, every gradient and the sequence's ds0 -- with resets (one on a segment's first token), an
initial state and a final-state gradient.  The composition kernel itself is held to an fp64 matrix
product.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from linear_recurrent_lm_b200 import inputs as I
from tests.gpu_util import f64, to_dev
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


@pytest.mark.parametrize("N", [64, 128])
@pytest.mark.parametrize("transpose", [False, True])
def test_state_compose(W, N, transpose):
    import torch
    rng = np.random.default_rng(700 + N)
    B, H = 3, 5
    S, P, U = (rng.standard_normal((B, H, N, N)).astype(np.float32) for _ in range(3))
    Sd, Pd, Ud = to_dev(S), to_dev(P), to_dev(U)
    PP = np.swapaxes(P, -1, -2) if transpose else P
    ref = S.astype(np.float64) @ PP.astype(np.float64) + U
    out = W.state_compose(Sd, Pd, Ud, transpose=transpose)
    assert err_rms(f64(out), ref) <= 1e-5
    assert torch.equal(W.state_compose(None, None, Ud), Ud)                   # S = 0: out = U
    no_u = W.state_compose(Sd, Pd, None, transpose=transpose)
    assert err_rms(f64(no_u), S.astype(np.float64) @ PP) <= 1e-5
    W.state_compose(Sd, Pd, Ud, out=Ud, transpose=transpose)                   # in place on U
    assert torch.equal(Ud, out)


def _problem(B, T, H, dtype, seed, log_decay=False):
    rng = np.random.default_rng(seed)
    d = I.draw_inputs(rng, (B, T, H, 64), dtype, log_decay=log_decay)
    dy = I.to_storage(rng.standard_normal((B, T, H, 64)), dtype)
    s0 = rng.standard_normal((B, H, 64, 64)).astype(np.float32)
    dsT = rng.standard_normal((B, H, 64, 64)).astype(np.float32)
    reset = np.zeros((B, T), np.uint8)
    reset[0, T // 3] = 1
    return d, dy, s0, dsT, reset


def _run_cp(d, dy, s0, dsT, reset, world, algo, log_decay=False):
    import torch
    from linear_recurrent_lm_b200 import context_parallel as cp
    T = d["r"].shape[1]
    bounds = cp.split_tokens(T, world)
    segs, dys = [], []
    for p in range(world):
        t0, t1 = bounds[p], bounds[p + 1]
        segs.append(cp.Segment([to_dev(np.ascontiguousarray(d[n][:, t0:t1])) for n in I.NAMES],
                               to_dev(np.ascontiguousarray(reset[:, t0:t1]))))
        dys.append(to_dev(np.ascontiguousarray(dy[:, t0:t1])))
    ys, ends, ctxs = cp.emulate_forward(segs, to_dev(s0), algo=algo, log_decay=log_decay)
    gs = cp.emulate_backward(ctxs, dys, to_dev(dsT))
    y = torch.cat(ys, dim=1)
    g = {n: torch.cat([gp[n] for gp in gs], dim=1) for n in GRADS}
    g["ds0"] = gs[0]["ds0"]
    return y, ends[-1], g, bounds


def _check(d, dy, s0, dsT, reset, y, s, g, dtype, log_decay=False):
    args = [I.to_f64(d[n]) for n in I.NAMES]
    yo, so, _ = oracle.forward(*args, s0=s0, reset=reset, log_decay=log_decay)
    go, _ = oracle.backward(*args, I.to_f64(dy), s0=s0, reset=reset, dsT=dsT, log_decay=log_decay)
    tol = TOL[dtype]
    errs = {"y": err_rms_excess(f64(y), yo, dtype), "s_out": err_rms(f64(s), so),
            "ds0": err_rms(f64(g["ds0"]), go["ds0"])}
    for n in GRADS:
        errs[n] = err_rms_excess(f64(g[n]), go[n], dtype)
        assert cosine(f64(g[n]), go[n]) >= 0.999, n
    bad = {k: v for k, v in errs.items() if v > tol}
    assert not bad, bad
    return errs


@pytest.mark.parametrize("world", [2, 3, 4])
@pytest.mark.parametrize("algo,dtype", [("auto", "bf16"), ("chunked_fused", "f16"), ("scan", "f32")])
def test_context_parallel_matches_one_run(W, world, algo, dtype):
    d, dy, s0, dsT, reset = _problem(2, 300, 3, dtype, 710 + world)
    reset[1, [160, 112, 80]] = 1          # first tokens of segments: 2 segments at 160, 3 at 112, 4 at 80
    y, s, g, _ = _run_cp(d, dy, s0, dsT, reset, world, algo)
    _check(d, dy, s0, dsT, reset, y, s, g, dtype)


def test_context_parallel_log_decay(W):
    d, dy, s0, dsT, reset = _problem(2, 200, 2, "bf16", 720, log_decay=True)
    y, s, g, _ = _run_cp(d, dy, s0, dsT, reset, 3, "auto", log_decay=True)
    _check(d, dy, s0, dsT, reset, y, s, g, "bf16", log_decay=True)


def test_context_parallel_packed_batch_all_units(W):
    """The packed training batch (B=8, T=4096, H=32, documents with resets) split over 4 segments
    of 1024 tokens, every (b, h) unit against the oracle's single run."""
    wl = I.make_workload(3)
    rng = np.random.default_rng(730)
    s0 = np.zeros((wl.B, wl.H, 64, 64), np.float32)
    dsT = rng.standard_normal((wl.B, wl.H, 64, 64)).astype(np.float32)
    y, s, g, _ = _run_cp(wl.inputs, wl.dy, s0, dsT, wl.reset, 4, "auto")
    errs = _check(wl.inputs, wl.dy, s0, dsT, wl.reset, y, s, g, "bf16")
    print("context parallel, 4 segments, packed batch: " + ", ".join(f"{k} {v:.4f}" for k, v in errs.items()))
