"""GPU backward parity against the CPU oracle's hand-derived reverse mode.

Every gradient and dS0 is held element by element: max|gpu - oracle| / RMS(oracle) after the
half-ulp that storing the result in the output dtype costs (``err_rms_excess``) must stay within the
bound of the input dtype (f32 1e-4, bf16 2e-2, f16 5e-3), and the fp64 cosine of each whole tensor
must reach 0.999.  The full-size packed batch is compared on all of its (b,h) units.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from linear_recurrent_lm_b200 import inputs as I
from tests.gpu_util import f64, inputs_dev, inputs_f64, to_dev
from tests.metrics import cosine, err_rms, err_rms_excess

pytestmark = pytest.mark.gpu

GRADS = ("dr", "dw", "dk", "dv", "da", "db")
TOL = {"f32": 1e-4, "bf16": 2e-2, "f16": 5e-3}
COS = 0.999


@pytest.fixture(scope="module")
def W():
    import torch
    from linear_recurrent_lm_b200 import wkv7
    torch.cuda.set_device(0)
    return wkv7


def fwd_bwd(W, d, dy, s0=None, reset=None, dsT=None, algo="auto"):
    xs = inputs_dev(d)
    s0d = None if s0 is None else to_dev(s0)
    rd = None if reset is None else to_dev(reset)
    y, s, ws = W.forward(*xs, s0=s0d, reset=rd, algo=algo)
    g = W.backward(*xs, to_dev(dy), ws, s0=s0d, reset=rd, dsT=None if dsT is None else to_dev(dsT), algo=algo)
    return y, s, g


def grad_errors(g, go, dtype):
    """{name: (err_rms_excess, cosine)} for the six gradients (output dtype) and dS0 (fp32)."""
    out = {}
    for n in GRADS:
        x = f64(g[n])
        out[n] = (err_rms_excess(x, go[n], dtype), cosine(x, go[n]))
    if g.get("ds0") is not None and "ds0" in go:
        x = f64(g["ds0"])
        out["ds0"] = (err_rms(x, go["ds0"]), cosine(x, go["ds0"]))
    return out


def check_grads(g, go, dtype, where=""):
    errs = grad_errors(g, go, dtype)
    bad = {n: e for n, e in errs.items() if not (e[0] <= TOL[dtype] and e[1] >= COS)}
    assert not bad, (where, bad)
    return errs


@pytest.mark.parametrize("algo", ("scan", "chunked_fused", "chunked_split"))
def test_config1_fwd_bwd(W, algo):
    """184M-model layer shape: B=2, T=512, H=12, bf16, checkpoint every 16 tokens."""
    wl = I.make_workload(1)
    _, _, g = fwd_bwd(W, wl.inputs, wl.dy, algo=algo)
    go, _ = oracle.backward(*inputs_f64(wl.inputs), I.to_f64(wl.dy))
    check_grads(g, go, "bf16", algo)


@pytest.fixture(scope="module")
def config3_oracle():
    """Workload 3 (B=8, T=4096, H=32, packed documents): the oracle's gradients of every unit."""
    wl = I.make_workload(3)
    go, _ = oracle.backward(*inputs_f64(wl.inputs), I.to_f64(wl.dy), reset=wl.reset)
    return wl, go


@pytest.mark.parametrize("algo", ("chunked_fused", "chunked_split", "scan"))
def test_config3_full_size_all_units(W, config3_oracle, algo):
    """B=8, T=4096, H=32 packed documents with resets: all 256 (b,h) units, every element."""
    wl, go = config3_oracle
    _, _, g = fwd_bwd(W, wl.inputs, wl.dy, reset=wl.reset, algo=algo)
    errs = check_grads(g, go, "bf16", algo)
    print(f"config3 {algo}: " + ", ".join(f"{n} {e[0]:.4f}/{e[1]:.6f}" for n, e in errs.items()))


def _ragged_cases():
    return [(a, dt) for a in ("scan", "chunked_fused", "chunked_split")
            for dt in ("f32", "bf16", "f16") if not (dt == "f32" and a != "scan")]


@pytest.mark.parametrize("algo,dtype", _ragged_cases())
@pytest.mark.parametrize("T", [1, 15, 17, 40, 100])
def test_ragged_with_state_resets_and_dsT(W, algo, dtype, T):
    rng = np.random.default_rng(100 + T)
    B, H = 2, 3
    d = I.draw_inputs(rng, (B, T, H, 64), dtype)
    dy = I.to_storage(rng.standard_normal((B, T, H, 64)), dtype)
    s0 = rng.standard_normal((B, H, 64, 64)).astype(np.float32)
    dsT = rng.standard_normal((B, H, 64, 64)).astype(np.float32)
    reset = np.zeros((B, T), np.uint8)
    reset[1, 0] = 1
    for t in (5, 6, 16, T - 1):
        if 0 < t < T:
            reset[0, t] = 1
    _, _, g = fwd_bwd(W, d, dy, s0=s0, reset=reset, dsT=dsT, algo=algo)
    go, _ = oracle.backward(*inputs_f64(d), I.to_f64(dy), s0=s0, reset=reset, dsT=dsT)
    check_grads(g, go, dtype, (algo, dtype, T))
    # row 1 is reset at t=0: nothing reaches s0
    assert np.all(f64(g["ds0"])[1] == 0.0)


@pytest.mark.parametrize("algo", ("scan", "chunked_fused", "chunked_split"))
def test_small_decay_segments(W, algo):
    """Decays far below the generator's range (prod w < 2^-16 over a chunk) and w = 0: the chunked
    backward hands those heads to the exact scan, whose results must still hold the bound."""
    rng = np.random.default_rng(7)
    dt = "f32" if algo == "scan" else "bf16"
    d = I.draw_inputs(rng, (1, 64, 2, 64), dt)
    w = I.to_f64(d["w"])
    w[:, 10:26] *= 0.2
    w[:, 40:42] = 0.0
    d["w"] = I.to_storage(w, dt)
    dy = I.to_storage(rng.standard_normal((1, 64, 2, 64)), dt)
    _, _, g = fwd_bwd(W, d, dy, algo=algo)
    go, _ = oracle.backward(*inputs_f64(d), I.to_f64(dy))
    check_grads(g, go, dt, algo)


def test_flagged_and_chunked_heads_in_one_batch(W):
    """bf16 batch where some (b, h) heads hold a decay the 1/L scaling cannot take (w = 0 or
    w < 1/16 inside a chunk) and the rest do not: the chunked pass marks exactly those heads, the
    exact scan redoes them, and every head's gradients and dS0 must match the oracle."""
    rng = np.random.default_rng(17)
    B, T, H = 2, 200, 3
    d = I.draw_inputs(rng, (B, T, H, 64), "bf16")
    w = I.to_f64(d["w"])
    w[0, 70:72, 1] = 0.0            # head (0, 1): w = 0 in chunk 4
    w[1, 150, 2, :8] = 0.03         # head (1, 2): w < 1/16 in chunk 9
    d["w"] = I.to_storage(w, "bf16")
    dy = I.to_storage(rng.standard_normal((B, T, H, 64)), "bf16")
    reset = np.zeros((B, T), np.uint8)
    reset[0, 120] = 1
    s0 = rng.standard_normal((B, H, 64, 64)).astype(np.float32)
    dsT = rng.standard_normal((B, H, 64, 64)).astype(np.float32)
    _, _, g = fwd_bwd(W, d, dy, s0=s0, reset=reset, dsT=dsT)
    go, _ = oracle.backward(*inputs_f64(d), I.to_f64(dy), s0=s0.astype(np.float64), reset=reset,
                            dsT=dsT.astype(np.float64))
    check_grads(g, go, "bf16")
    for b in range(B):
        for h in range(H):
            for n in GRADS:
                assert cosine(f64(g[n])[b, :, h], go[n][b, :, h]) >= COS, (b, h, n)
            assert cosine(f64(g["ds0"])[b, h], go["ds0"][b, h]) >= COS, (b, h, "ds0")


def test_backward_chaining(W):
    """dS0 of the second half fed as dS_T of the first equals one backward over the whole row, bit for
    bit: the split falls on a chunk boundary, so both run the same arithmetic on the same fp32 state
    and carried gradient."""
    import torch
    wl = I.make_workload(1, B=1, T=96, H=2)
    xs = inputs_dev(wl.inputs)
    dy = to_dev(wl.dy)
    _, _, ws = W.forward(*xs)
    g = W.backward(*xs, dy, ws)
    first = [x[:, :48].contiguous() for x in xs]
    second = [x[:, 48:].contiguous() for x in xs]
    _, s1, ws1 = W.forward(*first)
    _, _, ws2 = W.forward(*second, s0=s1)
    g2 = W.backward(*second, dy[:, 48:].contiguous(), ws2, s0=s1)
    g1 = W.backward(*first, dy[:, :48].contiguous(), ws1, dsT=g2["ds0"])
    for n in GRADS:
        joined = torch.cat([g1[n], g2[n]], dim=1)
        assert torch.equal(joined, g[n]), n


def test_backward_is_deterministic(W):
    import torch
    wl = I.make_workload(1)
    _, _, g1 = fwd_bwd(W, wl.inputs, wl.dy)
    _, _, g2 = fwd_bwd(W, wl.inputs, wl.dy)
    assert all(torch.equal(g1[n], g2[n]) for n in GRADS + ("ds0",))
