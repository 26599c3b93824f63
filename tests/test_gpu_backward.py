"""GPU backward parity against the CPU oracle's hand-derived reverse mode."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from linear_recurrent_lm_b200 import inputs as I
from tests.gpu_util import f64, inputs_dev, inputs_f64, sample_units, to_dev
from tests.metrics import cosine

pytestmark = pytest.mark.gpu

GRADS = ("dr", "dw", "dk", "dv", "da", "db")
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


def check_grads(g, go, sl=slice(None)):
    out = {}
    for n in GRADS:
        out[n] = cosine(f64(g[n])[sl], go[n])
    if "ds0" in go and g.get("ds0") is not None:
        out["ds0"] = cosine(f64(g["ds0"])[sl[:1] + sl[2:3] if isinstance(sl, tuple) else sl], go["ds0"])
    bad = {k: v for k, v in out.items() if not v >= COS}
    assert not bad, bad
    return out


@pytest.mark.parametrize("algo", ("scan", "chunked_fused", "chunked_split"))
def test_config1_fwd_bwd(W, algo):
    """184M-model layer shape: B=2, T=512, H=12, bf16, checkpoint every 16 tokens."""
    wl = I.make_workload(1)
    _, _, g = fwd_bwd(W, wl.inputs, wl.dy, algo=algo)
    go, _ = oracle.backward(*inputs_f64(wl.inputs), I.to_f64(wl.dy))
    check_grads(g, go)


@pytest.mark.parametrize("algo", ("scan", "chunked_fused", "chunked_split"))
def test_config3_full_size_sampled_units(W, algo):
    """B=8, T=4096, H=32 packed documents with resets, gradients of sampled units."""
    wl = I.make_workload(3)
    _, _, g = fwd_bwd(W, wl.inputs, wl.dy, reset=wl.reset, algo=algo)
    gg = {n: f64(g[n]) for n in GRADS}
    for (b, h) in sample_units(8, 32, 6, seed=4):
        part = {n: wl.inputs[n][b:b + 1, :, h:h + 1] for n in I.NAMES}
        go, _ = oracle.backward(*inputs_f64(part), I.to_f64(wl.dy[b:b + 1, :, h:h + 1]), reset=wl.reset[b:b + 1])
        for n in GRADS:
            c = cosine(gg[n][b:b + 1, :, h:h + 1], go[n])
            assert c >= COS, ((b, h), n, c)


@pytest.mark.parametrize("algo,dtype", [(a, dt) for a in ("scan", "chunked_fused", "chunked_split")
                                         for dt in ("f32", "bf16", "f16") if not (dt == "f32" and a != "scan")])
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
    for n in GRADS + ("ds0",):
        c = cosine(f64(g[n]), go[n])
        assert c >= COS, (n, c)
    # row 1 is reset at t=0: nothing reaches s0
    assert np.all(f64(g["ds0"])[1] == 0.0)


@pytest.mark.parametrize("algo", ("scan", "chunked_fused", "chunked_split"))
def test_small_decay_segments(W, algo):
    """Decays far below the generator's range (prod w < 2^-16 over a chunk) and w = 0."""
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
    for n in GRADS + ("ds0",):
        c = cosine(f64(g[n]), go[n])
        assert c >= COS, (n, c)


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
    for b in range(B):
        for h in range(H):
            for n in GRADS:
                c = cosine(f64(g[n])[b, :, h], go[n][b, :, h])
                assert c >= COS, (b, h, n, c)
            c = cosine(f64(g["ds0"])[b, h], go["ds0"][b, h])
            assert c >= COS, (b, h, "ds0", c)


def test_backward_chaining(W):
    """dS0 of the second half fed as dS_T of the first equals one backward over the whole row."""
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
        assert cosine(f64(joined), f64(g[n])) >= 0.99999, n


def test_backward_is_deterministic(W):
    import torch
    wl = I.make_workload(1)
    _, _, g1 = fwd_bwd(W, wl.inputs, wl.dy)
    _, _, g2 = fwd_bwd(W, wl.inputs, wl.dy)
    assert all(torch.equal(g1[n], g2[n]) for n in GRADS + ("ds0",))
