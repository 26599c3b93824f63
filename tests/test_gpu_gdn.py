"""GPU parity of the N = 128 heads and the gated-DeltaNet front end (rwkv-lab page, "Highlight result
-- GDN in RWKV-7"): the token-order forward and the decode step at N = 128 against the oracle; the
map (wkv7_gdn_map) against the map oracle; and a GDN layer run as map -> recurrence against the
gated delta rule written in its own form, on the page's head geometry (value heads sharing key
heads), with ragged lengths, resets, an initial state, and decode steps.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from oracle import gdn as G
from linear_recurrent_lm_b200 import inputs as I
from tests.gpu_util import f64, inputs_dev, inputs_f64, sample_units, to_dev
from tests.metrics import cosine, err_rms, err_rms_excess

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2, "f16": 5e-3}
MAP_OUT = ("r", "x", "kw", "a", "b")


@pytest.fixture(scope="module")
def W():
    import torch
    from linear_recurrent_lm_b200 import wkv7
    torch.cuda.set_device(0)
    return wkv7


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("T", [1, 16, 45])
@pytest.mark.parametrize("log_decay", [False, True])
def test_scan_forward_n128(W, dtype, T, log_decay):
    """y, s_out and every 16-token checkpoint (row-major at N = 128) against the oracle."""
    import torch
    rng = np.random.default_rng(600 + T)
    B, H, N = 2, 3, 128
    d = I.draw_inputs(rng, (B, T, H, N), dtype, log_decay=log_decay)
    s0 = rng.normal(0.0, 0.5, (B, H, N, N)).astype(np.float32)
    reset = np.zeros((B, T), np.uint8)
    if T > 6:
        reset[1, T // 2] = 1
    y, s, ws = W.forward(*inputs_dev(d), s0=to_dev(s0), reset=to_dev(reset), algo="auto", log_decay=log_decay)
    assert y.shape == (B, T, H, N) and s.shape == (B, H, N, N)
    args = inputs_f64(d)
    yo, so, _ = oracle.forward(*args, s0=s0, reset=reset, log_decay=log_decay)
    assert err_rms_excess(f64(y), yo, dtype) <= TOL[dtype]
    assert err_rms(f64(s), so) <= TOL[dtype]
    n_ck = (T + 15) // 16
    ck = f64(ws[:B * H * n_ck * N * N * 4].view(torch.float32).view(B, H, n_ck, N, N))
    for c in range(n_ck):                   # checkpoint c: the state after token min(16(c+1), T) - 1
        te = min(16 * (c + 1), T)
        _, sc, _ = oracle.forward(*(x[:, :te] for x in args), s0=s0, reset=reset[:, :te], log_decay=log_decay)
        assert err_rms(ck[:, :, c], sc) <= TOL[dtype], c


def test_chunked_forms_refuse_n128(W):
    import torch
    x = torch.zeros((1, 16, 1, 128), device="cuda", dtype=torch.bfloat16)
    for algo in ("chunked", "chunked_fused", "chunked_split"):
        with pytest.raises(W.WKV7Error) as e:
            W.forward(x, x, x, x, x, x, algo=algo)
        assert e.value.status == W.ERR_UNSUPPORTED


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_steps_n128(W, dtype):
    """Ragged decode steps at N = 128 against the oracle stepped alongside; finished rows keep
    their state bit for bit and get y = 0."""
    import torch
    rng = np.random.default_rng(610)
    B, H, N, steps = 20, 3, 128, 10
    state = rng.normal(0.0, 0.1, (B, H, N, N)).astype(np.float32)
    st_d = to_dev(state)
    st_o = state.astype(np.float64)
    lengths = rng.integers(1, steps + 1, B)
    for s in range(steps):
        d = I.draw_inputs(rng, (B, H, N), dtype)
        act = (lengths > s).astype(np.uint8)
        before = st_d.clone()
        y = W.step(*(to_dev(d[n]) for n in I.NAMES), st_d, to_dev(act))
        yo, st_o = oracle.step(*(I.to_f64(d[n]) for n in I.NAMES), st_o, act)
        assert err_rms_excess(f64(y), yo, dtype) <= TOL[dtype], s
        idle = torch.from_numpy(act == 0).cuda()
        assert torch.equal(st_d[idle], before[idle]) and not y[idle].any()
    assert err_rms(f64(st_d), st_o) <= TOL[dtype]


def _gdn_case(rng, B, T, H, Hk, N, dtype):
    d = I.draw_gdn_inputs(rng, B, T, H, Hk, N, dtype)
    dev = {n: to_dev(d[n]) for n in ("q", "k", "v", "g", "beta")}
    return d, dev


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("N,H,Hk", [(128, 4, 2), (128, 3, 3), (64, 6, 1)])
def test_gdn_map(W, dtype, N, H, Hk):
    """Every output of the map against the map oracle applied to the same stored q, k, g, beta;
    x = -inf exactly where g = 0."""
    rng = np.random.default_rng(620 + N + H)
    B, T = 2, 37
    d, dev = _gdn_case(rng, B, T, H, Hk, N, dtype)
    d["g"][0, 5, 0] = 0.0
    dev["g"] = to_dev(d["g"])
    m = W.gdn_map(dev["q"], dev["k"], dev["g"], dev["beta"], H, eps=1e-6)
    mo = G.gdn_map(I.to_f64(d["q"]), I.to_f64(d["k"]), d["g"], d["beta"], H, 1e-6, N ** -0.5)
    xg = f64(m["x"])
    assert np.all(xg[0, 5, 0] == -np.inf)
    fin = np.isfinite(mo["x"])
    for n in MAP_OUT:
        got, ref = f64(m[n]), mo[n]
        if n == "x":
            got, ref = got[fin], ref[fin]
        assert err_rms_excess(got, ref, dtype) <= TOL[dtype], n


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_gdn_layer_through_the_recurrence(W, dtype):
    """A GDN layer as map -> forward (log-space decay, token-order scan): y against the oracle's
    forward on the map's stored outputs (the recurrence's parity bound), and against the gated
    delta rule on the stored q, k, v (cosine: the map's outputs are rounded to the dtype)."""
    rng = np.random.default_rng(630)
    B, T, H, Hk, N = 2, 150, 4, 2, 128
    d, dev = _gdn_case(rng, B, T, H, Hk, N, dtype)
    s0 = rng.normal(0.0, 0.3, (B, H, N, N)).astype(np.float32)
    m = W.gdn_map(dev["q"], dev["k"], dev["g"], dev["beta"], H, eps=1e-6)
    y, s, _ = W.forward(m["r"], m["x"], m["kw"], dev["v"], m["a"], m["b"], s0=to_dev(s0), log_decay=True)
    stored = [f64(m[n]) for n in ("r", "x", "kw")] + [I.to_f64(d["v"])] + [f64(m[n]) for n in ("a", "b")]
    yo, so, _ = oracle.forward(*stored, s0=s0, log_decay=True)
    assert err_rms_excess(f64(y), yo, dtype) <= TOL[dtype]
    assert err_rms(f64(s), so) <= TOL[dtype]
    og, sg = G.gated_delta_rule(I.to_f64(d["q"]), I.to_f64(d["k"]), I.to_f64(d["v"]), d["g"], d["beta"], 1e-6,
                                N ** -0.5, s0=s0)
    floor = 0.9999 if dtype == "bf16" else 0.9999999
    assert cosine(f64(y), og) >= floor and cosine(f64(s), sg) >= floor


def test_gdn_decode_through_the_step(W):
    """GDN decode: the map at T = 1 and the N = 128 step, 12 tokens, against the gated delta rule."""
    rng = np.random.default_rng(640)
    B, H, Hk, N, steps = 4, 4, 2, 128, 12
    s0 = rng.normal(0.0, 0.3, (B, H, N, N)).astype(np.float32)
    st = to_dev(s0)
    d, dev = _gdn_case(rng, B, steps, H, Hk, N, "f32")
    ys = []
    for t in range(steps):
        one = {n: dev[n][:, t:t + 1].contiguous() for n in dev}
        m = W.gdn_map(one["q"], one["k"], one["g"], one["beta"], H, eps=1e-6)
        sq = {n: m[n][:, 0].contiguous() for n in MAP_OUT}
        ys.append(f64(W.step(sq["r"], sq["x"], sq["kw"], one["v"][:, 0].contiguous(), sq["a"], sq["b"], st,
                             log_decay=True)))
    og, sg = G.gated_delta_rule(d["q"], d["k"], d["v"], d["g"], d["beta"], 1e-6, N ** -0.5, s0=s0)
    y = np.stack(ys, axis=1)
    assert err_rms(y, og) <= 1e-4
    assert err_rms(f64(st), sg) <= 1e-4


def test_gdn_layer_full_size_sampled_units(W):
    """The GDN layer at full size (B=8, T=4096, 32 value heads over 16 key heads of 128, bf16) in
    the launch configuration the benchmark times, checked on sampled (b, h) units against the
    oracle's forward on the map's stored outputs, and on its map outputs everywhere by their
    invariants (|a| = 1 up to bf16, kw = -beta a)."""
    import torch
    rng = np.random.default_rng(650)
    B, T, H, Hk, N = 8, 4096, 32, 16, 128
    d, dev = _gdn_case(rng, B, T, H, Hk, N, "bf16")
    m = W.gdn_map(dev["q"], dev["k"], dev["g"], dev["beta"], H, eps=1e-6)
    y, s, _ = W.forward(m["r"], m["x"], m["kw"], dev["v"], m["a"], m["b"], log_decay=True, need_workspace=False)
    an = torch.linalg.vector_norm(m["a"].float(), dim=-1)
    assert float((an - 1).abs().max()) <= 3e-3
    kw_ref = -dev["beta"][..., None] * m["a"].float()
    assert float((m["kw"].float() - kw_ref).abs().max()) <= 8e-3
    for b, h in sample_units(B, H, 4, seed=3):
        one = lambda t: f64(t[b:b + 1, :, h:h + 1])   # noqa: E731
        args = [one(m["r"]), one(m["x"]), one(m["kw"]), I.to_f64(d["v"][b:b + 1, :, h:h + 1]), one(m["a"]),
                one(m["b"])]
        yo, so, _ = oracle.forward(*args, log_decay=True)
        assert err_rms_excess(one(y), yo, "bf16") <= 2e-2, (b, h)
        assert err_rms(f64(s[b:b + 1, h:h + 1]), so) <= 2e-2, (b, h)
