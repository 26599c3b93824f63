"""GPU parity of the WKV epilogue (per-head GroupNorm, bonus term, output gating) against the epilogue
oracle, alone and composed with the recurrence: forward y -> out, and backward dout -> an fp32 block
(dy for the recurrence's backward, then the bonus parts of dr, dk, dv, which that backward adds to
its own: WKV7_FLAG_EPILOGUE_GRADS) -- including a head that the chunked backward hands to the exact
re-run.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from oracle import epilogue as E
from linear_recurrent_lm_b200 import inputs as I
from tests.gpu_util import f64, inputs_dev, inputs_f64, to_dev
from tests.metrics import cosine, err_rms, err_rms_excess

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2, "f16": 5e-3}
EPS = 64e-5


@pytest.fixture(scope="module")
def W():
    import torch
    from linear_recurrent_lm_b200 import wkv7
    torch.cuda.set_device(0)
    return wkv7


def _params(rng, H):
    ln_w = (1.0 + 0.3 * rng.standard_normal((H, 64))).astype(np.float32)
    ln_b = (0.2 * rng.standard_normal((H, 64))).astype(np.float32)
    r_k = (0.5 * rng.standard_normal((H, 64))).astype(np.float32)
    return ln_w, ln_b, r_k


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("shape", [(1, 1, 1), (2, 37, 3), (3, 200, 12)])
def test_epilogue_alone(W, dtype, shape):
    """out, and every gradient of the epilogue, from the same stored inputs as the oracle's."""
    B, T, H = shape
    rng = np.random.default_rng(7 + T)
    x = {n: I.to_storage(rng.standard_normal((B, T, H, 64)) * (3.0 if n == "y" else 1.0), dtype)
         for n in ("y", "r", "k", "v", "g", "dout")}
    ln_w, ln_b, r_k = _params(rng, H)
    xd = {n: to_dev(x[n]) for n in x}
    pd = [to_dev(a) for a in (ln_w, ln_b, r_k)]
    out = W.epilogue_forward(xd["y"], xd["r"], xd["k"], xd["v"], xd["g"], *pd, EPS)
    xo = {n: I.to_f64(x[n]) for n in x}
    oo, _, _ = E.forward(xo["y"], xo["r"], xo["k"], xo["v"], xo["g"], ln_w, ln_b, r_k, EPS)
    assert err_rms_excess(f64(out), oo, dtype) <= TOL[dtype]
    g = W.epilogue_backward(xd["y"], xd["r"], xd["k"], xd["v"], xd["g"], xd["dout"], *pd, EPS)
    go = E.backward(xo["dout"], xo["y"], xo["r"], xo["k"], xo["v"], xo["g"], ln_w, ln_b, r_k, EPS)
    assert err_rms_excess(f64(g["dg"]), go["dg"], dtype) <= TOL[dtype]
    for m, n in enumerate(("dy", "dr", "dk", "dv")):      # fp32 parts of the block
        assert err_rms(f64(g["eg"][m]), go[n]) <= 1e-4, n
    for n, m in (("dln_w", "dgamma"), ("dln_b", "dbeta"), ("dr_k", "drk")):
        assert err_rms(f64(g[n]), go[m]) <= 1e-4, n   # fp32 sums of the same stored values


def _compose_oracle(d, dy_out, g, params, reset, s0, y_stored):
    """The oracle's backward through the epilogue and the recurrence, in fp64.  The epilogue's input
    is y as the forward stores it (the value at this boundary; the forward's own y is held to the
    fp64 oracle by the forward tests)."""
    args = inputs_f64(d)
    y = y_stored
    r, k, v = args[0], args[2], args[3]
    out, _, _ = E.forward(y, r, k, v, g, *params, EPS)
    ge = E.backward(dy_out, y, r, k, v, g, *params, EPS)
    gr, _ = oracle.backward(*args, ge["dy"], s0=s0, reset=reset)
    grads = {n: gr[n] for n in ("dw", "da", "db")}
    for n in ("dr", "dk", "dv"):
        grads[n] = gr[n] + ge[n]
    grads["dg"], grads["ds0"] = ge["dg"], gr["ds0"]
    return out, grads


@pytest.mark.parametrize("algo", ("scan", "chunked_fused", "chunked_split"))
@pytest.mark.parametrize("flag_a_head", (False, True))
def test_recurrence_and_epilogue_composed(W, algo, flag_a_head):
    """y -> out and dout -> every gradient through both stages, against the oracle composed in fp64.
    With ``flag_a_head`` one head holds a decay below 1/16 in a late chunk: the chunked backward
    stops there and the exact re-run recomputes that head, the epilogue's parts included."""
    import torch
    rng = np.random.default_rng(31 if flag_a_head else 30)
    B, T, H = 2, 200, 3
    d = I.draw_inputs(rng, (B, T, H, 64), "bf16")
    if flag_a_head:
        w = I.to_f64(d["w"])
        w[1, 170, 2, :6] = 0.03
        d["w"] = I.to_storage(w, "bf16")
    gate = I.to_storage(rng.standard_normal((B, T, H, 64)), "bf16")
    dout = I.to_storage(rng.standard_normal((B, T, H, 64)), "bf16")
    s0 = rng.standard_normal((B, H, 64, 64)).astype(np.float32)
    reset = np.zeros((B, T), np.uint8)
    reset[0, 77] = 1
    params = _params(rng, H)
    xs = inputs_dev(d)
    gd, dod, s0d, rd = to_dev(gate), to_dev(dout), to_dev(s0), to_dev(reset)
    pd = [to_dev(a) for a in params]
    y, _, ws = W.forward(*xs, s0=s0d, reset=rd, algo=algo)
    out = W.epilogue_forward(y, xs[0], xs[2], xs[3], gd, *pd, EPS)
    ge = W.epilogue_backward(y, xs[0], xs[2], xs[3], gd, dod, *pd, EPS)
    g = W.backward(*xs, ge["eg"], ws, s0=s0d, reset=rd, algo=algo)
    if flag_a_head and algo != "scan":
        n_ck = B * H * ((T + 15) // 16) * 64 * 64 * 4
        marks = ws[n_ck:n_ck + 4 * B * H].view(torch.int32).cpu().numpy()
        assert marks[1 * H + 2] > 1 and (marks != 0).sum() == 1   # stopped after finishing late chunks
    yo, _, _ = oracle.forward(*inputs_f64(d), s0=s0.astype(np.float64), reset=reset)
    assert err_rms_excess(f64(y), yo, "bf16") <= 2e-2          # the stored y itself
    oo, go = _compose_oracle(d, I.to_f64(dout), I.to_f64(gate), params, reset, s0.astype(np.float64), f64(y))
    assert err_rms_excess(f64(out), oo, "bf16") <= 2e-2
    for n in ("dr", "dw", "dk", "dv", "da", "db"):
        e = err_rms_excess(f64(g[n]), go[n], "bf16")
        assert e <= 2e-2 and cosine(f64(g[n]), go[n]) >= 0.999, (n, e)
    assert err_rms_excess(f64(ge["dg"]), go["dg"], "bf16") <= 2e-2
    assert err_rms(f64(g["ds0"]), go["ds0"]) <= 2e-2


@pytest.mark.parametrize("algo", ("chunked_fused", "chunked_split", "scan", "auto"))
@pytest.mark.parametrize("want_y", (True, False))
@pytest.mark.parametrize("T", (40, 333))
def test_forward_with_fused_epilogue(W, algo, want_y, T):
    """wkv7_forward_epilogue: out is bit for bit the epilogue of the stored y (fused into the chunked
    forward's y write-out, or the two kernels back to back), y and s_out equal the plain forward's;
    a head with a decay out of the 1/L range takes the token path inside the fused kernel."""
    import torch
    rng = np.random.default_rng(400 + T)
    B, H = 2, 5
    d = I.draw_inputs(rng, (B, T, H, 64), "bf16")
    w = I.to_f64(d["w"])
    w[1, T // 2, 3, :4] = 0.0                   # one chunk of one head runs token by token
    d["w"] = I.to_storage(w, "bf16")
    gate = to_dev(I.to_storage(rng.standard_normal((B, T, H, 64)), "bf16"))
    s0 = to_dev(rng.standard_normal((B, H, 64, 64)).astype(np.float32))
    reset = np.zeros((B, T), np.uint8)
    reset[0, 21] = 1
    rd = to_dev(reset)
    pd = [to_dev(a) for a in _params(rng, H)]
    xs = inputs_dev(d)
    y, s, _ = W.forward(*xs, s0=s0, reset=rd, algo=algo)
    ref = W.epilogue_forward(y, xs[0], xs[2], xs[3], gate, *pd, EPS)
    out, y2, s2, _ = W.forward_epilogue(*xs, gate, *pd, EPS, s0=s0, reset=rd, algo=algo, want_y=want_y)
    assert torch.equal(out, ref)
    assert torch.equal(s2, s)
    if want_y:
        assert torch.equal(y2, y)
    yo, _, _ = oracle.forward(*inputs_f64(d), s0=f64(s0), reset=reset)
    oo, _, _ = E.forward(f64(y), *(inputs_f64(d)[i] for i in (0, 2, 3)), f64(gate), *(f64(t) for t in pd), EPS)
    assert err_rms_excess(f64(out), oo, "bf16") <= 2e-2
    assert err_rms_excess(f64(y), yo, "bf16") <= 2e-2
