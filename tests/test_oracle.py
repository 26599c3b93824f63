"""Pins for the CPU oracle (no GPU).

The oracle is the plain definition of the WKV-7 recurrence; these tests tie it
to facts that do not come from the oracle itself: a hand-worked example,
closed forms of special cases (causal linear attention, retention, last-write),
the delta-rule overwrite property, the gated-delta-rule map printed on the
rwkv-lab page ("GDN subset of RWKV-7"), an independent dense matrix-product
form, linearity, reset/chaining identities and, for the backward, central
finite differences in fp64.
"""
from __future__ import annotations

import json
import os

import numpy as np
import pytest

import oracle
from oracle import numpy_twin
from linear_recurrent_lm_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rel(x, ref):
    x, ref = np.asarray(x), np.asarray(ref)
    return float(np.max(np.abs(x - ref)) / max(np.max(np.abs(ref)), 1e-300))


def gen(B, T, H, N, seed, *, s0=False, reset_p=0.0):
    """Generator-shaped fp64 inputs (recipe of the synthetic workloads) for general N."""
    rng = np.random.default_rng(seed)
    x = I.draw_inputs(rng, (B, T, H, N), "f32")
    x = {n: x[n].astype(np.float64) for n in I.NAMES}
    out = dict(x)
    out["s0"] = rng.standard_normal((B, H, N, N)) if s0 else None
    out["reset"] = (rng.random((B, T)) < reset_p).astype(np.uint8) if reset_p else None
    return out


def args(d):
    return [d[n] for n in I.NAMES]


# ------------------------------------------------------------------ worked example
def test_hand_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "worked_example_n2.json")))
    N = g["N"]
    toks = g["tokens"]
    T = len(toks)
    arr = {n: np.array([[t[n] for t in toks]], dtype=np.float64).reshape(1, T, 1, N) for n in I.NAMES}
    s0 = np.array(g["s0"], dtype=np.float64).reshape(1, 1, N, N)
    y, s, _ = oracle.forward(*args(arr), s0=s0)
    np.testing.assert_array_equal(y.reshape(T, N), np.array(g["expected_y"]))
    np.testing.assert_array_equal(s.reshape(N, N), np.array(g["expected_state"]))
    y2, s2 = numpy_twin.forward(*args(arr), s0=s0)
    np.testing.assert_array_equal(y2.reshape(T, N), np.array(g["expected_y"]))


# ------------------------------------------------------------------ two oracles
@pytest.mark.parametrize("N,reset_p,s0", [(64, 0.0, False), (64, 0.08, True), (8, 0.15, True)])
def test_c_and_numpy_twins_agree(N, reset_p, s0):
    d = gen(2, 41, 3, N, seed=7 + N, s0=s0, reset_p=reset_p)
    y, s, _ = oracle.forward(*args(d), s0=d["s0"], reset=d["reset"])
    y2, s2 = numpy_twin.forward(*args(d), s0=d["s0"], reset=d["reset"])
    assert rel(y, y2) < 1e-12 and rel(s, s2) < 1e-12
    rng = np.random.default_rng(3)
    dy = rng.standard_normal(y.shape)
    dsT = rng.standard_normal(s.shape)
    g, _ = oracle.backward(*args(d), dy, s0=d["s0"], reset=d["reset"], dsT=dsT)
    g2 = numpy_twin.backward(*args(d), dy, s0=d["s0"], reset=d["reset"], dsT=dsT)
    for n in g:
        assert rel(g[n], g2[n]) < 1e-12, n


# ------------------------------------------------------------------ closed forms
def test_running_sum_is_causal_linear_attention():
    """w=1, a=b=0: S_t = sum v k^T, so Y = tril(R K^T) V per head."""
    d = gen(2, 37, 2, 16, seed=11)
    d["w"][:] = 1.0
    d["a"][:] = 0.0
    d["b"][:] = 0.0
    y, s, _ = oracle.forward(*args(d))
    for b in range(2):
        for h in range(2):
            R, K, V = d["r"][b, :, h], d["k"][b, :, h], d["v"][b, :, h]
            ref = np.tril(R @ K.T) @ V
            assert rel(y[b, :, h], ref) < 1e-12
            assert rel(s[b, h], V.T @ K) < 1e-12


def test_zero_decay_keeps_last_write():
    """w=0, a=b=0: S_t = v_t k_t^T and y_t = (k_t . r_t) v_t."""
    d = gen(1, 9, 2, 8, seed=12, s0=True)
    d["w"][:] = 0.0
    d["a"][:] = 0.0
    d["b"][:] = 0.0
    y, s, _ = oracle.forward(*args(d), s0=d["s0"])
    ref = np.sum(d["k"] * d["r"], axis=-1, keepdims=True) * d["v"]
    assert rel(y, ref) < 1e-14
    assert rel(s[0, 1], np.outer(d["v"][0, -1, 1], d["k"][0, -1, 1])) < 1e-14


def test_scalar_decay_is_retention():
    """w = gamma (all channels), a=b=0: y_t = sum_{tau<=t} gamma^(t-tau) (r_t . k_tau) v_tau."""
    d = gen(1, 30, 1, 8, seed=13)
    g = 0.83
    d["w"][:] = g
    d["a"][:] = 0.0
    d["b"][:] = 0.0
    y, _, _ = oracle.forward(*args(d))
    R, K, V = d["r"][0, :, 0], d["k"][0, :, 0], d["v"][0, :, 0]
    t = np.arange(30)
    decay = np.where(t[:, None] >= t[None, :], g ** (t[:, None] - t[None, :]).clip(min=0), 0.0)
    assert rel(y[0, :, 0], ((R @ K.T) * decay) @ V) < 1e-12


def test_delta_rule_overwrites_key_slot():
    """w=1, a=-k, b=k, unit k: S_t = S_{t-1}(I - k k^T) + v k^T, hence S_t k_t = v_t exactly."""
    d = gen(1, 25, 2, 16, seed=14, s0=True)
    kh = d["k"] / np.linalg.norm(d["k"], axis=-1, keepdims=True)
    d["k"], d["a"], d["b"], d["w"][:] = kh, -kh, kh, 1.0
    d["r"] = kh                                   # read back through the key just written
    y, _, _ = oracle.forward(*args(d), s0=d["s0"])
    assert rel(y, d["v"]) < 1e-12


def test_gated_delta_rule_map():
    """The GDN map on the rwkv-lab page ("GDN subset of RWKV-7"): with unit q,k, scalar
    log-decay g and write strength beta, feeding r=q, w=exp(g), k=beta*k, a=-k,
    b=k*exp(g)*beta reproduces the gated delta rule
    S_t = alpha_t S_{t-1} (I - beta_t k k^T) + beta_t v k^T,  o_t = S_t q_t."""
    rng = np.random.default_rng(15)
    T, N = 33, 16
    q = rng.standard_normal((T, N)); q /= np.linalg.norm(q, axis=1, keepdims=True)
    k = rng.standard_normal((T, N)); k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, N))
    g = -np.abs(rng.standard_normal(T)) * 0.3
    beta = rng.uniform(0.1, 1.0, T)
    # gated delta rule, written in its own form
    S = np.zeros((N, N))
    o = np.zeros((T, N))
    for t in range(T):
        alpha = np.exp(g[t])
        S = alpha * S @ (np.eye(N) - beta[t] * np.outer(k[t], k[t])) + beta[t] * np.outer(v[t], k[t])
        o[t] = S @ q[t]
    sh = (1, T, 1, N)
    w = np.repeat(np.exp(g)[:, None], N, axis=1)
    y, _, _ = oracle.forward(q.reshape(sh), w.reshape(sh), (beta[:, None] * k).reshape(sh), v.reshape(sh),
                             (-k).reshape(sh), (k * (np.exp(g) * beta)[:, None]).reshape(sh))
    assert rel(y.reshape(T, N), o) < 1e-12


def test_identity_token_leaves_state_bitwise():
    """w=1, a=b=k=0: the state passes through unchanged (the padding semantics)."""
    d = gen(2, 7, 2, 64, seed=16, s0=True)
    d["w"][:] = 1.0
    d["a"][:] = 0.0
    d["b"][:] = 0.0
    d["k"][:] = 0.0
    _, s, _ = oracle.forward(*args(d), s0=d["s0"])
    np.testing.assert_array_equal(s, d["s0"])


def test_dense_product_form():
    """Independent formulation: S_T = S_0 prod_t G_t + sum_t v_t k_t^T prod_{s>t} G_s,
    G_t = diag(w_t) + a_t b_t^T, built as explicit N x N matrices."""
    d = gen(1, 23, 1, 64, seed=17, s0=True)
    _, s, _ = oracle.forward(*args(d), s0=d["s0"])
    T, N = 23, 64
    G = [np.diag(d["w"][0, t, 0]) + np.outer(d["a"][0, t, 0], d["b"][0, t, 0]) for t in range(T)]
    ref = d["s0"][0, 0].copy()
    for t in range(T):
        ref = ref @ G[t]
    for t in range(T):
        term = np.outer(d["v"][0, t, 0], d["k"][0, t, 0])
        for s_ in range(t + 1, T):
            term = term @ G[s_]
        ref = ref + term
    assert rel(s[0, 0], ref) < 1e-12


def test_linearity():
    """y is linear in (S_0, V) jointly and linear in r."""
    d = gen(1, 19, 2, 16, seed=18, s0=True)
    rng = np.random.default_rng(19)
    s0b = rng.standard_normal(d["s0"].shape)
    vb = rng.standard_normal(d["v"].shape)
    y1, _, _ = oracle.forward(*args(d), s0=d["s0"])
    d2 = dict(d); d2["v"] = vb
    y2, _, _ = oracle.forward(*args(d2), s0=s0b)
    d3 = dict(d); d3["v"] = 2.0 * d["v"] - 3.0 * vb
    y3, _, _ = oracle.forward(*args(d3), s0=2.0 * d["s0"] - 3.0 * s0b)
    assert rel(y3, 2.0 * y1 - 3.0 * y2) < 1e-11
    d4 = dict(d); d4["r"] = 2.5 * d["r"]
    y4, _, _ = oracle.forward(*args(d4), s0=d["s0"])
    assert rel(y4, 2.5 * y1) < 1e-14


# ------------------------------------------------------------------ reset / chaining
def test_reset_equals_fresh_call_and_packing():
    """Packed = concatenation of independent zero-state runs (state reset at each boundary)."""
    d = gen(1, 50, 2, 16, seed=20, s0=True)
    reset = np.zeros((1, 50), np.uint8)
    cuts = [0, 13, 14, 31, 50]
    for c in cuts[:-1]:
        reset[0, c] = 1
    y, s, _ = oracle.forward(*args(d), s0=d["s0"], reset=reset)
    for lo, hi in zip(cuts[:-1], cuts[1:]):
        part = {n: d[n][:, lo:hi] for n in I.NAMES}
        yp, sp, _ = oracle.forward(*args(part))
        np.testing.assert_allclose(y[:, lo:hi], yp, rtol=0, atol=1e-12 * np.abs(yp).max())
    np.testing.assert_allclose(s, sp, rtol=0, atol=1e-12 * np.abs(sp).max())


def test_chained_calls_equal_single_call():
    d = gen(2, 40, 2, 16, seed=21, s0=True, reset_p=0.1)
    y, s, _ = oracle.forward(*args(d), s0=d["s0"], reset=d["reset"])
    first = {n: d[n][:, :17] for n in I.NAMES}
    second = {n: d[n][:, 17:] for n in I.NAMES}
    y1, s1, _ = oracle.forward(*args(first), s0=d["s0"], reset=d["reset"][:, :17])
    y2, s2, _ = oracle.forward(*args(second), s0=s1, reset=d["reset"][:, 17:])
    assert rel(np.concatenate([y1, y2], axis=1), y) < 1e-13 and rel(s2, s) < 1e-13
    rng = np.random.default_rng(22)
    dy = rng.standard_normal(y.shape)
    dsT = rng.standard_normal(s.shape)
    g, _ = oracle.backward(*args(d), dy, s0=d["s0"], reset=d["reset"], dsT=dsT)
    g2, _ = oracle.backward(*args(second), dy[:, 17:], s0=s1, reset=d["reset"][:, 17:], dsT=dsT)
    g1, _ = oracle.backward(*args(first), dy[:, :17], s0=d["s0"], reset=d["reset"][:, :17], dsT=g2["ds0"])
    for n in ("dr", "dw", "dk", "dv", "da", "db"):
        assert rel(np.concatenate([g1[n], g2[n]], axis=1), g[n]) < 1e-12, n
    assert rel(g1["ds0"], g["ds0"]) < 1e-12


# ------------------------------------------------------------------ backward vs finite differences
def _loss(d, s0, reset, dy, dsT):
    y, s, _ = oracle.forward(*args(d), s0=s0, reset=reset)
    return float(np.sum(dy * y) + np.sum(dsT * s))


@pytest.mark.parametrize("N", [4, 8])
def test_backward_matches_central_differences(N):
    """Every gradient entry against (L(x+h) - L(x-h)) / 2h in fp64, T=20 (crosses 16), one reset."""
    T = 20
    d = gen(1, T, 1, N, seed=30 + N, s0=True)
    reset = np.zeros((1, T), np.uint8)
    reset[0, 11] = 1
    rng = np.random.default_rng(40 + N)
    dy = rng.standard_normal((1, T, 1, N))
    dsT = rng.standard_normal((1, 1, N, N))
    g, _ = oracle.backward(*args(d), dy, s0=d["s0"], reset=reset, dsT=dsT)
    h = 1e-6
    for name in I.NAMES:
        num = np.zeros_like(d[name])
        for idx in np.ndindex(d[name].shape):
            dp = {n: d[n].copy() for n in I.NAMES}
            dm = {n: d[n].copy() for n in I.NAMES}
            dp[name][idx] += h
            dm[name][idx] -= h
            num[idx] = (_loss(dp, d["s0"], reset, dy, dsT) - _loss(dm, d["s0"], reset, dy, dsT)) / (2 * h)
        assert rel(g["d" + name], num) < 1e-6, name
    num = np.zeros_like(d["s0"])
    for idx in np.ndindex(d["s0"].shape):
        sp, sm = d["s0"].copy(), d["s0"].copy()
        sp[idx] += h
        sm[idx] -= h
        num[idx] = (_loss(d, sp, reset, dy, dsT) - _loss(d, sm, reset, dy, dsT)) / (2 * h)
    assert rel(g["ds0"], num) < 1e-6
    # no gradient crosses the reset: inputs before it see only their own segment
    assert np.all(g["dw"][0, 11] == 0.0) and np.all(g["da"][0, 11] == 0.0)


def test_backward_adjoint_identity_n64():
    """<dy, J delta> + <dS_T, J_S delta> = <J^T(dy, dS_T), delta> for a random direction, N=64."""
    T = 21
    d = gen(1, T, 2, 64, seed=50, s0=True, reset_p=0.1)
    rng = np.random.default_rng(51)
    dy = rng.standard_normal((1, T, 2, 64))
    dsT = rng.standard_normal((1, 2, 64, 64))
    g, _ = oracle.backward(*args(d), dy, s0=d["s0"], reset=d["reset"], dsT=dsT)
    delta = {n: rng.standard_normal(d[n].shape) for n in I.NAMES}
    ds0 = rng.standard_normal(d["s0"].shape)
    eps = 1e-5
    dp = {n: d[n] + eps * delta[n] for n in I.NAMES}
    dm = {n: d[n] - eps * delta[n] for n in I.NAMES}
    lp = _loss(dp, d["s0"] + eps * ds0, d["reset"], dy, dsT)
    lm = _loss(dm, d["s0"] - eps * ds0, d["reset"], dy, dsT)
    directional = (lp - lm) / (2 * eps)
    adjoint = sum(float(np.sum(g["d" + n] * delta[n])) for n in I.NAMES) + float(np.sum(g["ds0"] * ds0))
    assert abs(directional - adjoint) <= 1e-7 * abs(adjoint)


# ------------------------------------------------------------------ decode step
def test_step_equals_one_token_forward_and_masks_rows():
    d = gen(4, 1, 3, 64, seed=60, s0=True)
    active = np.array([1, 0, 1, 0], np.uint8)
    st = d["s0"]
    y, st2 = oracle.step(*(d[n][:, 0] for n in I.NAMES), st, active)
    yf, sf, _ = oracle.forward(*args(d), s0=st)
    for b in range(4):
        if active[b]:
            assert rel(y[b], yf[b, 0]) < 1e-14 and rel(st2[b], sf[b]) < 1e-14
        else:
            np.testing.assert_array_equal(st2[b], st[b])
            np.testing.assert_array_equal(y[b], 0.0)


def test_zero_tokens():
    d = gen(1, 0, 2, 8, seed=61, s0=True)
    y, s, _ = oracle.forward(*args(d), s0=d["s0"])
    assert y.shape == (1, 0, 2, 8)
    np.testing.assert_array_equal(s, d["s0"])
