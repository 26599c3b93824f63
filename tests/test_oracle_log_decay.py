"""Pins for the oracle's log-space decay input (no GPU).

With the log-space convention the decay input holds x and the recurrence uses w = exp(-exp(x))
(log w = -exp(x); the rwkv-lab page, "Highlight result -- GDN in RWKV-7", passes the wkv7 kernel
its decay in log space).  The map is pinned at points where it has a closed form, the forward
through the retention and causal-linear-attention closed forms, and the backward (dL/dx) by
central finite differences in fp64 taken on x itself.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from linear_recurrent_lm_b200 import inputs as I
from tests.test_oracle import args, gen, rel


def test_map_closed_forms():
    # exp(-exp(log(log 2))) = exp(-log 2) = 1/2;  exp(-exp(0)) = 1/e;  x -> -inf gives 1
    assert abs(oracle.decay_of_log(np.log(np.log(2.0))) - 0.5) < 1e-15
    assert abs(oracle.decay_of_log(0.0) - np.exp(-1.0)) < 1e-16
    assert oracle.decay_of_log(-60.0) == 1.0
    assert oracle.decay_of_log(10.0) == 0.0


def test_constant_x_is_retention():
    """x = log(-log gamma) everywhere, a=b=0: y_t = sum_{tau<=t} gamma^(t-tau) (r_t . k_tau) v_tau."""
    d = gen(1, 30, 1, 8, seed=113)
    g = 0.83
    d["w"][:] = np.log(-np.log(g))
    d["a"][:] = 0.0
    d["b"][:] = 0.0
    y, _, _ = oracle.forward(*args(d), log_decay=True)
    R, K, V = d["r"][0, :, 0], d["k"][0, :, 0], d["v"][0, :, 0]
    t = np.arange(30)
    decay = np.where(t[:, None] >= t[None, :], g ** (t[:, None] - t[None, :]).clip(min=0), 0.0)
    assert rel(y[0, :, 0], ((R @ K.T) * decay) @ V) < 1e-12


def test_far_negative_x_is_causal_linear_attention():
    """x = -60 (w = 1 to fp64), a=b=0: y = tril(R K^T) V."""
    d = gen(1, 25, 2, 16, seed=114)
    d["w"][:] = -60.0
    d["a"][:] = 0.0
    d["b"][:] = 0.0
    y, _, _ = oracle.forward(*args(d), log_decay=True)
    for h in range(2):
        R, K, V = d["r"][0, :, h], d["k"][0, :, h], d["v"][0, :, h]
        assert rel(y[0, :, h], np.tril(R @ K.T) @ V) < 1e-13


def _loss(d, s0, reset, dy, dsT):
    y, s, _ = oracle.forward(*args(d), s0=s0, reset=reset, log_decay=True)
    return float(np.sum(dy * y) + np.sum(dsT * s))


@pytest.mark.parametrize("N", [4, 8])
def test_backward_dx_matches_central_differences(N):
    """dL/dx (and the other gradients) against (L(x+h) - L(x-h)) / 2h in fp64, T=20, one reset."""
    T = 20
    rng = np.random.default_rng(130 + N)
    d = {n: v.astype(np.float64) for n, v in I.draw_inputs(rng, (1, T, 1, N), "f32", log_decay=True).items()}
    s0 = rng.standard_normal((1, 1, N, N))
    reset = np.zeros((1, T), np.uint8)
    reset[0, 9] = 1
    dy = rng.standard_normal((1, T, 1, N))
    dsT = rng.standard_normal((1, 1, N, N))
    g, _ = oracle.backward(*args(d), dy, s0=s0, reset=reset, dsT=dsT, log_decay=True)
    h = 1e-6
    for name in ("w", "k", "a"):   # x itself, and two inputs whose gradients run through the decays
        num = np.zeros_like(d[name])
        for idx in np.ndindex(d[name].shape):
            dp = {n: d[n].copy() for n in I.NAMES}
            dm = {n: d[n].copy() for n in I.NAMES}
            dp[name][idx] += h
            dm[name][idx] -= h
            num[idx] = (_loss(dp, s0, reset, dy, dsT) - _loss(dm, s0, reset, dy, dsT)) / (2 * h)
        assert rel(g["d" + name], num) < 1e-6, name
    # the reset stops the gradient: x of the reset token sees nothing of the state before it
    assert np.all(g["dw"][0, 9] == 0.0)


def test_step_with_log_decay_is_one_token_forward():
    rng = np.random.default_rng(140)
    d = {n: v.astype(np.float64) for n, v in I.draw_inputs(rng, (3, 1, 2, 64), "f32", log_decay=True).items()}
    st = rng.standard_normal((3, 2, 64, 64))
    y, st2 = oracle.step(*(d[n][:, 0] for n in I.NAMES), st, np.array([1, 1, 0], np.uint8), log_decay=True)
    yf, sf, _ = oracle.forward(*args(d), s0=st, log_decay=True)
    assert rel(y[:2], yf[:2, 0]) < 1e-14 and rel(st2[:2], sf[:2]) < 1e-14
    assert np.array_equal(st2[2], st[2]) and np.all(y[2] == 0.0)
