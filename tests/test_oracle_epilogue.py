"""Pins for the epilogue oracle (GroupNorm per head, bonus term, output gating; no GPU).

Closed forms: the GroupNorm of 1..N, the bonus alone (y = 0) with r = k, gating by 0 and 1, the
GroupNorm's invariance to a shift of y (and to a scale with eps = 0); the backward against fp64
central differences on every input and parameter.
"""
from __future__ import annotations

import numpy as np
import pytest

from oracle import epilogue as E


def _rand(shape, rng):
    return rng.standard_normal(shape)


def _params(H, N, rng):
    return 1.0 + 0.3 * rng.standard_normal((H, N)), 0.2 * rng.standard_normal((H, N)), 0.5 * rng.standard_normal((H, N))


def test_groupnorm_of_one_to_n():
    N = 64
    y = np.arange(1, N + 1, dtype=np.float64).reshape(1, 1, 1, N)
    z0 = np.zeros_like(y)
    eps = 1e-5
    out, mu, rstd = E.forward(y, z0, z0, z0, np.ones_like(y), np.ones((1, N)), np.zeros((1, N)), np.zeros((1, N)), eps)
    var = (N * N - 1) / 12.0                        # variance of 1..N
    assert abs(mu[0, 0, 0] - (N + 1) / 2) < 1e-13 and abs(rstd[0, 0, 0] - 1 / np.sqrt(var + eps)) < 1e-15
    ref = (np.arange(1, N + 1) - (N + 1) / 2) / np.sqrt(var + eps)
    assert np.max(np.abs(out[0, 0, 0] - ref)) < 1e-13


def test_bonus_alone_with_r_equal_k():
    """y = 0 normalises to 0, so out = (beta + s v) g with s = sum_j r_j^2 rk_j."""
    rng = np.random.default_rng(1)
    B, T, H, N = 2, 3, 2, 16
    r = _rand((B, T, H, N), rng)
    v = _rand((B, T, H, N), rng)
    g = _rand((B, T, H, N), rng)
    gamma, beta, rk = _params(H, N, rng)
    out, _, _ = E.forward(np.zeros_like(r), r, r, v, g, gamma, beta, rk, 1e-5)
    s = np.einsum("bthj,hj->bth", r * r, rk)
    assert np.max(np.abs(out - (beta[None, None] + s[..., None] * v) * g)) < 1e-13


def test_gating_by_zero_and_one_and_shift_invariance():
    rng = np.random.default_rng(2)
    B, T, H, N = 1, 4, 3, 8
    y, r, k, v = (_rand((B, T, H, N), rng) for _ in range(4))
    gamma, beta, rk = _params(H, N, rng)
    ones, zeros = np.ones_like(y), np.zeros_like(y)
    z, _, _ = E.forward(y, r, k, v, ones, gamma, beta, rk, 1e-5)
    out0, _, _ = E.forward(y, r, k, v, zeros, gamma, beta, rk, 1e-5)
    assert np.all(out0 == 0.0)
    zs, _, _ = E.forward(y + 3.25, r, k, v, ones, gamma, beta, rk, 1e-5)   # a shift of y changes nothing
    assert np.max(np.abs(zs - z)) < 1e-12
    z1, _, _ = E.forward(y, r, k, v, ones, gamma, beta, rk, 0.0)
    z2, _, _ = E.forward(7.0 * y, r, k, v, ones, gamma, beta, rk, 0.0)    # nor a scale, with eps = 0
    assert np.max(np.abs(z1 - z2)) < 1e-12
    g = E.backward(rng.standard_normal(y.shape), y, r, k, v, zeros, gamma, beta, rk, 1e-5)
    assert all(np.all(g[n] == 0.0) for n in ("dy", "dr", "dk", "dv", "dgamma", "dbeta", "drk"))


@pytest.mark.parametrize("N", [4, 8])
def test_backward_matches_central_differences(N):
    rng = np.random.default_rng(10 + N)
    B, T, H = 2, 3, 2
    eps = 1e-3
    x = {n: _rand((B, T, H, N), rng) for n in ("y", "r", "k", "v", "g")}
    gamma, beta, rk = _params(H, N, rng)
    p = {"gamma": gamma, "beta": beta, "rk": rk}
    dout = rng.standard_normal((B, T, H, N))

    def loss(xx, pp):
        out, _, _ = E.forward(xx["y"], xx["r"], xx["k"], xx["v"], xx["g"], pp["gamma"], pp["beta"], pp["rk"], eps)
        return float(np.sum(dout * out))

    gr = E.backward(dout, x["y"], x["r"], x["k"], x["v"], x["g"], gamma, beta, rk, eps)
    h = 1e-6
    for name, arr, key in [(n, x, "d" + n) for n in x] + [(n, p, "d" + n) for n in p]:
        num = np.zeros_like(arr[name])
        for idx in np.ndindex(arr[name].shape):
            ap = {m: a.copy() for m, a in arr.items()}
            am = {m: a.copy() for m, a in arr.items()}
            ap[name][idx] += h
            am[name][idx] -= h
            if arr is x:
                num[idx] = (loss(ap, p) - loss(am, p)) / (2 * h)
            else:
                num[idx] = (loss(x, ap) - loss(x, am)) / (2 * h)
        err = np.max(np.abs(gr[key] - num)) / max(np.max(np.abs(num)), 1e-300)
        assert err < 1e-6, (name, err)
