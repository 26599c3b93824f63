"""Gated-delta-rule (GDN) front-end map oracle -- TEST INFRASTRUCTURE ONLY (fp64 NumPy).

The rwkv-lab page ("Highlight result -- GDN in RWKV-7") states that a gated DeltaNet layer's
recurrence is the wkv7 recurrence fed through a fixed map of its inputs, at matched head sizes
(its target model: 32 value heads and 16 key heads of 128).  From GDN's per-token inputs q, k
[B,T,Hk,N], v [B,T,H,N], scalar log-decay g <= 0 and write strength beta [B,T,H]:

    q^ = normalize(q),  k^ = normalize(k)            (L2 over the head's N channels)
    r  = q^ * r_scale                                (the page scales the output by 1/sqrt(N);
                                                      y = S r is linear in r, so the scale is
                                                      taken into r)
    decay: log w = g on every channel               (here in the recurrence's log-space input
                                                      x, w = exp(-exp(x)), so x = log(-g))
    k_write = beta k^,   a = -k^,   b = k^ exp(g) beta

The readings taken where the page is silent:
* normalize(x) = x / sqrt(sum x^2 + eps), the usual guarded L2 normalisation (eps = 0: x / |x|);
* value head h reads key head h // (H // Hk) (the target model has two value heads per key head);
* g = 0 (no decay) maps to x = -inf, which the log-space decay takes to w = 1.

``gated_delta_rule`` is the recurrence GDN itself runs, written in its own form (not through the
map), so that the map can be pinned against it:

    S_t = exp(g_t) S_{t-1} (I - beta_t k^_t k^_t^T) + beta_t v_t k^_t^T,   o_t = S_t q^_t r_scale.
"""
from __future__ import annotations

import numpy as np


def _f(x):
    return np.asarray(x, dtype=np.float64)


def normalize(x, eps):
    """x / sqrt(sum over the last axis of x^2 + eps)."""
    x = _f(x)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def key_head_of(H, Hk):
    """Index of the key head that each of the H value heads reads."""
    if Hk <= 0 or H % Hk != 0:
        raise ValueError(f"H={H} value heads do not share Hk={Hk} key heads evenly")
    return np.arange(H) // (H // Hk)


def gdn_map(q, k, g, beta, H, eps, r_scale):
    """The page's map, in its order.  q, k [B,T,Hk,N]; g, beta [B,T,H].  Returns a dict of r, x,
    kw (k_write), a, b, each [B,T,H,N]; x is the log-space decay input (log w = -exp(x) = g)."""
    q, k, g, beta = _f(q), _f(k), _f(g), _f(beta)
    kh = key_head_of(H, q.shape[2])
    qn = normalize(q, eps)[:, :, kh]
    kn = normalize(k, eps)[:, :, kh]
    N = q.shape[-1]
    with np.errstate(divide="ignore"):
        x = np.log(-g)
    return {
        "r": qn * r_scale,
        "x": np.repeat(x[..., None], N, axis=-1),
        "kw": beta[..., None] * kn,
        "a": -kn,
        "b": kn * (np.exp(g) * beta)[..., None],
    }


def gated_delta_rule(q, k, v, g, beta, eps, r_scale, s0=None):
    """GDN's own recurrence, token by token.  q, k [B,T,Hk,N]; v [B,T,H,N]; g, beta [B,T,H];
    s0 [B,H,N,N] or None.  Returns (o [B,T,H,N], S_T [B,H,N,N])."""
    q, k, v, g, beta = _f(q), _f(k), _f(v), _f(g), _f(beta)
    B, T, H, N = v.shape
    kh = key_head_of(H, q.shape[2])
    qn = normalize(q, eps)
    kn = normalize(k, eps)
    S = np.zeros((B, H, N, N)) if s0 is None else _f(s0).copy()
    o = np.zeros((B, T, H, N))
    eye = np.eye(N)
    for bi in range(B):
        for h in range(H):
            for t in range(T):
                kk = kn[bi, t, kh[h]]
                S[bi, h] = np.exp(g[bi, t, h]) * S[bi, h] @ (eye - beta[bi, t, h] * np.outer(kk, kk)) \
                    + beta[bi, t, h] * np.outer(v[bi, t, h], kk)
                o[bi, t, h] = S[bi, h] @ qn[bi, t, kh[h]] * r_scale
    return o, S
