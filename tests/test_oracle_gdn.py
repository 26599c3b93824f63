"""Pins for the GDN front-end map oracle (no GPU).

The gated delta rule is pinned by its closed forms (no write: pure decay of s0; one write from
zero; the delta rule's overwrite S_t k_t = v_t), the key-head sharing by an explicit assignment,
and the map (rwkv-lab page, "Highlight result -- GDN in RWKV-7") by feeding its outputs through the
recurrence oracle with the log-space decay and comparing with the gated delta rule written in its
own form -- on shared key heads, with an initial state, at N = 16 and at the page's N = 128.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from oracle import gdn as G
from tests.test_oracle import rel


def _draw(rng, B, T, H, Hk, N, g_scale=0.3):
    q = rng.standard_normal((B, T, Hk, N))
    k = rng.standard_normal((B, T, Hk, N))
    v = rng.standard_normal((B, T, H, N))
    g = -np.abs(rng.standard_normal((B, T, H))) * g_scale
    beta = rng.uniform(0.05, 1.0, (B, T, H))
    return q, k, v, g, beta


def test_normalize_closed_form():
    np.testing.assert_allclose(G.normalize(np.array([3.0, 4.0]), 0.0), [0.6, 0.8], rtol=0, atol=1e-16)
    np.testing.assert_allclose(G.normalize(np.array([3.0, 4.0]), 11.0), [0.5, 4.0 / 6.0], rtol=0, atol=1e-16)


def test_key_head_assignment():
    np.testing.assert_array_equal(G.key_head_of(4, 2), [0, 0, 1, 1])
    np.testing.assert_array_equal(G.key_head_of(32, 16)[:6], [0, 0, 1, 1, 2, 2])
    with pytest.raises(ValueError):
        G.key_head_of(6, 4)


def test_rule_without_writes_is_pure_decay():
    """beta = 0: S_t = exp(g_1 + ... + g_t) s0 and o_t = S_t q^_t r_scale."""
    rng = np.random.default_rng(900)
    q, k, v, g, beta = _draw(rng, 1, 9, 2, 1, 8)
    beta[:] = 0.0
    s0 = rng.standard_normal((1, 2, 8, 8))
    o, S = G.gated_delta_rule(q, k, v, g, beta, 0.0, 0.5, s0=s0)
    c = np.cumsum(g, axis=1)                                    # [1, T, H]
    qn = q[0, :, 0] / np.linalg.norm(q[0, :, 0], axis=-1, keepdims=True)
    for h in range(2):
        ref = np.exp(c[0, :, h])[:, None] * (qn @ s0[0, h].T) * 0.5
        assert rel(o[0, :, h], ref) < 1e-13
    assert rel(S, np.exp(c[0, -1])[None, :, None, None] * s0) < 1e-13


def test_rule_one_write_from_zero():
    """One token from S = 0: S_1 = beta v k^T (unit k), o_1 = beta (k . q^) v r_scale."""
    rng = np.random.default_rng(901)
    q, k, v, g, beta = _draw(rng, 1, 1, 1, 1, 8)
    o, S = G.gated_delta_rule(q, k, v, g, beta, 0.0, 0.25)
    kn = k[0, 0, 0] / np.linalg.norm(k[0, 0, 0])
    qn = q[0, 0, 0] / np.linalg.norm(q[0, 0, 0])
    assert rel(S[0, 0], beta[0, 0, 0] * np.outer(v[0, 0, 0], kn)) < 1e-14
    assert rel(o[0, 0, 0], beta[0, 0, 0] * (kn @ qn) * 0.25 * v[0, 0, 0]) < 1e-14


def test_rule_overwrite_reads_back_the_value():
    """beta = 1, g = 0 (the plain delta rule): S_t k^_t = v_t after every token; with q = k the
    output is v_t itself."""
    rng = np.random.default_rng(902)
    q, k, v, g, beta = _draw(rng, 1, 20, 1, 1, 16)
    beta[:] = 1.0
    g[:] = 0.0
    o, _ = G.gated_delta_rule(k, k, v, g, beta, 0.0, 1.0, s0=rng.standard_normal((1, 1, 16, 16)))
    assert rel(o, v) < 1e-12


def test_map_closed_forms():
    rng = np.random.default_rng(903)
    q, k, _, g, beta = _draw(rng, 2, 5, 4, 2, 16)
    g[0, 0, 0] = 0.0
    m = G.gdn_map(q, k, g, beta, 4, 0.0, 0.125)
    assert rel(np.linalg.norm(m["a"], axis=-1), np.ones((2, 5, 4))) < 1e-14
    assert rel(np.linalg.norm(m["r"], axis=-1), np.full((2, 5, 4), 0.125)) < 1e-14
    assert rel(m["kw"], -beta[..., None] * m["a"]) < 1e-15
    assert rel(m["b"], -(np.exp(g) * beta)[..., None] * m["a"]) < 1e-15
    assert rel(oracle.decay_of_log(m["x"]), np.repeat(np.exp(g)[..., None], 16, axis=-1)) < 1e-14
    assert m["x"][0, 0, 0, 0] == -np.inf and oracle.decay_of_log(m["x"][0, 0, 0]).tolist() == [1.0] * 16
    # value heads 2 and 3 read key head 1
    kn1 = k[1, 3, 1] / np.linalg.norm(k[1, 3, 1])
    assert rel(m["a"][1, 3, 2], -kn1) < 1e-15 and rel(m["a"][1, 3, 3], -kn1) < 1e-15


@pytest.mark.parametrize("B,T,H,Hk,N,eps", [(2, 23, 4, 2, 16, 0.0), (1, 40, 2, 1, 16, 1e-3), (1, 6, 2, 1, 128, 1e-6)])
def test_map_through_the_recurrence_is_the_gated_delta_rule(B, T, H, Hk, N, eps):
    rng = np.random.default_rng(904 + N + T)
    q, k, v, g, beta = _draw(rng, B, T, H, Hk, N)
    s0 = rng.standard_normal((B, H, N, N))
    scale = 1.0 / np.sqrt(N)
    m = G.gdn_map(q, k, g, beta, H, eps, scale)
    y, s, _ = oracle.forward(m["r"], m["x"], m["kw"], v, m["a"], m["b"], s0=s0, log_decay=True)
    o, S = G.gated_delta_rule(q, k, v, g, beta, eps, scale, s0=s0)
    assert rel(y, o) < 1e-11
    assert rel(s, S) < 1e-11


def test_map_without_the_decay_in_b_is_not_the_rule():
    """The comparison above is sharp: b without its exp(g) factor (a plausible slip) moves the
    output far outside the bound."""
    rng = np.random.default_rng(905)
    q, k, v, g, beta = _draw(rng, 1, 30, 2, 1, 16, g_scale=1.0)
    m = G.gdn_map(q, k, g, beta, 2, 0.0, 0.25)
    y, _, _ = oracle.forward(m["r"], m["x"], m["kw"], v, m["a"], m["kw"], log_decay=True)
    o, _ = G.gated_delta_rule(q, k, v, g, beta, 0.0, 0.25)
    assert rel(y, o) > 1e-3
