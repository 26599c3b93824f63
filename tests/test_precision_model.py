"""A model of the chunked forward's roundings, checked against the oracle on the CPU.

Not the oracle and not the kernels: a NumPy restatement of the 16-token chunk formulas in which
every operand of a tensor-core product is rounded to tf32 (nearest, ties away from zero, as the
kernels' conversions do), products are kept in fp32 and the state stays in fp32 -- the
arithmetic both chunked forms (fused and split) are designed to.  It shows that this precision
budget fits the bf16 tolerance with room to spare, which is why the chunked kernels may run the
state products in tf32; the kernels themselves are held to the oracle by the GPU parity tests.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from linear_recurrent_lm_b200 import inputs as I
from tests.metrics import err_rms, err_rms_excess

F32 = np.float32


def tf32(x):
    """Round fp32 values to tf32 (10 explicit mantissa bits), nearest, ties away from zero."""
    u = np.asarray(x, F32).view(np.uint32).astype(np.uint64)
    return ((u + 0x1000) & 0xFFFFE000).astype(np.uint32).view(F32)


def mm(a, b):
    """Product of tf32-rounded operands, rounded to fp32 (summed in fp64: the tensor core's fp32
    accumulation adds errors near 2^-24, far below the 2^-11 of the operand rounding)."""
    return (tf32(a).astype(np.float64) @ tf32(b).astype(np.float64)).astype(F32)


def chunk_model(r, w, k, v, a, b, reset, form):
    """One (b,h) unit, inputs [T,64] fp32 (already bf16 values). Returns y [T,64], S [64,64]."""
    T, N = r.shape
    S = np.zeros((N, N), F32)
    y = np.zeros((T, N), F32)
    for c0 in range(0, T, 16):
        sl = slice(c0, c0 + 16)
        rr, ww, kk, vv, aa, bb = (x[sl] for x in (r, w, k, v, a, b))
        C = rr.shape[0]
        rs = reset[sl]
        lam = np.cumprod(ww, axis=0, dtype=F32)
        lamp = np.vstack([np.ones((1, N), F32), lam[:-1]])
        At, Rt, Bh, Kh = aa * lamp, rr * lam, bb / lam, kk / lam
        first = int(np.argmax(rs)) if rs.any() else C
        seg = np.cumsum(np.concatenate([[0], rs[1:]]))
        same = seg[:, None] == seg[None, :]
        strict = np.tril(np.ones((C, C), bool), -1) & same
        lower = np.tril(np.ones((C, C), bool)) & same
        G = mm(np.vstack([At, Rt]), np.vstack([Bh, Kh]).T)
        Lab, Lak = G[:C, :C] * strict, tf32(G[:C, C:] * strict)
        Mrb, Mrk = tf32(G[C:, :C] * lower), G[C:, C:] * lower
        Tm = np.eye(C, dtype=F32)                          # (I - Lab)^-1 by substitution in fp32
        for t in range(1, C):
            Tm[t, :t] = Lab[t, :t] @ Tm[:t, :t]
        Tm = tf32(Tm)
        m0 = (np.arange(C) < first).astype(F32)[:, None]
        W = tf32(mm(Tm, m0 * At))
        X = tf32(mm(Tm, Lak))
        M = tf32(mm(Mrb, Tm))
        Q = tf32(m0 * Rt + mm(M, m0 * At))
        Z = tf32(Mrk + mm(M, Lak))
        ls = (seg == seg[-1]).astype(F32)[:, None] if rs.any() else np.ones((C, 1), F32)
        Bl, Kl = tf32(ls * Bh), tf32(ls * Kh)
        keep = F32(0.0 if rs.any() else 1.0)
        Y = mm(Q, S.T) + mm(Z, vv)
        if form == "fused":                                 # SA read back as tf32 for the update
            SA = mm(W, S.T) + mm(X, vv)
            D = mm(SA.T, Bl) + mm(vv.T, Kl)
        else:                                               # SA0 = W S0^T, Kx = X^T Bl + Kl
            Kx = tf32(mm(X.T, Bl) + Kl)
            D = mm(mm(S, W.T), Bl) + mm(vv.T, Kx)
        y[sl] = Y
        S = ((keep * S + D) * lam[-1][None, :]).astype(F32)
    return y, S


@pytest.mark.parametrize("form", ["fused", "split"])
def test_tf32_budget_fits_the_bf16_tolerance(form):
    """Packed documents with resets (workload 3 recipe, T cut to 768): y rounded to bf16 and the
    fp32 state stay within a third of the 2e-2 bound against the oracle."""
    wl = I.make_workload(3, T=768)
    ey = es = 0.0
    for (b, h) in [(0, 0), (3, 17), (7, 31)]:
        x = {n: I.to_f64(wl.inputs[n][b, :, h]).astype(F32) for n in I.NAMES}
        y, S = chunk_model(*(x[n] for n in I.NAMES), wl.reset[b], form)
        part = {n: I.to_f64(wl.inputs[n][b:b + 1, :, h:h + 1]) for n in I.NAMES}
        yo, so, _ = oracle.forward(*(part[n] for n in I.NAMES), reset=wl.reset[b:b + 1])
        yb = I.to_f64(I.to_storage(y.astype(np.float64), "bf16"))
        ey = max(ey, err_rms_excess(yb, yo[0, :, 0], "bf16"))
        es = max(es, err_rms(S, so[0, 0]))
    assert ey <= 2e-2 / 3, ey
    assert es <= 2e-2 / 3, es


def test_model_without_rounding_is_the_recurrence():
    """With the roundings taken out the same code reproduces the oracle to fp32 accuracy, so the
    error measured above is the tf32 budget and not a flaw of the model."""
    global tf32
    keep_tf32 = tf32
    tf32 = lambda x: np.asarray(x, F32)                      # noqa: E731
    try:
        wl = I.make_workload(3, T=256)
        x = {n: I.to_f64(wl.inputs[n][2, :, 5]).astype(F32) for n in I.NAMES}
        for form in ("fused", "split"):
            y, S = chunk_model(*(x[n] for n in I.NAMES), wl.reset[2], form)
            part = {n: I.to_f64(wl.inputs[n][2:3, :, 5:6]) for n in I.NAMES}
            yo, so, _ = oracle.forward(*(part[n] for n in I.NAMES), reset=wl.reset[2:3])
            assert err_rms(y, yo[0, :, 0]) < 1e-4 and err_rms(S, so[0, 0]) < 1e-4, form
    finally:
        tf32 = keep_tf32
