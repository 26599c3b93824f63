"""WKV epilogue oracle -- TEST INFRASTRUCTURE ONLY (fp64 NumPy, plain definitions).

The step after the recurrence in an RWKV-7 time-mix block: per-head GroupNorm of y (rwkv-metal
page, architecture table: "ln_x ... GroupNorm (per head)" for the official-weights model), the
RWKV "bonus" term and output gating (rwkv-lab page, "Native RWKV megakernel backend": the fp32
state update fused "through GroupNorm, the RWKV bonus, and output gating").  The pages print no
formulas; the readings taken, per (b, t, h) with channels i, j = 0..N-1:

    mu = mean_i y_i,  var = mean_i (y_i - mu)^2,  rstd = 1 / sqrt(var + eps)
    yn_i = (y_i - mu) rstd                                    (GroupNorm, one group per head)
    s    = sum_j r_j k_j rk[h, j]                             (bonus weight of the token)
    z_i  = yn_i gamma[h, i] + beta[h, i] + s v_i              (normalised y plus the bonus s v)
    out_i = z_i g_i                                           (output gating)

with r, k, v the recurrence's own inputs, g the gate [B,T,H,N], and gamma, beta, rk [H,N]
parameters.  ``backward`` is the reverse mode of these lines, written out below; the parameter
gradients are summed over (b, t).
"""
from __future__ import annotations

import numpy as np


def _f(x):
    return np.asarray(x, dtype=np.float64)


def forward(y, r, k, v, g, gamma, beta, rk, eps):
    """Returns (out, mu, rstd): out [B,T,H,N]; mu, rstd [B,T,H]."""
    y, r, k, v, g = (_f(x) for x in (y, r, k, v, g))
    gamma, beta, rk = (_f(x) for x in (gamma, beta, rk))
    mu = y.mean(axis=-1)
    var = ((y - mu[..., None]) ** 2).mean(axis=-1)
    rstd = 1.0 / np.sqrt(var + eps)
    yn = (y - mu[..., None]) * rstd[..., None]
    s = np.sum(r * k * rk[None, None], axis=-1)
    z = yn * gamma[None, None] + beta[None, None] + s[..., None] * v
    return z * g, mu, rstd


def backward(dout, y, r, k, v, g, gamma, beta, rk, eps):
    """Reverse mode.  Returns a dict: dy, dg, and the bonus parts of dr, dk, dv [B,T,H,N]; dgamma,
    dbeta, drk [H,N] (summed over batch and time)."""
    dout, y, r, k, v, g = (_f(x) for x in (dout, y, r, k, v, g))
    gamma, beta, rk = (_f(x) for x in (gamma, beta, rk))
    mu = y.mean(axis=-1, keepdims=True)
    var = ((y - mu) ** 2).mean(axis=-1, keepdims=True)
    rstd = 1.0 / np.sqrt(var + eps)
    yn = (y - mu) * rstd
    s = np.sum(r * k * rk[None, None], axis=-1, keepdims=True)
    z = yn * gamma[None, None] + beta[None, None] + s * v
    # out = z g
    dg = dout * z
    dz = dout * g
    # z = yn gamma + beta + s v
    dgamma = np.sum(dz * yn, axis=(0, 1))
    dbeta = np.sum(dz, axis=(0, 1))
    dv = s * dz
    ds = np.sum(dz * v, axis=-1, keepdims=True)
    dyn = dz * gamma[None, None]
    # s = sum_j r_j k_j rk_j
    dr = ds * k * rk[None, None]
    dk = ds * r * rk[None, None]
    drk = np.sum(ds * r * k, axis=(0, 1))
    # yn = (y - mu) rstd with mu, rstd functions of y:
    # dy_i = rstd (dyn_i - mean(dyn) - yn_i mean(dyn yn))
    dy = rstd * (dyn - dyn.mean(axis=-1, keepdims=True) - yn * np.mean(dyn * yn, axis=-1, keepdims=True))
    return {"dy": dy, "dg": dg, "dr": dr, "dk": dk, "dv": dv, "dgamma": dgamma, "dbeta": dbeta, "drk": drk}
