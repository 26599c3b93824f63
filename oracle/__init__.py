"""WKV-7 CPU oracle -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The CUDA library and its Python binding never
do, and nothing here imports them: the two implementations share no code.

Two independent fp64 implementations of the same definition:

* ``forward`` / ``backward`` / ``step``: the plain C oracle
  (``wkv7_oracle.c``), token-order loops, threaded over the independent
  (batch, head) units.
* ``numpy_twin``: a separately written NumPy version (vectorised over units,
  Python loop over tokens), used on small shapes to cross-check the C code.

The recurrence (rwkv-metal page, "The Metal WKV-7 kernel"; RWKV-MLX page,
"Key Design Decisions"), per (b,h), token t, state S (row i = value, column
j = key):  sa = S a_t;  S = S diag(w_t) + sa b_t^T + v_t k_t^T;  y_t = S r_t.
A reset flag at t zeroes the incoming state first (HF model card page: packed
sequences reset the state at each boundary).  The backward is hand-derived
(the pages print none); see ``wkv7_oracle.c`` for the derivation.

Arrays: r,w,k,v,a,b,y,dy and gradients [B,T,H,N] float64; states
[B,H,N,N] float64 (S[i][j] at [..., i, j]); reset [B,T] uint8.

Log-space decay (``log_decay=True``): the ``w`` argument then holds x and the decay is
w = exp(-exp(x)), i.e. log w = -exp(x) (the rwkv-lab page, "Highlight result -- GDN in RWKV-7",
hands the wkv7 kernel its decay in log space; this is the RWKV-7 parametrisation of the decay),
and the backward's ``dw`` entry is dL/dx = dL/dw * (-w exp(x)), by the chain rule.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

from . import build as _build

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        i64 = ctypes.c_int64
        L.wkv7_oracle_forward.restype = ctypes.c_int
        L.wkv7_oracle_forward.argtypes = [i64, i64, i64, i64] + [dp] * 7 + [u8p, dp, dp, ctypes.c_int]
        L.wkv7_oracle_backward.restype = ctypes.c_int
        L.wkv7_oracle_backward.argtypes = [i64, i64, i64, i64] + [dp] * 7 + [u8p, dp, dp] + [dp] * 7 + [ctypes.c_int]
        L.wkv7_oracle_step.restype = None
        L.wkv7_oracle_step.argtypes = [i64, i64, i64] + [dp] * 7 + [u8p, dp]
        _lib = L
    return _lib


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float64)


def _dp(x: Optional[np.ndarray]):
    if x is None:
        return None
    return x.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _u8(x: Optional[np.ndarray]):
    if x is None:
        return None, None
    x = np.ascontiguousarray(x, dtype=np.uint8)
    return x, x.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8))


def _shape(r: np.ndarray):
    B, T, H, N = r.shape
    return int(B), int(T), int(H), int(N)


def decay_of_log(x) -> np.ndarray:
    """w = exp(-exp(x)) in fp64 (the log-space decay input)."""
    return np.exp(-np.exp(_f64(x)))


def forward(r, w, k, v, a, b, s0=None, reset=None, nthreads: int = 0, log_decay: bool = False):
    """Token-order forward.  Returns (y [B,T,H,N], s_out [B,H,N,N], threads used).  With
    ``log_decay`` the ``w`` argument holds x and the decay is exp(-exp(x))."""
    if log_decay:
        w = decay_of_log(w)
    r, w, k, v, a, b = (_f64(x) for x in (r, w, k, v, a, b))
    B, T, H, N = _shape(r)
    s0 = None if s0 is None else _f64(s0)
    reset, rp = _u8(reset)
    y = np.zeros((B, T, H, N))
    s_out = np.zeros((B, H, N, N))
    used = lib().wkv7_oracle_forward(B, T, H, N, *(_dp(x) for x in (r, w, k, v, a, b, s0)), rp,
                                     _dp(y), _dp(s_out), int(nthreads))
    if used < 0:
        raise MemoryError("oracle forward: allocation failed")
    return y, s_out, used


def backward(r, w, k, v, a, b, dy, s0=None, reset=None, dsT=None, nthreads: int = 0, log_decay: bool = False):
    """Hand-derived reverse mode.  Returns (dict of dr..db [B,T,H,N] and ds0 [B,H,N,N], threads).
    With ``log_decay`` the ``w`` argument holds x and ``dw`` is returned as dL/dx."""
    x_log = _f64(w) if log_decay else None
    if log_decay:
        w = decay_of_log(x_log)
    r, w, k, v, a, b, dy = (_f64(x) for x in (r, w, k, v, a, b, dy))
    B, T, H, N = _shape(r)
    s0 = None if s0 is None else _f64(s0)
    dsT = None if dsT is None else _f64(dsT)
    reset, rp = _u8(reset)
    g = {n: np.zeros((B, T, H, N)) for n in ("dr", "dw", "dk", "dv", "da", "db")}
    g["ds0"] = np.zeros((B, H, N, N))
    used = lib().wkv7_oracle_backward(B, T, H, N, *(_dp(x) for x in (r, w, k, v, a, b, s0)), rp,
                                      _dp(dy), _dp(dsT), *(_dp(g[n]) for n in ("dr", "dw", "dk", "dv", "da", "db", "ds0")),
                                      int(nthreads))
    if used < 0:
        raise MemoryError("oracle backward: allocation failed")
    if log_decay:   # chain rule through w = exp(-exp(x)): dw/dx = -w exp(x)
        g["dw"] = g["dw"] * (-w * np.exp(x_log))
    return g, used


def step(r, w, k, v, a, b, state, active=None, log_decay: bool = False):
    """One decode token on ``state`` [B,H,N,N] (returned updated copy) -> (y [B,H,N], state)."""
    if log_decay:
        w = decay_of_log(w)
    r, w, k, v, a, b = (_f64(x) for x in (r, w, k, v, a, b))
    B, H, N = (int(s) for s in r.shape)
    st = np.array(state, dtype=np.float64, copy=True, order="C")
    active, ap = _u8(active)
    y = np.zeros((B, H, N))
    lib().wkv7_oracle_step(B, H, N, *(_dp(x) for x in (r, w, k, v, a, b)), _dp(st), ap, _dp(y))
    return y, st
