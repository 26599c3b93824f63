"""NumPy fp64 twin of the WKV-7 oracle -- TEST INFRASTRUCTURE ONLY.

Written separately from ``wkv7_oracle.c`` so that the two can be checked
against each other.  Vectorised over all (batch, head) units with a Python
loop over tokens; meant for small shapes.  Same definition and layouts as the
C oracle (rwkv-metal page, "The Metal WKV-7 kernel"): per token
``S <- S @ (diag(w) + a b^T) + v k^T`` and ``y = S r``, with ``S`` zeroed
before a token whose reset flag is set.
"""
from __future__ import annotations

import numpy as np


def forward(r, w, k, v, a, b, s0=None, reset=None):
    r, w, k, v, a, b = (np.asarray(x, dtype=np.float64) for x in (r, w, k, v, a, b))
    B, T, H, N = r.shape
    S = np.zeros((B, H, N, N)) if s0 is None else np.array(s0, dtype=np.float64)
    y = np.zeros_like(r)
    for t in range(T):
        if reset is not None:
            S = S * (1.0 - np.asarray(reset[:, t], dtype=np.float64))[:, None, None, None]
        wt, kt, vt, at, bt, rt = (x[:, t] for x in (w, k, v, a, b, r))   # [B,H,N]
        sa = np.einsum("bhij,bhj->bhi", S, at)
        S = S * wt[:, :, None, :] + sa[..., :, None] * bt[..., None, :] + vt[..., :, None] * kt[..., None, :]
        y[:, t] = np.einsum("bhij,bhj->bhi", S, rt)
    return y, S


def backward(r, w, k, v, a, b, dy, s0=None, reset=None, dsT=None):
    """Reverse mode through the stored per-token states (no checkpoints)."""
    r, w, k, v, a, b, dy = (np.asarray(x, dtype=np.float64) for x in (r, w, k, v, a, b, dy))
    B, T, H, N = r.shape
    S = np.zeros((B, H, N, N)) if s0 is None else np.array(s0, dtype=np.float64)
    prev, sas, outs = [], [], []
    for t in range(T):
        if reset is not None:
            S = S * (1.0 - np.asarray(reset[:, t], dtype=np.float64))[:, None, None, None]
        prev.append(S)
        sa = np.einsum("bhij,bhj->bhi", S, a[:, t])
        sas.append(sa)
        S = S * w[:, t][:, :, None, :] + sa[..., :, None] * b[:, t][..., None, :] + v[:, t][..., :, None] * k[:, t][..., None, :]
        outs.append(S)
    G = np.zeros((B, H, N, N)) if dsT is None else np.array(dsT, dtype=np.float64)
    grads = {n: np.zeros_like(r) for n in ("dr", "dw", "dk", "dv", "da", "db")}
    for t in range(T - 1, -1, -1):
        G = G + dy[:, t][..., :, None] * r[:, t][..., None, :]
        grads["dr"][:, t] = np.einsum("bhij,bhi->bhj", outs[t], dy[:, t])
        grads["dv"][:, t] = np.einsum("bhij,bhj->bhi", G, k[:, t])
        grads["dk"][:, t] = np.einsum("bhij,bhi->bhj", G, v[:, t])
        dsa = np.einsum("bhij,bhj->bhi", G, b[:, t])
        grads["db"][:, t] = np.einsum("bhij,bhi->bhj", G, sas[t])
        grads["dw"][:, t] = np.einsum("bhij,bhij->bhj", G, prev[t])
        grads["da"][:, t] = np.einsum("bhij,bhi->bhj", prev[t], dsa)
        G = G * w[:, t][:, :, None, :] + dsa[..., :, None] * a[:, t][..., None, :]
        if reset is not None:
            G = G * (1.0 - np.asarray(reset[:, t], dtype=np.float64))[:, None, None, None]
    grads["ds0"] = G
    return grads
