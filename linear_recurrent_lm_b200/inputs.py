"""Seeded synthetic inputs for the WKV-7 workloads.

This module is the one piece shared by the CUDA path's tests/bench and by the
CPU oracle's tests.  It holds no WKV-7 arithmetic: it only draws random numbers
and applies the input recipe (decay parametrisation, key normalisation,
in-context learning rate) that defines the synthetic workloads, then rounds to
the storage dtype.

Recipe (one ``numpy.random.default_rng(seed)`` stream, fp64 draws, in this
order): r, k, v, z_w, kk_raw, z_iclr -- each standard normal of shape
[B,T,H,N] -- then the optional extras (dy, reset lengths, decode state,
active lengths).  Derived values are computed in fp64, rounded to fp32 (RNE),
and, for 16-bit storage, rounded once more to bf16/fp16 (RNE):

* w = exp(-exp(x)), x = -softplus(-z_w) - 0.5, so w lies in (0.545, 1)
* kk = kk_raw / ||kk_raw||_2 over the N channels of each (b,t,h)
* a = -kk,  b = kk * sigmoid(z_iclr)

This is the RWKV-7 in-context-learning-rate parametrisation: the decay is
data-dependent and kept inside (0,1), the removal key ``a`` is a unit vector
and ``b`` scales it by a gate in (0,1) (RWKV-MLX page, "Architecture" and
"Key Design Decisions"; rwkv-lab page, "GDN subset of RWKV-7", where the same
roles appear as the delta-rule removal key and the in-context learning rate).

16-bit values are carried as ``uint16`` bit patterns for bf16 (NumPy has no
bf16) and as ``float16`` for fp16.  ``to_f64`` decodes any storage array to
float64 exactly.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np

DTYPES = ("f32", "bf16", "f16")
NAMES = ("r", "w", "k", "v", "a", "b")


# ----------------------------------------------------------------- rounding
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    bias = ((u >> 16) & 1) + 0x7FFF
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def to_storage(x64: np.ndarray, dtype: str) -> np.ndarray:
    """fp64 -> fp32 (RNE) -> storage dtype (RNE)."""
    x32 = np.asarray(x64, dtype=np.float64).astype(np.float32)
    if dtype == "f32":
        return x32
    if dtype == "bf16":
        return f32_to_bf16_bits(x32)
    if dtype == "f16":
        return x32.astype(np.float16)
    raise ValueError(f"unknown dtype {dtype!r}")


def to_f64(x: np.ndarray, dtype: Optional[str] = None) -> np.ndarray:
    """Exact fp64 value of a storage array (uint16 is read as bf16 bits)."""
    x = np.asarray(x)
    if x.dtype == np.uint16 or dtype == "bf16":
        return bf16_bits_to_f32(x).astype(np.float64)
    return x.astype(np.float64)


# ----------------------------------------------------------------- recipe
def _softplus(u: np.ndarray) -> np.ndarray:
    return np.logaddexp(0.0, u)


def _sigmoid(u: np.ndarray) -> np.ndarray:
    return 0.5 * (1.0 + np.tanh(0.5 * u))


def draw_inputs(rng: np.random.Generator, shape, dtype: str, log_decay: bool = False) -> Dict[str, np.ndarray]:
    """Draw r,w,k,v,a,b of ``shape`` (last axis = N) in storage dtype.  With ``log_decay`` the "w"
    entry holds the decay's log-space parameter x (w = exp(-exp(x))) instead of w; the random draws
    are the same either way."""
    shape = tuple(int(s) for s in shape)
    r = rng.standard_normal(shape)
    k = rng.standard_normal(shape)
    v = rng.standard_normal(shape)
    z_w = rng.standard_normal(shape)
    kk_raw = rng.standard_normal(shape)
    z_iclr = rng.standard_normal(shape)
    x = -_softplus(-z_w) - 0.5
    w = np.exp(-np.exp(x))
    kk = kk_raw / np.sqrt(np.sum(kk_raw * kk_raw, axis=-1, keepdims=True))
    a = -kk
    b = kk * _sigmoid(z_iclr)
    out = {}
    for name, val in zip(NAMES, (r, x if log_decay else w, k, v, a, b)):
        out[name] = to_storage(val, dtype)
    return out


GDN_NAMES = ("q", "k", "v")


def draw_gdn_inputs(rng: np.random.Generator, B: int, T: int, H: int, Hk: int, N: int, dtype: str) -> Dict[str, np.ndarray]:
    """Gated-DeltaNet layer inputs (the rwkv-lab page's GDN target: 32 value heads and 16 key heads
    of 128 channels).  Draw order: q, k [B,T,Hk,N], v [B,T,H,N], z_g, z_beta [B,T,H] standard
    normal, then per value head A ~ U(1, 16) and dt ~ log-uniform on [1e-3, 1e-1].  Returns q, k, v
    in storage dtype and fp32 g = -A softplus(z_g + softplus^-1(dt)) (a log-decay <= 0 whose
    typical size is A dt) and beta = sigmoid(z_beta) (the write strength, in (0, 1)).  The pages
    give no distributions for these inputs; this is the common GDN parametrisation of the decay
    and the write gate."""
    q = rng.standard_normal((B, T, Hk, N))
    k = rng.standard_normal((B, T, Hk, N))
    v = rng.standard_normal((B, T, H, N))
    z_g = rng.standard_normal((B, T, H))
    z_beta = rng.standard_normal((B, T, H))
    A = rng.uniform(1.0, 16.0, H)
    dt = np.exp(rng.uniform(np.log(1e-3), np.log(1e-1), H))
    dt_bias = dt + np.log(-np.expm1(-dt))              # softplus(dt_bias) = dt
    g = -A * _softplus(z_g + dt_bias)
    beta = _sigmoid(z_beta)
    out = {n: to_storage(x, dtype) for n, x in zip(GDN_NAMES, (q, k, v))}
    out["g"] = g.astype(np.float32)
    out["beta"] = beta.astype(np.float32)
    return out


def geometric_resets(rng: np.random.Generator, B: int, T: int, mean_len: float) -> np.ndarray:
    """Per-token reset flags [B,T] u8 for packed documents.

    Document lengths are drawn one after another per row from a geometric
    distribution on {1,2,...} with success probability 1/mean_len; the last
    document of a row is cut at the row end.  Every row starts a document at
    t=0, so reset[b,0] = 1.
    """
    reset = np.zeros((B, T), dtype=np.uint8)
    p = 1.0 / float(mean_len)
    for bi in range(B):
        t = 0
        while t < T:
            reset[bi, t] = 1
            t += int(rng.geometric(p))
    return reset


@dataclasses.dataclass
class Workload:
    """One seeded synthetic workload (all arrays host-side, storage dtype)."""
    name: str
    B: int
    T: int
    H: int
    N: int
    dtype: str
    seed: int
    inputs: Dict[str, np.ndarray]
    s0: Optional[np.ndarray] = None          # [B,H,N,N] f32
    reset: Optional[np.ndarray] = None       # [B,T] u8
    dy: Optional[np.ndarray] = None          # [B,T,H,N] storage dtype
    prior: Optional[Dict[str, np.ndarray]] = None   # inputs of the prior tokens (prefill)
    state0: Optional[np.ndarray] = None      # decode: [B,H,N,N] f32
    steps: Optional[list] = None             # decode: list of per-step input dicts [B,H,N]
    lengths: Optional[np.ndarray] = None     # decode: active length per row

    def active(self, step: int) -> np.ndarray:
        return (self.lengths > step).astype(np.uint8)


# Shapes of the five workloads (184M-model layer: H=12; 1.5B-model layer: H=32).
SPECS = {
    0: dict(name="fwd_f32_B1_T64_H2", B=1, T=64, H=2, dtype="f32"),
    1: dict(name="train_bf16_B2_T512_H12", B=2, T=512, H=12, dtype="bf16"),
    2: dict(name="prefill_bf16_B1_T1024_H32_prior256", B=1, T=1024, H=32, dtype="bf16"),
    3: dict(name="packed_train_bf16_B8_T4096_H32", B=8, T=4096, H=32, dtype="bf16"),
    4: dict(name="decode_bf16_B256_H32_steps128", B=256, T=1, H=32, dtype="bf16"),
}
N_HEAD = 64
PRIOR_TOKENS = 256          # tokens run before the prefill to build its initial state
DECODE_STEPS = 128
DOC_MEAN = 512


def make_workload(idx: int, seed: Optional[int] = None, *, B: Optional[int] = None,
                  T: Optional[int] = None, H: Optional[int] = None, N: int = N_HEAD,
                  dtype: Optional[str] = None, log_decay: bool = False) -> Workload:
    """Build workload ``idx`` (0..4); size overrides give scaled-down copies.  ``log_decay`` hands
    out the decays' log-space parameter x in the "w" entries (same draws)."""
    spec = dict(SPECS[idx])
    seed = 1000 + idx if seed is None else int(seed)
    B = spec["B"] if B is None else B
    T = spec["T"] if T is None else T
    H = spec["H"] if H is None else H
    dtype = spec["dtype"] if dtype is None else dtype
    rng = np.random.default_rng(seed)
    if idx == 4:
        steps = DECODE_STEPS if T in (None, 1) else T
        state0 = rng.normal(0.0, 0.1, size=(B, H, N, N)).astype(np.float32)
        lengths = rng.integers(1, steps + 1, size=B)
        step_inputs = [draw_inputs(rng, (B, H, N), dtype, log_decay) for _ in range(steps)]
        return Workload(spec["name"], B, 1, H, N, dtype, seed, inputs={}, state0=state0,
                        steps=step_inputs, lengths=lengths)
    inputs = draw_inputs(rng, (B, T, H, N), dtype, log_decay)
    wl = Workload(spec["name"], B, T, H, N, dtype, seed, inputs)
    if idx in (1, 3):
        wl.dy = to_storage(rng.standard_normal((B, T, H, N)), dtype)
    if idx == 3:
        wl.reset = geometric_resets(rng, B, T, DOC_MEAN)
    if idx == 2:
        wl.prior = draw_inputs(rng, (B, PRIOR_TOKENS, H, N), dtype, log_decay)
    return wl
