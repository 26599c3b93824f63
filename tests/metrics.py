"""Error metrics shared by the parity tests.

* ``err_rms``: max |x - ref| / RMS(ref) -- the forward tolerance metric.
* ``err_rms_excess``: the same, after removing, element by element, the half
  unit-in-the-last-place that storing the result in a 16-bit format costs
  (|bf16(x) - x| <= ulp/2).  The output y is stored in the input dtype; on these
  workloads max|y| is about 10x RMS(y), so bf16 storage alone moves y by up to
  ~2.1e-2 RMS.  The tolerance applies to the error beyond that rounding.
* ``cosine``: fp64 cosine similarity of the flattened tensors (gradients).
"""
from __future__ import annotations

import numpy as np

_MANT = {"bf16": 7, "f16": 10, "f32": 23}


def rms(x) -> float:
    x = np.asarray(x, dtype=np.float64)
    return float(np.sqrt(np.mean(x * x))) if x.size else 0.0


def err_rms(x, ref) -> float:
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    d = float(np.max(np.abs(x - ref)))
    r = rms(ref)
    return d / r if r > 0 else d


def half_ulp(x, dtype: str) -> np.ndarray:
    """Half the spacing of ``dtype`` at |x| (normal range)."""
    ax = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(ax, 1e-300)))
    return np.where(ax > 0, np.ldexp(1.0, (e - _MANT[dtype] - 1).astype(np.int64)), 0.0)


def err_rms_excess(x, ref, dtype: str) -> float:
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    allowance = half_ulp(np.maximum(np.abs(x), np.abs(ref)), dtype) if dtype != "f32" else 0.0
    d = np.maximum(np.abs(x - ref) - allowance, 0.0)
    r = rms(ref)
    return float(d.max()) / r if r > 0 else float(d.max())


def cosine(x, ref) -> float:
    x = np.asarray(x, dtype=np.float64).ravel()
    ref = np.asarray(ref, dtype=np.float64).ravel()
    nx, nr = np.linalg.norm(x), np.linalg.norm(ref)
    if nx == 0 and nr == 0:
        return 1.0
    if nx == 0 or nr == 0:
        return 0.0
    return float(np.dot(x, ref) / (nx * nr))
