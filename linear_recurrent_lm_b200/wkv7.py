"""Python binding of libwkv7 (the C ABI in include/wkv7.h).

Argument marshalling only: every step of the WKV-7 path runs in the CUDA
kernels of ``libwkv7.so``.  PyTorch provides device memory and the current
stream.  The same entry points as the C ABI:

* ``forward(r, w, k, v, a, b, s0=None, reset=None, ...)``  -> (y, s_out, workspace)
* ``backward(r, w, k, v, a, b, dy, workspace, s0=None, reset=None, dsT=None, ...)``
  -> dict(dr, dw, dk, dv, da, db, ds0)
* ``step(r, w, k, v, a, b, state, active=None, ...)`` -> y   (state updated in place)
* ``gdn_map(q, k, g, beta, H, ...)`` -> dict(r, x, kw, a, b)   (gated-DeltaNet inputs -> WKV-7 inputs)
* ``state_compose(S, P, U, ...)`` -> S P + U (or S P^T + U) per (b, h)   (context parallelism)
* ``workspace_bytes(B, T, H, dtype)``
* ``device_status(clear=True)`` -> OK, ERR_TIMEOUT, ERR_BOUNDS or ERR_NONFINITE (synchronises the device)
* ``use_build("release" | "debug")``: route every call through ``libwkv7.so`` (default) or its
  bounds-checked twin ``libwkv7_debug.so`` (same ABI; ``WKV7_BUILD=debug`` in the environment
  selects it at import)

Tensors are [B,T,H,N] (token inputs), [B,H,N,N] fp32 (states), [B,T] uint8
(reset), [B] uint8 (active), all on one CUDA device and contiguous.  The head size N is 64; the
token-order forward and the decode step also take N = 128 (the gated-delta-rule map's heads).  If the
library is missing, importing this module raises: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATHS = {"release": os.path.join(_HERE, "libwkv7.so"), "debug": os.path.join(_HERE, "libwkv7_debug.so")}
LIB_PATH = LIB_PATHS["release"]

(OK, ERR_NULL, ERR_SHAPE, ERR_DTYPE, ERR_ALIGN, ERR_WORKSPACE, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT,
 ERR_SCRATCH_LIMIT, ERR_NONFINITE, ERR_BOUNDS) = range(12)
NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024   # WKV7_NOALLOC_SCRATCH_BYTES
FLAG_TEST_WAIT_TIMEOUT = 0x80000000        # WKV7_FLAG_TEST_WAIT_TIMEOUT (test hook, T <= 16)
FLAG_CHECK_FINITE = 0x1                    # WKV7_FLAG_CHECK_FINITE: scan outputs for NaN / Inf
FLAG_LOG_DECAY = 0x2                       # WKV7_FLAG_LOG_DECAY: w holds x, decay = exp(-exp(x))
FLAG_EPILOGUE_GRADS = 0x4                  # WKV7_FLAG_EPILOGUE_GRADS: dy is the epilogue's fp32 block
DTYPE_CODE = {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}
ALGO_CODE = {"auto": 0, "scan": 1, "chunked": 2, "chunked_fused": 3, "chunked_split": 4}
N_HEAD = 64
HEAD_SIZES = (64, 128)
CHUNK = 16


class Desc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("T", ctypes.c_int64), ("H", ctypes.c_int64), ("N", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("algo", ctypes.c_int32), ("flags", ctypes.c_uint32)]


class Epilogue(ctypes.Structure):
    """wkv7_epilogue_t: fp32 [H,64] GroupNorm weight and bias, bonus weights, and eps."""
    _fields_ = [("ln_w", ctypes.c_void_p), ("ln_b", ctypes.c_void_p), ("r_k", ctypes.c_void_p),
                ("eps", ctypes.c_float)]


class Gdn(ctypes.Structure):
    """wkv7_gdn_t: key heads, the L2-normalisation guard and the scale taken into r."""
    _fields_ = [("Hk", ctypes.c_int64), ("eps", ctypes.c_float), ("r_scale", ctypes.c_float)]


class WKV7Error(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {lib().wkv7_status_string(status).decode()} (status {status})")
        self.status = status


_loaded: Dict[str, ctypes.CDLL] = {}
_active = os.environ.get("WKV7_BUILD", "release")
if _active not in LIB_PATHS:
    raise ValueError(f"WKV7_BUILD must be one of {sorted(LIB_PATHS)}, got {_active!r}")


def _load(variant: str) -> ctypes.CDLL:
    path = LIB_PATHS[variant]
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m linear_recurrent_lm_b200.build` "
                          "(or __graft_entry__.build()); the WKV-7 path has no CPU fallback")
    L = ctypes.CDLL(path)
    vp = ctypes.c_void_p
    dp = ctypes.POINTER(Desc)
    L.wkv7_version.restype = ctypes.c_int
    L.wkv7_status_string.restype = ctypes.c_char_p
    L.wkv7_status_string.argtypes = [ctypes.c_int]
    L.wkv7_workspace_bytes.restype = ctypes.c_size_t
    L.wkv7_workspace_bytes.argtypes = [dp]
    L.wkv7_forward.restype = ctypes.c_int
    L.wkv7_forward.argtypes = [dp] + [vp] * 12
    L.wkv7_backward.restype = ctypes.c_int
    L.wkv7_backward.argtypes = [dp] + [vp] * 19
    L.wkv7_step.restype = ctypes.c_int
    L.wkv7_step.argtypes = [dp] + [vp] * 10
    L.wkv7_train_step_noalloc.restype = ctypes.c_int
    L.wkv7_train_step_noalloc.argtypes = [dp] + [vp] * 20
    L.wkv7_get_device_status.restype = ctypes.c_int
    L.wkv7_get_device_status.argtypes = [ctypes.c_int]
    L.wkv7_debug_checks.restype = ctypes.c_int
    L.wkv7_debug_checks.argtypes = []
    ep = ctypes.POINTER(Epilogue)
    L.wkv7_epilogue_forward.restype = ctypes.c_int
    L.wkv7_epilogue_forward.argtypes = [dp, ep] + [vp] * 7
    L.wkv7_forward_epilogue.restype = ctypes.c_int
    L.wkv7_forward_epilogue.argtypes = [dp, ep] + [vp] * 14
    L.wkv7_epilogue_backward.restype = ctypes.c_int
    L.wkv7_epilogue_backward.argtypes = [dp, ep] + [vp] * 12
    L.wkv7_state_compose.restype = ctypes.c_int
    L.wkv7_state_compose.argtypes = [dp, vp, vp, vp, vp, ctypes.c_int, vp]
    L.wkv7_gdn_map.restype = ctypes.c_int
    L.wkv7_gdn_map.argtypes = [dp, ctypes.POINTER(Gdn)] + [vp] * 10
    return L


def lib() -> ctypes.CDLL:
    """The library every call goes through (raises if it has not been built)."""
    if _active not in _loaded:
        _loaded[_active] = _load(_active)
    return _loaded[_active]


def use_build(variant: str) -> str:
    """Route every later call through ``variant`` ("release" or "debug"); return the previous one.

    The two builds are separate CUDA modules: each has its own device status word, which
    ``device_status`` reads from the build in use."""
    global _active
    if variant not in LIB_PATHS:
        raise ValueError(f"unknown build {variant!r}; expected one of {sorted(LIB_PATHS)}")
    prev = _active
    _active = variant
    try:
        lib()
    except ImportError:
        _active = prev
        raise
    return prev


def active_build() -> str:
    return _active


lib()   # fail at import time if the CUDA library is absent


def make_desc(B: int, T: int, H: int, dtype, algo: str = "auto", N: int = N_HEAD, flags: int = 0) -> Desc:
    code = DTYPE_CODE[dtype] if isinstance(dtype, torch.dtype) else int(dtype)
    return Desc(int(B), int(T), int(H), int(N), code, ALGO_CODE[algo] if isinstance(algo, str) else int(algo), int(flags))


def workspace_bytes(B: int, T: int, H: int, dtype=torch.bfloat16, N: int = N_HEAD) -> int:
    return int(lib().wkv7_workspace_bytes(ctypes.byref(make_desc(B, T, H, dtype, N=N))))


def device_status(clear: bool = True) -> int:
    """The device status word of the current device (synchronises it): OK, ERR_TIMEOUT, ERR_BOUNDS or
    ERR_NONFINITE (in that order of precedence)."""
    return int(lib().wkv7_get_device_status(1 if clear else 0))


def _ptr(x: Optional[torch.Tensor]):
    """Device address of a contiguous CUDA tensor (the C ABI takes device pointers only)."""
    if x is None:
        return None
    if not x.is_cuda:
        raise ValueError(f"WKV-7 tensors must be on a CUDA device, got a {x.device} tensor of shape {tuple(x.shape)}")
    if not x.is_contiguous():
        raise ValueError(f"WKV-7 tensors must be contiguous, got strides {x.stride()} for shape {tuple(x.shape)}")
    return ctypes.c_void_p(x.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, where: str):
    if status != OK:
        raise WKV7Error(status, where)


def _token_shape(x: torch.Tensor, sizes=(N_HEAD,)):
    if x.dim() != 4 or x.shape[-1] not in sizes:
        raise ValueError(f"expected [B,T,H,N] with N in {sizes}, got {tuple(x.shape)}")
    return tuple(int(s) for s in x.shape[:3])


def _flags(flags: int, log_decay: bool) -> int:
    return int(flags) | (FLAG_LOG_DECAY if log_decay else 0)


def forward(r, w, k, v, a, b, s0=None, reset=None, *, y=None, s_out=None, workspace=None,
            need_workspace: bool = True, want_state: bool = True, algo: str = "auto", stream=None, flags: int = 0,
            log_decay: bool = False):
    """WKV-7 forward over [B,T,H,N] inputs (N = 64, or 128 with the token-order scan).  Returns (y,
    s_out, workspace).  With ``log_decay`` the ``w`` tensor holds x and the decay is exp(-exp(x))."""
    B, T, H = _token_shape(r, HEAD_SIZES)
    N = int(r.shape[-1])
    dev = r.device
    if y is None:
        y = torch.empty_like(r)
    if s_out is None and want_state:
        s_out = torch.empty((B, H, N, N), device=dev, dtype=torch.float32)
    if workspace is None and need_workspace:
        workspace = torch.empty(max(workspace_bytes(B, T, H, r.dtype, N), 16), device=dev, dtype=torch.uint8)
    d = make_desc(B, T, H, r.dtype, algo, N=N, flags=_flags(flags, log_decay))
    st = lib().wkv7_forward(ctypes.byref(d), *(_ptr(x) for x in (r, w, k, v, a, b, s0, reset, y, s_out, workspace)),
                            _stream(stream))
    _check(st, "wkv7_forward")
    return y, s_out, workspace


def backward(r, w, k, v, a, b, dy, workspace, s0=None, reset=None, dsT=None, *, grads=None,
             want_ds0: bool = True, algo: str = "auto", stream=None, flags: int = 0,
             log_decay: bool = False) -> Dict[str, torch.Tensor]:
    """WKV-7 backward from the checkpoints written by ``forward``.  With ``log_decay`` (as in the
    forward) ``w`` holds x and the "dw" entry receives dL/dx.  ``dy`` may be the fp32 block
    [4,B,T,H,64] that ``epilogue_backward`` returns as "eg" (dy, then the epilogue's parts of dr, dk,
    dv, which are added in)."""
    if dy.dim() == 5:
        if dy.dtype != torch.float32 or tuple(dy.shape) != (4,) + tuple(r.shape):
            raise ValueError(f"the epilogue's gradient block must be fp32 [4,B,T,H,64], got {tuple(dy.shape)}")
        flags = int(flags) | FLAG_EPILOGUE_GRADS
    B, T, H = _token_shape(r)
    g = dict(grads) if grads is not None else {}
    for n in ("dr", "dw", "dk", "dv", "da", "db"):
        if g.get(n) is None:
            g[n] = torch.empty_like(r)
    if g.get("ds0") is None and want_ds0:
        g["ds0"] = torch.empty((B, H, N_HEAD, N_HEAD), device=r.device, dtype=torch.float32)
    d = make_desc(B, T, H, r.dtype, algo, flags=_flags(flags, log_decay))
    st = lib().wkv7_backward(ctypes.byref(d), *(_ptr(x) for x in (r, w, k, v, a, b, s0, reset, dy, dsT, workspace)),
                             *(_ptr(g[n]) for n in ("dr", "dw", "dk", "dv", "da", "db")), _ptr(g.get("ds0")),
                             _stream(stream))
    _check(st, "wkv7_backward")
    return g


def step(r, w, k, v, a, b, state, active=None, *, y=None, stream=None, flags: int = 0, log_decay: bool = False):
    """One decode token on ``state`` [B,H,N,N] (in place).  Inputs [B,H,N], N = 64 or 128.  Returns y."""
    if r.dim() != 3 or r.shape[-1] not in HEAD_SIZES:
        raise ValueError(f"expected [B,H,N] with N in {HEAD_SIZES}, got {tuple(r.shape)}")
    B, H = int(r.shape[0]), int(r.shape[1])
    if y is None:
        y = torch.empty_like(r)
    d = make_desc(B, 1, H, r.dtype, N=int(r.shape[-1]), flags=_flags(flags, log_decay))
    st = lib().wkv7_step(ctypes.byref(d), *(_ptr(x) for x in (r, w, k, v, a, b, state, active, y)), _stream(stream))
    _check(st, "wkv7_step")
    return y


def train_step_noalloc(r, w, k, v, a, b, dy, s0=None, reset=None, dsT=None, *, y=None, s_out=None, grads=None,
                       want_ds0: bool = True, algo: str = "auto", stream=None, log_decay: bool = False):
    """Forward + backward with the library's fixed scratch instead of a workspace (nothing is
    allocated by the library; outputs not given are allocated here by torch).  For callers that
    cannot allocate device memory themselves: pass every output.  Returns (y, s_out, grads)."""
    B, T, H = _token_shape(r)
    if y is None:
        y = torch.empty_like(r)
    if s_out is None:
        s_out = torch.empty((B, H, N_HEAD, N_HEAD), device=r.device, dtype=torch.float32)
    g = dict(grads) if grads is not None else {}
    for n in ("dr", "dw", "dk", "dv", "da", "db"):
        if g.get(n) is None:
            g[n] = torch.empty_like(r)
    if g.get("ds0") is None and want_ds0:
        g["ds0"] = torch.empty((B, H, N_HEAD, N_HEAD), device=r.device, dtype=torch.float32)
    flags = FLAG_EPILOGUE_GRADS if dy.dim() == 5 else 0   # the epilogue's fp32 block (see backward)
    d = make_desc(B, T, H, r.dtype, algo, flags=_flags(flags, log_decay))
    st = lib().wkv7_train_step_noalloc(ctypes.byref(d), *(_ptr(x) for x in (r, w, k, v, a, b, s0, reset, y, s_out, dy, dsT)),
                                       *(_ptr(g[n]) for n in ("dr", "dw", "dk", "dv", "da", "db")), _ptr(g.get("ds0")),
                                       _stream(stream))
    _check(st, "wkv7_train_step_noalloc")
    return y, s_out, g


def _epi(ln_w, ln_b, r_k, eps) -> Epilogue:
    for t in (ln_w, ln_b, r_k):
        if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("epilogue parameters must be contiguous fp32 CUDA tensors [H,64]")
    return Epilogue(ln_w.data_ptr(), ln_b.data_ptr(), r_k.data_ptr(), float(eps))


def epilogue_forward(y, r, k, v, g, ln_w, ln_b, r_k, eps: float, *, out=None, stream=None, flags: int = 0):
    """The WKV epilogue: out = (GroupNorm_h(y) ln_w + ln_b + (sum r k r_k) v) g, per (b,t,h).  Token
    tensors [B,T,H,64]; ln_w, ln_b, r_k fp32 [H,64]."""
    B, T, H = _token_shape(y)
    if out is None:
        out = torch.empty_like(y)
    d = make_desc(B, T, H, y.dtype, flags=flags)
    ep = _epi(ln_w, ln_b, r_k, eps)
    st = lib().wkv7_epilogue_forward(ctypes.byref(d), ctypes.byref(ep), *(_ptr(x) for x in (y, r, k, v, g, out)),
                                     _stream(stream))
    _check(st, "wkv7_epilogue_forward")
    return out


def epilogue_backward(y, r, k, v, g, dout, ln_w, ln_b, r_k, eps: float, *, grads=None, want_params: bool = True,
                      stream=None, flags: int = 0) -> Dict[str, torch.Tensor]:
    """Reverse mode of ``epilogue_forward``: dict of "eg" (fp32 [4,B,T,H,64]: dy, then the bonus parts
    of dr, dk, dv -- pass it to ``backward`` as its dy), "dg" [B,T,H,64], and (zeroed here, then summed
    over b and t) dln_w, dln_b, dr_k [H,64]."""
    B, T, H = _token_shape(y)
    g_ = dict(grads) if grads is not None else {}
    if g_.get("eg") is None:
        g_["eg"] = torch.empty((4,) + tuple(y.shape), device=y.device, dtype=torch.float32)
    if g_.get("dg") is None:
        g_["dg"] = torch.empty_like(y)
    if want_params:
        for n in ("dln_w", "dln_b", "dr_k"):
            g_[n] = torch.zeros((H, N_HEAD), device=y.device, dtype=torch.float32)
    d = make_desc(B, T, H, y.dtype, flags=flags)
    ep = _epi(ln_w, ln_b, r_k, eps)
    st = lib().wkv7_epilogue_backward(ctypes.byref(d), ctypes.byref(ep), *(_ptr(x) for x in (y, r, k, v, g, dout)),
                                      _ptr(g_["eg"]), _ptr(g_["dg"]),
                                      *(_ptr(g_.get(n)) for n in ("dln_w", "dln_b", "dr_k")), _stream(stream))
    _check(st, "wkv7_epilogue_backward")
    return g_


def forward_epilogue(r, w, k, v, a, b, g, ln_w, ln_b, r_k, eps: float, s0=None, reset=None, *, out=None, y=None,
                     want_y: bool = True, s_out=None, workspace=None, need_workspace: bool = True,
                     want_state: bool = True, algo: str = "auto", stream=None, flags: int = 0,
                     log_decay: bool = False):
    """The forward with the WKV epilogue: out = epilogue(y) (fused into the recurrence's kernel in the
    fused chunked form).  Returns (out, y or None, s_out, workspace)."""
    B, T, H = _token_shape(r)
    dev = r.device
    if out is None:
        out = torch.empty_like(r)
    if y is None and want_y:
        y = torch.empty_like(r)
    if s_out is None and want_state:
        s_out = torch.empty((B, H, N_HEAD, N_HEAD), device=dev, dtype=torch.float32)
    if workspace is None and need_workspace:
        workspace = torch.empty(max(workspace_bytes(B, T, H, r.dtype), 16), device=dev, dtype=torch.uint8)
    d = make_desc(B, T, H, r.dtype, algo, flags=_flags(flags, log_decay))
    ep = _epi(ln_w, ln_b, r_k, eps)
    st = lib().wkv7_forward_epilogue(ctypes.byref(d), ctypes.byref(ep),
                                     *(_ptr(x) for x in (r, w, k, v, a, b, s0, reset, g, y, out, s_out, workspace)),
                                     _stream(stream))
    _check(st, "wkv7_forward_epilogue")
    return out, y, s_out, workspace


def gdn_map(q, k, g, beta, H: int, eps: float = 1e-6, r_scale: Optional[float] = None, *, out=None, stream=None,
            flags: int = 0) -> Dict[str, torch.Tensor]:
    """The gated-DeltaNet front end (wkv7_gdn_map): q, k [B,T,Hk,N] and fp32 g, beta [B,T,H] ->
    dict of r, x, kw, a, b [B,T,H,N] for ``forward`` / ``step`` with ``log_decay=True`` and GDN's
    own v.  ``r_scale`` defaults to 1/sqrt(N)."""
    B, T, Hk = _token_shape(q, HEAD_SIZES)
    N = int(q.shape[-1])
    if tuple(k.shape) != tuple(q.shape) or k.dtype != q.dtype:
        raise ValueError(f"q and k must match, got {tuple(q.shape)} {q.dtype} and {tuple(k.shape)} {k.dtype}")
    for n, t in (("g", g), ("beta", beta)):
        if t.dtype != torch.float32 or tuple(t.shape) != (B, T, H):
            raise ValueError(f"{n} must be fp32 [B,T,H] = {(B, T, H)}, got {tuple(t.shape)} {t.dtype}")
    o = dict(out) if out is not None else {}
    for n in ("r", "x", "kw", "a", "b"):
        if o.get(n) is None:
            o[n] = torch.empty((B, T, H, N), device=q.device, dtype=q.dtype)
    d = make_desc(B, T, H, q.dtype, N=N, flags=flags)
    gd = Gdn(int(Hk), float(eps), float(N ** -0.5 if r_scale is None else r_scale))
    st = lib().wkv7_gdn_map(ctypes.byref(d), ctypes.byref(gd), *(_ptr(x) for x in (q, k, g, beta)),
                            *(_ptr(o[n]) for n in ("r", "x", "kw", "a", "b")), _stream(stream))
    _check(st, "wkv7_gdn_map")
    return o


def state_compose(S, P, U, *, out=None, transpose: bool = False, stream=None, flags: int = 0) -> torch.Tensor:
    """wkv7_state_compose: out = S P + U (S P^T + U with ``transpose``) per (b, h) unit, all fp32
    [B,H,N,N]; S or U may be None (zero).  ``out`` may be U itself."""
    ref = next(t for t in (S, P, U, out) if t is not None)
    if ref.dim() != 4 or ref.shape[-1] != ref.shape[-2] or ref.shape[-1] not in HEAD_SIZES:
        raise ValueError(f"expected fp32 states [B,H,N,N] with N in {HEAD_SIZES}, got {tuple(ref.shape)}")
    for t in (S, P, U, out):
        if t is not None and (t.dtype != torch.float32 or tuple(t.shape) != tuple(ref.shape)):
            raise ValueError(f"states must all be fp32 {tuple(ref.shape)}, got {tuple(t.shape)} {t.dtype}")
    B, H, N = int(ref.shape[0]), int(ref.shape[1]), int(ref.shape[-1])
    if out is None:
        out = torch.empty_like(ref)
    d = make_desc(B, 1, H, torch.float32, N=N, flags=flags)
    st = lib().wkv7_state_compose(ctypes.byref(d), _ptr(S), _ptr(P), _ptr(U), _ptr(out), 1 if transpose else 0,
                                  _stream(stream))
    _check(st, "wkv7_state_compose")
    return out
