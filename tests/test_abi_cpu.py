"""The C ABI without a GPU: the library loads, exports every function the
header declares, and rejects bad arguments before launching anything."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "wkv7.h")


@pytest.fixture(scope="module")
def L():
    from linear_recurrent_lm_b200 import build
    build.build_all()
    from linear_recurrent_lm_b200 import wkv7
    return wkv7


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(wkv7_[a-z_0-9]+)\s*\(", text)))


@pytest.mark.parametrize("variant", ("release", "debug"))
def test_exports_every_declared_symbol(L, variant):
    names = declared_functions()
    assert {"wkv7_forward", "wkv7_backward", "wkv7_step", "wkv7_workspace_bytes", "wkv7_debug_checks"} <= set(names)
    lib = ctypes.CDLL(L.LIB_PATHS[variant])
    for n in names:
        assert hasattr(lib, n), (variant, n)
    assert lib.wkv7_debug_checks() == (1 if variant == "debug" else 0)


def test_use_build_switches_library(L):
    assert L.active_build() == "release"
    prev = L.use_build("debug")
    try:
        assert prev == "release" and L.lib().wkv7_debug_checks() == 1
        d = L.make_desc(1, 16, 1, 1)
        d.N = 32
        assert call_fwd(L, d) == L.ERR_UNSUPPORTED     # same host-side validation in both builds
    finally:
        L.use_build(prev)
    assert L.lib().wkv7_debug_checks() == 0
    with pytest.raises(ValueError):
        L.use_build("fast")


def test_version_and_status_strings(L):
    lib = L.lib()
    assert lib.wkv7_version() >= 100
    strings = [lib.wkv7_status_string(s) for s in range(L.ERR_BOUNDS + 1)]
    assert all(strings) and b"unknown status" not in strings and len(set(strings)) == len(strings)
    assert lib.wkv7_status_string(12345) == b"unknown status"


def test_workspace_matches_checkpoint_memory_on_rwkv_mlx_page(L):
    """RWKV-MLX page ("Key Design Decisions" 2): checkpoints every 16 tokens cost
    about 12 MB at the 184M-model layer shape (B=2, T=512, 12 heads of 64)."""
    ckpt = 2 * 12 * (512 // 16) * 64 * 64 * 4
    assert ckpt == 12_582_912
    # checkpoints, then one int per head (rounded up to 16 bytes) for the backward's marks
    assert L.workspace_bytes(2, 512, 12) == ckpt + 96
    assert L.workspace_bytes(1, 17, 1) == 2 * 64 * 64 * 4 + 16        # ceil(17/16) = 2 checkpoints
    assert L.workspace_bytes(1, 0, 1) == 0


FAKE = 0x10000       # 16-byte aligned address that is never dereferenced (validation fails first)


def call_fwd(L, desc, ptrs=None, **over):
    p = dict(r=FAKE, w=FAKE, k=FAKE, v=FAKE, a=FAKE, b=FAKE, s0=None, reset=None, y=FAKE, s_out=None, ws=None)
    p.update(over)
    vp = lambda x: None if x is None else ctypes.c_void_p(x)
    return L.lib().wkv7_forward(None if desc is None else ctypes.byref(desc),
                                *(vp(p[n]) for n in ("r", "w", "k", "v", "a", "b", "s0", "reset", "y", "s_out", "ws")),
                                None)


def test_forward_validation_codes(L):
    import torch
    d = L.make_desc(1, 16, 1, torch.bfloat16)
    assert call_fwd(L, None) == L.ERR_NULL
    bad = L.make_desc(1, 16, 1, torch.bfloat16); bad.N = 32
    assert call_fwd(L, bad) == L.ERR_UNSUPPORTED
    bad = L.make_desc(1, 16, 1, torch.bfloat16); bad.flags = 8                 # no such flag bit
    assert call_fwd(L, bad) == L.ERR_UNSUPPORTED
    bad = L.make_desc(1, 17, 1, torch.bfloat16, flags=L.FLAG_TEST_WAIT_TIMEOUT)   # the test hook needs T <= 16
    assert call_fwd(L, bad) == L.ERR_UNSUPPORTED
    bad = L.make_desc(1, 16, 1, torch.bfloat16, flags=L.FLAG_TEST_WAIT_TIMEOUT | 8)
    assert call_fwd(L, bad) == L.ERR_UNSUPPORTED
    for algo in ("chunked", "chunked_fused", "chunked_split"):      # tf32 products cannot meet the f32 bound
        assert call_fwd(L, L.make_desc(1, 16, 1, torch.float32, algo), ws=FAKE) == L.ERR_UNSUPPORTED
    bad = L.make_desc(1, 16, 1, torch.bfloat16); bad.algo = 7
    assert call_fwd(L, bad) == L.ERR_UNSUPPORTED
    bad = L.make_desc(1, 16, 1, torch.bfloat16); bad.algo = -1
    assert call_fwd(L, bad) == L.ERR_UNSUPPORTED
    # the split chunked forward carries its first pass in the workspace: required even for inference
    assert call_fwd(L, L.make_desc(1, 16, 1, torch.bfloat16, "chunked_split")) == L.ERR_WORKSPACE
    assert call_fwd(L, L.make_desc(0, 16, 1, torch.bfloat16, "chunked_split"),
                    r=None, w=None, k=None, v=None, a=None, b=None, y=None) == L.OK   # nothing to run
    bad = L.make_desc(1, 16, 1, torch.bfloat16); bad.dtype = 9
    assert call_fwd(L, bad) == L.ERR_DTYPE
    assert call_fwd(L, L.make_desc(-1, 16, 1, torch.bfloat16)) == L.ERR_SHAPE
    assert call_fwd(L, L.make_desc(1, -3, 1, torch.bfloat16)) == L.ERR_SHAPE
    assert call_fwd(L, L.make_desc(1 << 40, 1 << 20, 1 << 10, torch.bfloat16)) == L.ERR_SHAPE
    assert call_fwd(L, L.make_desc(1 << 20, 1, 1 << 12, torch.bfloat16)) == L.ERR_SHAPE   # grid > 2^31-1
    assert call_fwd(L, d, k=None) == L.ERR_NULL
    assert call_fwd(L, d, y=None) == L.ERR_NULL
    assert call_fwd(L, d, v=FAKE + 2) == L.ERR_ALIGN
    assert call_fwd(L, d, s0=FAKE + 8) == L.ERR_ALIGN
    assert call_fwd(L, d, ws=FAKE + 4) == L.ERR_ALIGN
    # empty problems launch nothing and succeed
    assert call_fwd(L, L.make_desc(0, 16, 4, torch.bfloat16), r=None, w=None, k=None, v=None, a=None, b=None, y=None) == L.OK
    assert call_fwd(L, L.make_desc(3, 16, 0, torch.bfloat16), r=None, w=None, k=None, v=None, a=None, b=None, y=None) == L.OK


def test_workspace_byte_count_overflow_is_a_shape_error(L):
    """A descriptor whose token tensors fit in int64 bytes but whose checkpoint workspace does not
    (B*H*ceil(T/16)*16 KiB, four times the bytes of one bf16 input) is refused everywhere: the
    workspace size would be 0, and without its scratch the no-allocation entry point must not run
    the forward and skip the backward."""
    import torch
    d = L.make_desc(1, 1 << 54, 1, torch.bfloat16)       # 2^54 tokens: 2^62 bytes of f32 activations
    assert L.workspace_bytes(1, 1 << 54, 1) == 0
    assert call_fwd(L, d) == L.ERR_SHAPE
    lib = L.lib()
    vp = lambda x: None if x is None else ctypes.c_void_p(x)
    st = lib.wkv7_train_step_noalloc(ctypes.byref(d), *map(vp, [FAKE] * 6), None, None, vp(FAKE), None, vp(FAKE),
                                     None, *map(vp, [FAKE] * 6), None, None)
    assert st == L.ERR_SHAPE
    # one step below the limit is still a valid shape with a non-zero workspace
    assert L.workspace_bytes(1, 1 << 48, 1) == (1 << 44) * 16384 + 16


def test_backward_and_step_validation_codes(L):
    import torch
    lib = L.lib()
    vp = lambda x: None if x is None else ctypes.c_void_p(x)
    d = L.make_desc(1, 16, 1, torch.bfloat16)
    base = [FAKE] * 6 + [None, None, FAKE, None]     # r..b, s0, reset, dy, dsT
    grads = [FAKE] * 6 + [None]
    assert lib.wkv7_backward(ctypes.byref(d), *map(vp, base), None, *map(vp, grads), None) == L.ERR_WORKSPACE
    assert lib.wkv7_backward(ctypes.byref(d), *map(vp, base), vp(FAKE), *map(vp, [FAKE] * 5 + [None, None]), None) == L.ERR_NULL
    assert lib.wkv7_backward(ctypes.byref(d), *map(vp, base), vp(FAKE + 1), *map(vp, grads), None) == L.ERR_ALIGN
    s = L.make_desc(4, 2, 1, torch.bfloat16)      # a step takes exactly one token
    assert lib.wkv7_step(ctypes.byref(s), *map(vp, [FAKE] * 7), None, vp(FAKE), None) == L.ERR_UNSUPPORTED
    s = L.make_desc(4, 1, 1, torch.bfloat16)
    assert lib.wkv7_step(ctypes.byref(s), *map(vp, [FAKE] * 6), None, None, vp(FAKE), None) == L.ERR_NULL


def test_no_cpu_fallback_without_gpu(L):
    """On a host with no GPU a valid call must fail loudly (ERR_CUDA), never compute on the CPU."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("host has a GPU")
    d = L.make_desc(1, 16, 1, torch.bfloat16)
    assert call_fwd(L, d) == L.ERR_CUDA
    # the output check is a valid flag on its own and with the timeout hook (T <= 16)
    assert call_fwd(L, L.make_desc(1, 16, 1, torch.bfloat16, flags=L.FLAG_CHECK_FINITE)) == L.ERR_CUDA
    both = L.FLAG_CHECK_FINITE | L.FLAG_TEST_WAIT_TIMEOUT
    assert call_fwd(L, L.make_desc(1, 16, 1, torch.bfloat16, flags=both)) == L.ERR_CUDA
    assert L.device_status() == L.ERR_CUDA      # the status word cannot be read without a device


def test_binding_rejects_host_and_strided_tensors_before_any_call(L):
    """The binding passes device pointers only: a host tensor (or a strided view) is refused in Python,
    so a host address can never reach a kernel."""
    import torch
    x = torch.zeros(1, 16, 1, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        L.forward(x, x, x, x, x, x)
    with pytest.raises(ValueError, match="CUDA"):
        L._ptr(torch.zeros(4))



def test_log_decay_flag_is_accepted_by_validation(L):
    """WKV7_FLAG_LOG_DECAY passes the descriptor checks (on this host the call then fails to launch
    with WKV7_ERR_CUDA instead of being refused as an unknown flag)."""
    import torch
    d = L.make_desc(1, 16, 1, torch.bfloat16, flags=L.FLAG_LOG_DECAY)
    assert call_fwd(L, d) != L.ERR_UNSUPPORTED
    d = L.make_desc(1, 16, 1, torch.bfloat16, flags=L.FLAG_LOG_DECAY | L.FLAG_CHECK_FINITE)
    assert call_fwd(L, d) != L.ERR_UNSUPPORTED


def test_epilogue_validation_codes(L):
    """The epilogue entry points refuse bad arguments before any launch."""
    import torch
    lib = L.lib()
    vp = ctypes.c_void_p
    P = vp(0x10000)                                   # aligned, never dereferenced
    ep = L.Epilogue(0x10000, 0x10000, 0x10000, 6.4e-4)
    d = L.make_desc(1, 16, 1, torch.bfloat16)
    fwd = lambda desc, e, *p: lib.wkv7_epilogue_forward(desc, e, *p, None)   # noqa: E731
    assert fwd(None, ctypes.byref(ep), *([P] * 6)) == L.ERR_NULL
    assert fwd(ctypes.byref(d), None, *([P] * 6)) == L.ERR_NULL
    assert fwd(ctypes.byref(d), ctypes.byref(ep), None, *([P] * 5)) == L.ERR_NULL
    bad = L.Epilogue(0x10000, 0x10000, 0x10000, 0.0)
    assert fwd(ctypes.byref(d), ctypes.byref(bad), *([P] * 6)) == L.ERR_UNSUPPORTED
    bad = L.Epilogue(0x10002, 0x10000, 0x10000, 6.4e-4)
    assert fwd(ctypes.byref(d), ctypes.byref(bad), *([P] * 6)) == L.ERR_ALIGN
    dl = L.make_desc(1, 16, 1, torch.bfloat16, flags=L.FLAG_LOG_DECAY)
    assert fwd(ctypes.byref(dl), ctypes.byref(ep), *([P] * 6)) == L.ERR_UNSUPPORTED
    assert fwd(ctypes.byref(d), ctypes.byref(ep), vp(0x10008), *([P] * 5)) == L.ERR_ALIGN
    bwd = lambda desc, e, *p: lib.wkv7_epilogue_backward(desc, e, *p, None)   # noqa: E731
    # y, r, k, v, g, dout, eg, dg, then the three parameter gradients (optional)
    assert bwd(ctypes.byref(d), ctypes.byref(ep), *([P] * 7), None, None, None, None) == L.ERR_NULL
    assert bwd(ctypes.byref(d), ctypes.byref(ep), *([P] * 8), vp(0x10002), None, None) == L.ERR_ALIGN
    # T = 0: nothing to do, and no launch
    d0 = L.make_desc(1, 0, 1, torch.bfloat16)
    assert fwd(ctypes.byref(d0), ctypes.byref(ep), *([None] * 6)) == L.OK


def test_epilogue_grads_flag_is_accepted_by_validation(L):
    import torch
    d = L.make_desc(1, 16, 1, torch.bfloat16, flags=L.FLAG_EPILOGUE_GRADS)
    assert call_fwd(L, d) != L.ERR_UNSUPPORTED


def test_head_size_128_limits(L):
    """N = 128 (the gated-DeltaNet heads) runs the token-order forward and the decode step only:
    every chunked form, the backward, the no-alloc step and the epilogue refuse it before any
    launch; the workspace counts 128x128 checkpoints."""
    import torch
    lib = L.lib()
    P = ctypes.c_void_p(FAKE)
    for algo in ("chunked", "chunked_fused", "chunked_split"):
        d = L.make_desc(1, 16, 1, torch.bfloat16, algo, N=128)
        assert call_fwd(L, d, ws=FAKE) == L.ERR_UNSUPPORTED
    d = L.make_desc(1, 16, 1, torch.bfloat16, N=128)
    assert lib.wkv7_backward(ctypes.byref(d), *([P] * 6), None, None, P, None, P, *([P] * 6), None, None) \
        == L.ERR_UNSUPPORTED
    assert lib.wkv7_train_step_noalloc(ctypes.byref(d), *([P] * 6), None, None, P, None, P, None,
                                       *([P] * 6), None, None) == L.ERR_UNSUPPORTED
    ep = L.Epilogue(FAKE, FAKE, FAKE, 6.4e-4)
    assert lib.wkv7_epilogue_forward(ctypes.byref(d), ctypes.byref(ep), *([P] * 6), None) == L.ERR_UNSUPPORTED
    assert L.workspace_bytes(1, 17, 1, torch.bfloat16, N=128) == 2 * 128 * 128 * 4 + 16
    bad = L.make_desc(1, 16, 1, torch.bfloat16, N=96)
    assert call_fwd(L, bad) == L.ERR_UNSUPPORTED


def test_gdn_map_validation_codes(L):
    """wkv7_gdn_map refuses bad arguments before any launch."""
    import torch
    lib = L.lib()
    vp = ctypes.c_void_p
    P = vp(FAKE)
    d = L.make_desc(1, 16, 4, torch.bfloat16, N=128)
    call = lambda desc, gd, *p: lib.wkv7_gdn_map(desc, gd, *p, None)   # noqa: E731
    gd = L.Gdn(2, 1e-6, 128 ** -0.5)
    assert call(None, ctypes.byref(gd), *([P] * 9)) == L.ERR_NULL
    assert call(ctypes.byref(d), None, *([P] * 9)) == L.ERR_NULL
    for bad in (L.Gdn(3, 1e-6, 1.0), L.Gdn(0, 1e-6, 1.0), L.Gdn(2, -1.0, 1.0), L.Gdn(2, float("nan"), 1.0),
                L.Gdn(2, 1e-6, float("inf")), L.Gdn(2, 1e-6, float("nan"))):
        assert call(ctypes.byref(d), ctypes.byref(bad), *([P] * 9)) == L.ERR_UNSUPPORTED
    assert call(ctypes.byref(d), ctypes.byref(gd), None, *([P] * 8)) == L.ERR_NULL
    assert call(ctypes.byref(d), ctypes.byref(gd), P, P, None, *([P] * 6)) == L.ERR_NULL     # g
    assert call(ctypes.byref(d), ctypes.byref(gd), P, P, vp(FAKE + 2), *([P] * 6)) == L.ERR_ALIGN
    assert call(ctypes.byref(d), ctypes.byref(gd), *([P] * 4), vp(FAKE + 8), *([P] * 4)) == L.ERR_ALIGN
    dl = L.make_desc(1, 16, 4, torch.bfloat16, N=128, flags=L.FLAG_LOG_DECAY)
    assert call(ctypes.byref(dl), ctypes.byref(gd), *([P] * 9)) == L.ERR_UNSUPPORTED
    d96 = L.make_desc(1, 16, 4, torch.bfloat16, N=96)
    assert call(ctypes.byref(d96), ctypes.byref(gd), *([P] * 9)) == L.ERR_UNSUPPORTED
    d0 = L.make_desc(1, 0, 4, torch.bfloat16, N=128)                # nothing to do, no launch
    assert call(ctypes.byref(d0), ctypes.byref(gd), *([None] * 9)) == L.OK


def test_state_compose_validation_codes(L):
    import torch
    lib = L.lib()
    vp = ctypes.c_void_p
    P = vp(FAKE)
    d = L.make_desc(2, 1, 3, torch.float32)
    call = lambda desc, S, Pm, U, out, tr=0: lib.wkv7_state_compose(desc, S, Pm, U, out, tr, None)   # noqa: E731
    assert call(None, P, P, P, vp(FAKE + 4096)) == L.ERR_NULL
    assert call(ctypes.byref(d), P, P, P, None) == L.ERR_NULL                     # out
    assert call(ctypes.byref(d), P, None, P, vp(FAKE + 4096)) == L.ERR_NULL       # S without P
    assert call(ctypes.byref(d), vp(FAKE + 8), P, P, vp(FAKE + 4096)) == L.ERR_ALIGN
    assert call(ctypes.byref(d), P, vp(FAKE + 4096), P, vp(FAKE + 4096)) == L.ERR_UNSUPPORTED   # out == P
    assert call(ctypes.byref(d), vp(FAKE + 4096), P, P, vp(FAKE + 4096)) == L.ERR_UNSUPPORTED   # out == S
    bad = L.make_desc(2, 1, 3, torch.float32, N=96)
    assert call(ctypes.byref(bad), P, P, P, vp(FAKE + 4096)) == L.ERR_UNSUPPORTED
    bad = L.make_desc(2, 1, 3, torch.float32, flags=L.FLAG_LOG_DECAY)
    assert call(ctypes.byref(bad), P, P, P, vp(FAKE + 4096)) == L.ERR_UNSUPPORTED
    d0 = L.make_desc(0, 1, 3, torch.float32)
    assert call(ctypes.byref(d0), None, None, None, None) == L.OK               # no units, no launch


def test_plain_c_program_links_and_calls_the_library(L, tmp_path):
    """The boundary is a C ABI: a C99 program compiles against include/wkv7.h with -pedantic, links
    libwkv7.so and gets status codes back from it without a GPU (validation runs before anything
    touches a device)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use.c"
    src.write_text(r"""
#include <stdio.h>
#include <string.h>
#include "wkv7.h"
int main(void) {
  wkv7_desc_t d;
  memset(&d, 0, sizeof d);
  d.B = 1; d.T = 16; d.H = 1; d.N = 96; d.dtype = WKV7_BF16; d.algo = WKV7_ALGO_AUTO;
  if (wkv7_version() < 100) return 2;
  if (wkv7_forward(&d, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0) != WKV7_ERR_UNSUPPORTED) return 3;
  d.N = 64;
  if (wkv7_workspace_bytes(&d) != 64u * 64u * 4u + 16u) return 4;
  if (wkv7_forward(NULL, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0) != WKV7_ERR_NULL) return 5;
  printf("%s\n", wkv7_status_string(WKV7_ERR_SHAPE));
  return 0;
}
""")
    exe = tmp_path / "use"
    libdir = os.path.dirname(L.LIB_PATHS["release"])
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", f"-I{os.path.join(ROOT, 'include')}",
                    str(src), f"-L{libdir}", "-lwkv7", f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True)
    assert res.returncode == 0, (res.returncode, res.stderr)
    assert res.stdout.strip()
