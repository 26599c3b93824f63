"""wkv7_train_step_noalloc: forward + backward without any caller workspace.

Some callers cannot call cudaMalloc -- their device memory belongs to another
allocator (a framework's caching allocator, a serving engine that reserves all
free memory up front) or they run where allocating is not allowed.  For them
the library keeps the checkpoint scratch in a fixed device array.  These tests
call that entry point through the C ABI on several problems in a row (each
call reuses the scratch the previous one left behind: a large problem first,
then a small one whose backward has to re-run one head exactly, then the large
one again) and require every output to equal, bit for bit, what the regular
wkv7_forward + wkv7_backward pair returns on the same inputs: both run the
same kernels in the same form.  The file is collected last.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest

from linear_recurrent_lm_b200 import inputs as I
from tests.gpu_util import to_dev

pytestmark = pytest.mark.gpu

GRADS = ("dr", "dw", "dk", "dv", "da", "db")


def _case(seed, B, T, H, zero_decay_head=None):
    rng = np.random.default_rng(seed)
    d = I.draw_inputs(rng, (B, T, H, 64), "bf16")
    if zero_decay_head is not None:          # w = 0 inside a chunk: the chunked backward marks this head
        b, t, h = zero_decay_head
        w = I.to_f64(d["w"])
        w[b, t, h] = 0.0
        d["w"] = I.to_storage(w, "bf16")
    dy = I.to_storage(rng.standard_normal((B, T, H, 64)), "bf16")
    s0 = rng.standard_normal((B, H, 64, 64)).astype(np.float32)
    dsT = rng.standard_normal((B, H, 64, 64)).astype(np.float32)
    reset = np.zeros((B, T), np.uint8)
    reset[0, T // 3] = 1
    reset[B - 1, 0] = 1
    return d, dy, s0, dsT, reset


def _noalloc_call(W, xs, dy, s0, reset, dsT):
    """Call the C entry point directly; every output buffer is the caller's."""
    import torch
    B, T, H = (int(s) for s in xs[0].shape[:3])
    y = torch.empty_like(xs[0])
    s_out = torch.empty((B, H, 64, 64), device=xs[0].device, dtype=torch.float32)
    g = {n: torch.empty_like(xs[0]) for n in GRADS}
    g["ds0"] = torch.empty((B, H, 64, 64), device=xs[0].device, dtype=torch.float32)
    desc = W.make_desc(B, T, H, xs[0].dtype)
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    st = W.lib().wkv7_train_step_noalloc(ctypes.byref(desc), *(ptr(x) for x in xs), ptr(s0), ptr(reset), ptr(y),
                                         ptr(s_out), ptr(dy), ptr(dsT), *(ptr(g[n]) for n in GRADS), ptr(g["ds0"]),
                                         ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == W.OK, W.lib().wkv7_status_string(st)
    return y, s_out, g


def test_noalloc_equals_regular_entry_points_call_after_call():
    import torch
    from linear_recurrent_lm_b200 import wkv7 as W
    torch.cuda.set_device(0)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    large = (5, 160, 32)                       # 160 heads: more than one per SM, the fused forward form
    assert large[0] * large[2] > sms
    assert W.workspace_bytes(*large) <= W.NOALLOC_SCRATCH_BYTES
    cases = ((81, large, None), (82, (2, 100, 3), (1, 37, 2)), (83, large, None))
    for seed, (B, T, H), zero in cases:
        d, dy, s0, dsT, reset = _case(seed, B, T, H, zero)
        xs = [to_dev(d[n]) for n in I.NAMES]
        dyd, s0d, dsTd, rd = to_dev(dy), to_dev(s0), to_dev(dsT), to_dev(reset)
        y, s_out, g = _noalloc_call(W, xs, dyd, s0d, rd, dsTd)
        torch.cuda.synchronize()
        y_r, s_r, ws = W.forward(*xs, s0=s0d, reset=rd)
        g_r = W.backward(*xs, dyd, ws, s0=s0d, reset=rd, dsT=dsTd)
        torch.cuda.synchronize()
        if zero is not None:                   # the regular call did mark that head for the exact re-run
            n_ck = B * H * ((T + 15) // 16) * 64 * 64 * 4
            marks = ws[n_ck:n_ck + 4 * B * H].view(torch.int32).cpu().numpy()
            assert marks[zero[0] * H + zero[2]] >= 1 and (marks != 0).sum() == 1
        assert torch.equal(y, y_r) and torch.equal(s_out, s_r), (seed, "forward")
        for n in GRADS + ("ds0",):
            assert torch.equal(g[n], g_r[n]), (seed, n)


def test_noalloc_rejects_problems_beyond_its_scratch():
    from linear_recurrent_lm_b200 import wkv7 as W
    B, T, H = 8, 4096, 32                      # 1.07 GB of checkpoints, far above the fixed 32 MiB
    assert W.workspace_bytes(B, T, H) > W.NOALLOC_SCRATCH_BYTES
    desc = W.make_desc(B, T, H, __import__("torch").bfloat16)
    fake = ctypes.c_void_p(0x10000)            # never dereferenced: the size check comes first
    st = W.lib().wkv7_train_step_noalloc(ctypes.byref(desc), *([fake] * 6), None, None, fake, None, fake, None,
                                         *([fake] * 6), None, None)
    assert st == W.ERR_SCRATCH_LIMIT


def test_noalloc_with_log_decay_equals_the_pair():
    """With the log-space decay input the no-allocation call equals forward + backward bit for bit."""
    import torch
    from linear_recurrent_lm_b200 import wkv7 as W
    torch.cuda.set_device(0)
    rng = np.random.default_rng(901)
    B, T, H = 2, 40, 3
    d = I.draw_inputs(rng, (B, T, H, 64), "bf16", log_decay=True)
    xs = [to_dev(d[n]) for n in I.NAMES]
    dy = to_dev(I.to_storage(rng.standard_normal((B, T, H, 64)), "bf16"))
    s0 = to_dev(rng.standard_normal((B, H, 64, 64)).astype(np.float32))
    dsT = to_dev(rng.standard_normal((B, H, 64, 64)).astype(np.float32))
    reset = np.zeros((B, T), np.uint8)
    reset[0, 13] = 1
    rd = to_dev(reset)
    y, s, ws = W.forward(*xs, s0=s0, reset=rd, log_decay=True)
    g = W.backward(*xs, dy, ws, s0=s0, reset=rd, dsT=dsT, log_decay=True)
    y2, s2, g2 = W.train_step_noalloc(*xs, dy, s0=s0, reset=rd, dsT=dsT, log_decay=True)
    assert torch.equal(y, y2) and torch.equal(s, s2)
    for n in GRADS + ("ds0",):
        assert torch.equal(g[n], g2[n]), n
