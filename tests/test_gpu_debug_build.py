"""The bounds-checked build (libwkv7_debug.so) on every form of the path.

The debug build checks each index its kernels compute against the extent of the buffer it
addresses and reports a failure through the device status word (WKV7_ERR_BOUNDS) instead of
faulting.  Here every entry point -- forward and backward under each algorithm and dtype, the
decode step and the no-allocation train step -- runs under it on shapes that reach the edge
cases (T = 1, ragged last chunks, one head, more (b, h) units than SMs, state resets, s0 and dS_T):
no check may fail, and every output must equal the release build's bit for bit.
"""
from __future__ import annotations

import zlib

import numpy as np
import pytest

from linear_recurrent_lm_b200 import inputs as I
from tests.gpu_util import to_dev

pytestmark = pytest.mark.gpu

SHAPES = [(1, 1, 1), (1, 16, 1), (2, 40, 3), (1, 100, 2), (3, 48, 64)]


@pytest.fixture(scope="module")
def W():
    import torch
    from linear_recurrent_lm_b200 import wkv7
    torch.cuda.set_device(0)
    assert wkv7.active_build() == "release"
    return wkv7


def _host_case(B, T, H, dtype, seed):
    rng = np.random.default_rng(seed)
    d = I.draw_inputs(rng, (B, T, H, 64), dtype)
    dy = I.to_storage(rng.standard_normal((B, T, H, 64)), dtype)
    s0 = rng.standard_normal((B, H, 64, 64)).astype(np.float32)
    dsT = rng.standard_normal((B, H, 64, 64)).astype(np.float32)
    reset = np.zeros((B, T), np.uint8)
    if T > 1:
        reset[0, T // 2] = 1
    if B > 1:
        reset[1, 0] = 1
    return d, dy, s0, dsT, reset


def _fwd_bwd(W, host, algo, log_decay=False):
    d, dy, s0, dsT, reset = host
    xs = [to_dev(d[n]) for n in I.NAMES]
    y, s, ws = W.forward(*xs, s0=to_dev(s0), reset=to_dev(reset), algo=algo, log_decay=log_decay)
    g = W.backward(*xs, to_dev(dy), ws, s0=to_dev(s0), reset=to_dev(reset), dsT=to_dev(dsT), algo=algo,
                   log_decay=log_decay)
    out = {"y": y, "s_out": s, **g}
    B, T, H = y.shape[:3]
    if T > 0:   # the checkpoints themselves (the backward's input) must match too
        out["ckpt"] = ws[: B * H * ((T + 15) // 16) * 64 * 64 * 4]
    return out


def _step(W, dtype, seed):
    import torch
    rng = np.random.default_rng(seed)
    B, H = 3, 5
    d = I.draw_inputs(rng, (B, 1, H, 64), dtype)
    xs = [to_dev(d[n][:, 0]) for n in I.NAMES]
    state = to_dev(rng.standard_normal((B, H, 64, 64)).astype(np.float32))
    active = to_dev(np.array([1, 0, 1], np.uint8))
    ys = []
    for _ in range(3):
        ys.append(W.step(*xs, state, active=active).clone())
    return {"y": torch.stack(ys), "state": state}


def _noalloc(W, host):
    d, dy, s0, dsT, reset = host
    xs = [to_dev(d[n]) for n in I.NAMES]
    y, s, g = W.train_step_noalloc(*xs, to_dev(dy), s0=to_dev(s0), reset=to_dev(reset), dsT=to_dev(dsT))
    return {"y": y, "s_out": s, **g}


def _cases():
    out = []
    for B, T, H in SHAPES:
        for algo in ("scan", "chunked_fused", "chunked_split"):
            for dt in ("f32", "bf16", "f16"):
                if dt == "f32" and algo != "scan":
                    continue            # refused: tf32 products cannot meet the f32 bound
                if B * H > 64 and dt != "bf16":
                    continue
                out.append(("fwd_bwd", algo, dt, (B, T, H)))
    out += [("fwd_bwd_log_decay", algo, "bf16", (2, 40, 3)) for algo in ("scan", "chunked_fused", "chunked_split")]
    out += [("step", None, dt, None) for dt in ("f32", "bf16", "f16")]
    out += [("noalloc", None, "bf16", (2, 40, 3))]
    return out


def _run(W, case, seed):
    kind, algo, dt, shape = case
    if kind == "fwd_bwd":
        return _fwd_bwd(W, _host_case(*shape, dt, seed), algo)
    if kind == "fwd_bwd_log_decay":   # x in place of w (values of a decay parameter, not of a decay)
        d, dy, s0, dsT, reset = _host_case(*shape, dt, seed)
        d["w"] = I.to_storage(-np.abs(I.to_f64(d["r"])) - 0.5, dt)
        return _fwd_bwd(W, (d, dy, s0, dsT, reset), algo, log_decay=True)
    if kind == "step":
        return _step(W, dt, seed)
    return _noalloc(W, _host_case(*shape, dt, seed))


@pytest.mark.parametrize("case", _cases(), ids=lambda c: "-".join(str(x) for x in c if x is not None))
def test_debug_build_matches_release_without_a_failed_check(W, case):
    import torch
    seed = 1000 + zlib.crc32(repr(case).encode()) % 1000
    assert W.device_status() == W.OK
    rel = _run(W, case, seed)
    assert W.device_status() == W.OK
    prev = W.use_build("debug")
    try:
        assert W.lib().wkv7_debug_checks() == 1
        assert W.device_status() == W.OK            # the debug module's own word starts clear
        dbg = _run(W, case, seed)
        st = W.device_status()
    finally:
        W.use_build(prev)
    assert st == W.OK, (case, W.lib().wkv7_status_string(st).decode())
    assert set(rel) == set(dbg)
    for n in rel:
        if rel[n] is None:
            assert dbg[n] is None
            continue
        assert torch.equal(rel[n], dbg[n]), (case, n)
