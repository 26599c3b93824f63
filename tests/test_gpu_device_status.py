"""The device status word (wkv7_get_device_status) and the bounded waits behind it.

The chunked kernels stage input rows with bulk copies that complete on an
mbarrier, and every wait on it is bounded (about one second).  A wait that
runs out must not hang or fault the GPU: the kernel records it in the status
word, computes the chunk from global memory instead and finishes.  The test
hook WKV7_FLAG_TEST_WAIT_TIMEOUT makes a staging expect 16 bytes that are
never copied, so the wait runs out on purpose (nothing on the GPU faults);
the results must still match the oracle and the status must say TIMEOUT.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from linear_recurrent_lm_b200 import inputs as I
from tests.gpu_util import f64, inputs_dev, inputs_f64, to_dev
from tests.metrics import cosine, err_rms, err_rms_excess

pytestmark = pytest.mark.gpu

GRADS = ("dr", "dw", "dk", "dv", "da", "db")


@pytest.fixture(scope="module")
def W():
    import torch
    from linear_recurrent_lm_b200 import wkv7
    torch.cuda.set_device(0)
    return wkv7


def _case(T=16):
    rng = np.random.default_rng(5)
    d = I.draw_inputs(rng, (1, T, 2, 64), "bf16")
    dy = I.to_storage(rng.standard_normal((1, T, 2, 64)), "bf16")
    s0 = rng.standard_normal((1, 2, 64, 64)).astype(np.float32)
    return d, dy, s0


def test_status_is_ok_after_normal_calls(W):
    d, dy, s0 = _case(40)
    xs = inputs_dev(d)
    W.device_status(clear=True)
    _, _, ws = W.forward(*xs, s0=to_dev(s0))
    W.backward(*xs, to_dev(dy), ws, s0=to_dev(s0))
    assert W.device_status() == W.OK


def test_forward_wait_timeout_is_reported_and_results_stay_correct(W):
    d, dy, s0 = _case()
    xs = inputs_dev(d)
    W.device_status(clear=True)
    y, s, _ = W.forward(*xs, s0=to_dev(s0), flags=W.FLAG_TEST_WAIT_TIMEOUT)
    assert W.device_status(clear=False) == W.ERR_TIMEOUT
    assert W.device_status(clear=True) == W.ERR_TIMEOUT     # still set until cleared
    assert W.device_status() == W.OK
    yo, so, _ = oracle.forward(*inputs_f64(d), s0=s0.astype(np.float64))
    assert err_rms_excess(f64(y), yo, "bf16") <= 2e-2
    assert err_rms(f64(s), so) <= 2e-2


def test_backward_wait_timeout_is_reported_and_gradients_stay_correct(W):
    d, dy, s0 = _case()
    xs = inputs_dev(d)
    _, _, ws = W.forward(*xs, s0=to_dev(s0))
    W.device_status(clear=True)
    g = W.backward(*xs, to_dev(dy), ws, s0=to_dev(s0), flags=W.FLAG_TEST_WAIT_TIMEOUT)
    assert W.device_status() == W.ERR_TIMEOUT
    go, _ = oracle.backward(*inputs_f64(d), I.to_f64(dy), s0=s0.astype(np.float64))
    for n in GRADS:
        assert cosine(f64(g[n]), go[n]) >= 0.999, n
    assert cosine(f64(g["ds0"]), go["ds0"]) >= 0.999
    # the context is still usable
    _, _, ws = W.forward(*xs, s0=to_dev(s0))
    assert W.device_status() == W.OK


@pytest.mark.parametrize("algo", ("scan", "chunked_fused", "chunked_split"))
def test_check_finite_flags_nonfinite_outputs_only(W, algo):
    """WKV7_FLAG_CHECK_FINITE scans the outputs after the call: finite results leave the status
    OK; an infinity in v (which reaches y and the state) is reported as NONFINITE, and the
    results of the call are the same as without the flag."""
    import torch
    d, dy, s0 = _case(40)
    xs = inputs_dev(d)
    W.device_status(clear=True)
    y0, s_0, _ = W.forward(*xs, s0=to_dev(s0), algo=algo)
    y1, s_1, ws = W.forward(*xs, s0=to_dev(s0), algo=algo, flags=W.FLAG_CHECK_FINITE)
    assert W.device_status() == W.OK
    assert torch.equal(y0, y1) and torch.equal(s_0, s_1)
    g = W.backward(*xs, to_dev(dy), ws, s0=to_dev(s0), algo=algo, flags=W.FLAG_CHECK_FINITE)
    assert W.device_status() == W.OK
    v = I.to_f64(d["v"])
    v[0, 33, 1, 7] = np.inf
    bad = dict(d, v=I.to_storage(v, "bf16"))
    W.forward(*inputs_dev(bad), s0=to_dev(s0), algo=algo)            # unchecked: nothing recorded
    assert W.device_status() == W.OK
    W.forward(*inputs_dev(bad), s0=to_dev(s0), algo=algo, flags=W.FLAG_CHECK_FINITE)
    assert W.device_status(clear=False) == W.ERR_NONFINITE
    assert W.device_status() == W.ERR_NONFINITE                       # cleared by this read
    assert W.device_status() == W.OK
    dyb = I.to_f64(dy)
    dyb[0, 5, 0, 3] = np.nan
    W.backward(*xs, to_dev(I.to_storage(dyb, "bf16")), ws, s0=to_dev(s0), algo=algo, flags=W.FLAG_CHECK_FINITE)
    assert W.device_status() == W.ERR_NONFINITE


def test_check_finite_on_the_decode_step(W):
    rng = np.random.default_rng(8)
    d = I.draw_inputs(rng, (4, 1, 3, 64), "bf16")
    state = (0.1 * rng.standard_normal((4, 3, 64, 64))).astype(np.float32)
    W.device_status(clear=True)
    W.step(*(to_dev(d[n][:, 0]) for n in I.NAMES), to_dev(state), flags=W.FLAG_CHECK_FINITE)
    assert W.device_status() == W.OK
    state[2, 1, 10, 20] = np.inf
    W.step(*(to_dev(d[n][:, 0]) for n in I.NAMES), to_dev(state), flags=W.FLAG_CHECK_FINITE)
    assert W.device_status() == W.ERR_NONFINITE
