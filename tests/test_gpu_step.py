"""GPU decode step parity: 128 ragged steps on 256 x 32 resident fp32 states."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from linear_recurrent_lm_b200 import inputs as I
from tests.gpu_util import f64, to_dev
from tests.metrics import err_rms, err_rms_excess

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def W():
    import torch
    from linear_recurrent_lm_b200 import wkv7
    torch.cuda.set_device(0)
    return wkv7


def test_config4_ragged_decode(W):
    """All 256 rows x 32 heads, 128 ragged steps: y of every step and the final states against the
    oracle stepped alongside; padded rows keep their state bit for bit and get y = 0."""
    import torch
    wl = I.make_workload(4)
    state = to_dev(wl.state0)
    st_o = wl.state0.astype(np.float64)
    max_ey = 0.0
    for s, step_in in enumerate(wl.steps):
        act = wl.active(s)
        before = state.clone()
        y = W.step(*(to_dev(step_in[n]) for n in I.NAMES), state, to_dev(act))
        inactive = torch.from_numpy(act == 0).to(state.device)
        # padded rows: state bitwise unchanged, y = 0
        assert torch.equal(state[inactive], before[inactive])
        assert torch.count_nonzero(y[inactive]) == 0
        yo, st_o = oracle.step(*(I.to_f64(step_in[n]) for n in I.NAMES), st_o, act)
        max_ey = max(max_ey, err_rms_excess(f64(y), yo, "bf16"))
    es = err_rms(f64(state), st_o)
    print(f"decode: y {max_ey:.5f}, state {es:.2e}")
    assert max_ey <= 2e-2
    assert es <= 2e-2


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
def test_step_equals_one_token_forward(W, dtype):
    import torch
    rng = np.random.default_rng(3)
    d = I.draw_inputs(rng, (5, 1, 3, 64), dtype)
    s0 = rng.standard_normal((5, 3, 64, 64)).astype(np.float32)
    y_f, s_f, _ = W.forward(*(to_dev(d[n]) for n in I.NAMES), s0=to_dev(s0), algo="scan")
    st = to_dev(s0)
    y_s = W.step(*(to_dev(d[n][:, 0]) for n in I.NAMES), st)
    yo, so, _ = oracle.forward(*(I.to_f64(d[n]) for n in I.NAMES), s0=s0)
    tol = {"f32": 1e-4, "bf16": 2e-2, "f16": 5e-3}[dtype]
    assert err_rms_excess(f64(y_s), yo[:, 0], dtype) <= tol
    assert err_rms(f64(st), so) <= 1e-4
    assert err_rms(f64(st), f64(s_f)) <= 1e-5


@pytest.mark.parametrize("B,H", [(3, 2), (64, 8)])
def test_back_to_back_steps_see_each_others_state(W, B, H):
    """Steps launched back to back with no host work between them: every step must read the
    state its predecessor wrote (the launches overlap their predecessors' tails), whether the
    batch needs fewer CTAs than the GPU holds or many units per CTA."""
    import torch
    rng = np.random.default_rng(11)
    n_steps = 24
    toks = [I.draw_inputs(rng, (B, 1, H, 64), "bf16") for _ in range(n_steps)]
    acts = [(rng.random(B) < 0.8).astype(np.uint8) for _ in range(n_steps)]
    s0 = (0.1 * rng.standard_normal((B, H, 64, 64))).astype(np.float32)
    dev_in = [[to_dev(t[n][:, 0]) for n in I.NAMES] for t in toks]
    dev_act = [to_dev(a) for a in acts]
    ys = [torch.empty_like(dev_in[0][0]) for _ in range(n_steps)]
    state = to_dev(s0)
    torch.cuda.synchronize()
    for s in range(n_steps):
        W.step(*dev_in[s], state, dev_act[s], y=ys[s])
    torch.cuda.synchronize()
    st_o = s0.astype(np.float64)
    for s in range(n_steps):
        yo, st_o = oracle.step(*(I.to_f64(toks[s][n][:, 0], "bf16") for n in I.NAMES), st_o, acts[s])
        assert err_rms_excess(f64(ys[s]), yo, "bf16") <= 2e-2
    assert err_rms(f64(state), st_o) <= 2e-2
