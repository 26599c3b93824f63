"""GPU forward parity against the CPU oracle (both algorithms, all dtypes)."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from linear_recurrent_lm_b200 import inputs as I
from tests.gpu_util import checkpoint_states, f64, inputs_dev, inputs_f64, to_dev
from tests.metrics import err_rms, err_rms_excess

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2, "f16": 5e-3}
# "chunked" picks one of the two chunked forms by size; the tests force each of them.
ALGOS = ("scan", "chunked_fused", "chunked_split")


@pytest.fixture(scope="module")
def W():
    import torch
    from linear_recurrent_lm_b200 import wkv7
    torch.cuda.set_device(0)
    return wkv7


def run_fwd(W, d, s0=None, reset=None, algo="auto"):
    y, s, ws = W.forward(*inputs_dev(d), s0=None if s0 is None else to_dev(s0),
                         reset=None if reset is None else to_dev(reset), algo=algo)
    return y, s, ws


def check_fwd(y, s, yo, so, dtype, algo="scan"):
    tol = TOL[dtype]
    ey = err_rms_excess(f64(y), yo, dtype)
    es = err_rms(f64(s), so)
    assert ey <= tol, ("y", ey)
    assert es <= tol, ("s_out", es)
    return ey, es


@pytest.mark.parametrize("algo", ("auto", "scan"))
def test_config0_fp32(W, algo):
    """B=1, T=64, H=2, fp32 inputs, zero initial state: max|err|/RMS <= 1e-4 (AUTO runs the scan)."""
    wl = I.make_workload(0)
    y, s, _ = run_fwd(W, wl.inputs, algo=algo)
    yo, so, _ = oracle.forward(*inputs_f64(wl.inputs))
    assert err_rms(f64(y), yo) <= 1e-4
    assert err_rms(f64(s), so) <= 1e-4


@pytest.mark.parametrize("algo", ("chunked", "chunked_fused", "chunked_split"))
def test_chunked_algos_refuse_fp32_inputs(W, algo):
    """The chunked kernels' tf32 products cannot meet the f32 bound: an explicit request is refused
    before anything runs, and the outputs are left untouched."""
    import torch
    wl = I.make_workload(0)
    xs = inputs_dev(wl.inputs)
    y = torch.full_like(xs[0], 7.0)
    with pytest.raises(W.WKV7Error) as e:
        W.forward(*xs, algo=algo, y=y)
    assert e.value.status == W.ERR_UNSUPPORTED
    assert torch.all(y == 7.0)


@pytest.mark.parametrize("algo", ALGOS)
def test_config1_forward_and_checkpoints(W, algo):
    import torch
    wl = I.make_workload(1)
    y, s, ws = run_fwd(W, wl.inputs, algo=algo)
    yo, so, _ = oracle.forward(*inputs_f64(wl.inputs))
    check_fwd(y, s, yo, so, "bf16")
    # checkpoint c holds the state after token 16c+15: compare with the oracle run to that token
    ck = checkpoint_states(ws, 2, 12, 32)
    for c in (0, 7, 31):
        part = {n: wl.inputs[n][:, : 16 * (c + 1)] for n in I.NAMES}
        _, sc, _ = oracle.forward(*inputs_f64(part))
        assert err_rms(ck[:, :, c], sc) <= 2e-2


@pytest.mark.parametrize("algo", ALGOS)
def test_config2_prefill_chained_equals_single(W, algo):
    """1.5B-model shape: s0 from 256 prior tokens, then 1024 tokens; equals one 1280-token call."""
    import torch
    wl = I.make_workload(2)
    _, s_prior, _ = run_fwd(W, wl.prior, algo=algo)
    # inference call: no checkpoints wanted, but the split form needs the workspace for its first pass
    y, s, _ = W.forward(*inputs_dev(wl.inputs), s0=s_prior, algo=algo, need_workspace=algo == "chunked_split")
    full = {n: np.concatenate([wl.prior[n], wl.inputs[n]], axis=1) for n in I.NAMES}
    yf, sf, _ = run_fwd(W, full, algo=algo)
    # split at a multiple of 16: the same arithmetic in the same order
    assert torch.equal(yf[:, 256:], y) and torch.equal(sf, s)
    yo, so, _ = oracle.forward(*inputs_f64(full))
    check_fwd(y, s, yo[:, 256:], so, "bf16")


@pytest.fixture(scope="module")
def config3_oracle():
    """Workload 3 (B=8, T=4096, H=32, packed documents): the oracle's y and final state of every unit."""
    wl = I.make_workload(3)
    yo, so, _ = oracle.forward(*inputs_f64(wl.inputs), reset=wl.reset)
    return wl, yo, so


@pytest.mark.parametrize("algo", ALGOS)
def test_config3_full_size_all_units(W, config3_oracle, algo):
    """B=8, T=4096, H=32 packed documents with resets, at full size on the GPU, compared on all 256
    (b,h) units and every element."""
    wl, yo, so = config3_oracle
    y, s, _ = run_fwd(W, wl.inputs, reset=wl.reset, algo=algo)
    ey, es = check_fwd(y, s, yo, so, "bf16")
    print(f"config3 {algo}: y {ey:.5f}, s_out {es:.5f}")


EDGE_T = [1, 15, 16, 17, 40, 100]


def _algo_dtype_cases():
    # f32 inputs run on the exact scan only (the chunked algos refuse them)
    return [(a, dt) for a in ALGOS for dt in ("f32", "bf16", "f16") if not (dt == "f32" and a != "scan")]


@pytest.mark.parametrize("algo,dtype", _algo_dtype_cases())
@pytest.mark.parametrize("T", EDGE_T)
def test_ragged_lengths_state_and_resets(W, algo, dtype, T):
    rng = np.random.default_rng(T)
    B, H = 2, 3
    d = I.draw_inputs(rng, (B, T, H, 64), dtype)
    s0 = rng.standard_normal((B, H, 64, 64)).astype(np.float32)
    reset = np.zeros((B, T), np.uint8)
    reset[1, 0] = 1                                  # overrides s0 for row 1
    for t in (5, 6, 16, T - 1):                      # consecutive resets, a chunk boundary, the last token
        if 0 < t < T:
            reset[0, t] = 1
    y, s, _ = run_fwd(W, d, s0=s0, reset=reset, algo=algo)
    yo, so, _ = oracle.forward(*inputs_f64(d), s0=s0, reset=reset)
    check_fwd(y, s, yo, so, dtype, algo)


@pytest.mark.parametrize("algo", ALGOS)
def test_zero_decay_and_identity_tokens(W, algo):
    """w = 0 (keeps only the last write; the chunked path must not divide by the decay) and
    identity tokens (w=1, a=b=k=0) that leave the state bitwise unchanged."""
    import torch
    rng = np.random.default_rng(9)
    d = I.draw_inputs(rng, (1, 48, 2, 64), "bf16")
    w = I.to_f64(d["w"])
    w[:, 20:23] = 0.0
    d["w"] = I.to_storage(w, "bf16")
    y, s, _ = run_fwd(W, d, algo=algo)
    yo, so, _ = oracle.forward(*inputs_f64(d))
    check_fwd(y, s, yo, so, "bf16")
    s0 = rng.standard_normal((1, 2, 64, 64)).astype(np.float32)
    ident = {n: np.zeros((1, 32, 2, 64), np.uint16) for n in I.NAMES}
    ident["w"][:] = I.f32_to_bf16_bits(np.ones(1, np.float32))[0]
    _, s2, _ = run_fwd(W, ident, s0=s0, algo=algo)
    assert torch.equal(s2.cpu(), torch.from_numpy(s0))


@pytest.mark.parametrize("algo", ALGOS)
def test_scattered_token_path_chunks_between_tensor_core_chunks(W, algo):
    """Chunks the chunked path must run token by token (w = 0 somewhere inside) scattered
    between ordinary ones, with resets and an entering state: the chunked kernel alternates its
    two paths many times within one sequence and must stay on the oracle throughout."""
    rng = np.random.default_rng(13)
    B, T, H = 2, 300, 3
    d = I.draw_inputs(rng, (B, T, H, 64), "bf16")
    w = I.to_f64(d["w"])
    w[0, [5, 100, 101, 250]] = 0.0
    w[1, [33, 34, 160, 299]] = 0.0
    d["w"] = I.to_storage(w, "bf16")
    reset = np.zeros((B, T), np.uint8)
    reset[0, [50, 180]] = 1
    reset[1, [0, 161, 200]] = 1
    s0 = rng.standard_normal((B, H, 64, 64)).astype(np.float32)
    y, s, _ = run_fwd(W, d, s0=s0, reset=reset, algo=algo)
    yo, so, _ = oracle.forward(*inputs_f64(d), s0=s0.astype(np.float64), reset=reset)
    check_fwd(y, s, yo, so, "bf16")


@pytest.mark.parametrize("algo", ALGOS)
def test_zero_tokens_and_single_unit(W, algo):
    import torch
    rng = np.random.default_rng(11)
    d = I.draw_inputs(rng, (1, 0, 1, 64), "bf16")
    s0 = rng.standard_normal((1, 1, 64, 64)).astype(np.float32)
    _, s, _ = run_fwd(W, d, s0=s0, algo=algo)
    assert torch.equal(s.cpu(), torch.from_numpy(s0))


@pytest.mark.parametrize("algo", ("chunked_fused", "chunked_split"))
def test_forward_is_deterministic(W, algo):
    import torch
    wl = I.make_workload(1)
    a = run_fwd(W, wl.inputs, algo=algo)
    b = run_fwd(W, wl.inputs, algo=algo)
    n_ck = 2 * 12 * 32 * 64 * 64 * 4          # the checkpoints; the workspace tail belongs to the backward
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1]) and torch.equal(a[2][:n_ck], b[2][:n_ck])


def test_chunked_picks_split_for_few_units_with_a_workspace(W):
    """CHUNKED runs the split form when a workspace is given and B*H fits in one CTA per SM (its
    results then equal CHUNKED_SPLIT's bit for bit), the fused form otherwise; CHUNKED_SPLIT
    without a workspace is refused before anything is launched."""
    import torch
    wl = I.make_workload(1)                                # 24 (b,h) units
    xs = inputs_dev(wl.inputs)
    ya, sa, wa = W.forward(*xs, algo="chunked")
    yb, sb, wb = W.forward(*xs, algo="chunked_split")
    assert torch.equal(ya, yb) and torch.equal(sa, sb)
    yc, sc, _ = W.forward(*xs, algo="chunked", need_workspace=False)
    yd, sd, _ = W.forward(*xs, algo="chunked_fused", need_workspace=False)
    assert torch.equal(yc, yd) and torch.equal(sc, sd)
    with pytest.raises(W.WKV7Error):
        W.forward(*xs, algo="chunked_split", need_workspace=False)


def test_split_form_reuses_buffers_across_calls(W):
    """The split form leaves its first pass's results in the checkpoint slots and in y before
    overwriting them: a second call into the same buffers with other inputs (decays that force
    some chunks onto the token path this time) must not see anything of the first."""
    import torch
    rng = np.random.default_rng(21)
    B, T, H = 2, 96, 3
    d1 = I.draw_inputs(rng, (B, T, H, 64), "bf16")
    d2 = I.draw_inputs(rng, (B, T, H, 64), "bf16")
    w2 = I.to_f64(d2["w"])
    w2[0, 20] = 0.0
    w2[1, 70] = 0.0
    d2["w"] = I.to_storage(w2, "bf16")
    y, s, ws = W.forward(*inputs_dev(d1), algo="chunked_split")
    y2, s2, ws2 = W.forward(*inputs_dev(d2), algo="chunked_split", y=y, s_out=s, workspace=ws)
    assert y2.data_ptr() == y.data_ptr() and ws2.data_ptr() == ws.data_ptr()
    yo, so, _ = oracle.forward(*inputs_f64(d2))
    check_fwd(y2, s2, yo, so, "bf16")
    ck = checkpoint_states(ws2, B, H, T // 16)
    for c in (0, 1, 4, 5):
        part = {n: d2[n][:, : 16 * (c + 1)] for n in I.NAMES}
        _, sc, _ = oracle.forward(*inputs_f64(part))
        assert err_rms(ck[:, :, c], sc) <= 2e-2


@pytest.mark.parametrize("algo", ("chunked_fused", "chunked_split"))
def test_chunked_forms_run_full_chunks_on_the_tensor_cores(W, algo):
    """Both chunked forms fall back to the exact token path only for chunks that need it: on
    ordinary decays their final state differs from the fp32 scan's by tf32 rounding (well above
    the ~1e-6 of two fp32 token-order computations) while staying inside the bf16 bound."""
    rng = np.random.default_rng(31)
    d = I.draw_inputs(rng, (2, 256, 4, 64), "bf16")
    yc, sc, _ = run_fwd(W, d, algo=algo)
    ys, ss, _ = run_fwd(W, d, algo="scan")
    assert err_rms(f64(sc), f64(ss)) > 1e-5
    yo, so, _ = oracle.forward(*inputs_f64(d))
    check_fwd(yc, sc, yo, so, "bf16")
