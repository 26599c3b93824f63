"""The synthetic input recipe: the generator produces the value ranges, structure and shapes
that the workloads claim, so that the parity and bench inputs stand for what they say.

Checked on the drawn arrays (no WKV-7 arithmetic involved): the decay range of the
w = exp(-exp(-softplus(-z) - 0.5)) parametrisation, unit-norm kk with a = -kk and
b = kk * sigmoid(z) in [0, kk], the geometric document packing of the training batch,
the decode workload's states and ragged lengths, and that a seed fixes every array.
"""
from __future__ import annotations

import numpy as np
import pytest

from linear_recurrent_lm_b200 import inputs as I


def _f64(d, dtype):
    return {n: I.to_f64(d[n], dtype) for n in I.NAMES}


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decay_range_and_rank_one_structure(dtype):
    rng = np.random.default_rng(3)
    x = _f64(I.draw_inputs(rng, (4, 33, 3, 64), dtype), dtype)
    w = x["w"]
    # exp(-exp(u)) with u = -softplus(-z) - 0.5 < -0.5: w in (exp(-exp(-0.5)), 1) = (0.545, 1)
    assert w.min() > 0.545 - 1e-2 and w.max() <= 1.0
    assert np.exp(-np.exp(-0.5)) == pytest.approx(0.5452, abs=1e-4)
    # a = -kk with kk unit-norm over the 64 channels of each (b, t, h)
    norms = np.sqrt(np.sum(x["a"] ** 2, axis=-1))
    tol = 1e-6 if dtype == "f32" else 2e-2
    assert np.all(np.abs(norms - 1.0) < tol)
    # b = kk * sigmoid(z): same sign as -a, magnitude at most |a|
    kk = -x["a"]
    assert np.all(x["b"] * kk >= -1e-12)
    assert np.all(np.abs(x["b"]) <= np.abs(kk) * (1 + 1e-2) + 1e-6)


def test_packed_batch_documents_are_geometric_with_mean_512():
    wl = I.make_workload(3)
    assert wl.reset.shape == (8, 4096) and wl.reset.dtype == np.uint8
    assert np.all(wl.reset[:, 0] == 1)                       # every row starts a document
    starts = [np.flatnonzero(row) for row in wl.reset]
    lengths = np.concatenate([np.diff(np.append(s, 4096))[:-1] for s in starts])   # drop each row's cut-off last doc
    assert lengths.min() >= 1
    assert 300 < lengths.mean() < 800                        # geometric, p = 1/512
    assert wl.dy.shape == (8, 4096, 32, 64)


def test_decode_workload_states_and_ragged_lengths():
    wl = I.make_workload(4)
    assert wl.state0.shape == (256, 32, 64, 64) and wl.state0.dtype == np.float32
    assert abs(float(wl.state0.std()) - 0.1) < 2e-3 and abs(float(wl.state0.mean())) < 2e-3
    assert wl.lengths.min() >= 1 and wl.lengths.max() <= 128 and len(wl.steps) == 128
    act = np.stack([wl.active(s) for s in range(128)])
    assert np.all(act[0] == 1)                               # every row decodes at least one token
    assert np.all(np.diff(act.astype(int), axis=0) <= 0)      # a row, once padded, stays padded
    assert int(act.sum()) == int(wl.lengths.sum())


def test_prefill_prior_and_seeds():
    wl = I.make_workload(2)
    assert wl.prior["r"].shape == (1, I.PRIOR_TOKENS, 32, 64)
    a, b = I.make_workload(1), I.make_workload(1)
    for n in I.NAMES:
        assert np.array_equal(a.inputs[n], b.inputs[n])
    c = I.make_workload(1, seed=7)
    assert not np.array_equal(a.inputs["r"], c.inputs["r"])


def test_bf16_storage_round_trip_is_exact_on_representable_values():
    vals = np.array([0.0, 1.0, -2.5, 0.546875, 3.0e-5, 65280.0], dtype=np.float64)
    bits = I.to_storage(vals, "bf16")
    assert bits.dtype == np.uint16
    assert np.array_equal(I.to_f64(bits, "bf16"), I.bf16_bits_to_f32(I.f32_to_bf16_bits(vals.astype(np.float32))))
    assert I.to_f64(I.to_storage(np.array([1.0 + 2.0 ** -9]), "bf16"), "bf16")[0] == 1.0   # round to nearest even


def test_gdn_inputs_recipe():
    """The gated-DeltaNet inputs: seeded, q and k per key head, v per value head, a log-decay
    g <= 0 per value head whose typical size follows A * dt, and beta in (0, 1)."""
    import numpy as np
    from linear_recurrent_lm_b200 import inputs as I
    a = I.draw_gdn_inputs(np.random.default_rng(3), 2, 64, 8, 4, 128, "bf16")
    b = I.draw_gdn_inputs(np.random.default_rng(3), 2, 64, 8, 4, 128, "bf16")
    for n in ("q", "k", "v", "g", "beta"):
        np.testing.assert_array_equal(a[n], b[n])
    assert a["q"].shape == a["k"].shape == (2, 64, 4, 128) and a["q"].dtype == np.uint16
    assert a["v"].shape == (2, 64, 8, 128)
    assert a["g"].shape == a["beta"].shape == (2, 64, 8) and a["g"].dtype == np.float32
    assert np.all(a["g"] <= 0.0) and np.all(a["g"] > -1e3)
    assert np.all((a["beta"] > 0.0) & (a["beta"] < 1.0))
    # per head the median decay is near -A dt with A in [1, 16], dt in [1e-3, 1e-1]
    med = np.median(-a["g"], axis=(0, 1))
    assert np.all(med > 1e-3 * 0.3) and np.all(med < 16 * 0.1 * 3)
