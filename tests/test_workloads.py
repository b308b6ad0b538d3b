"""The seeded input generator: determinism, independence of slices, scale."""
import numpy as np

import workloads as W


def test_counter_based_slices_match():
    full = W.normal(11, W.STREAM_X, (64, 48), 1.0, "bf16")
    rows = np.array([0, 5, 63, 17])
    np.testing.assert_array_equal(W.normal_rows_bf16(11, W.STREAM_X, rows, 48, 1.0), full[rows])


def test_deterministic_and_stream_separated():
    a = W.normal(3, 1, (1000,), 1.0, "f32")
    b = W.normal(3, 1, (1000,), 1.0, "f32")
    c = W.normal(3, 2, (1000,), 1.0, "f32")
    d = W.normal(4, 1, (1000,), 1.0, "f32")
    assert np.array_equal(a, b)
    assert np.abs(np.corrcoef(a, c)[0, 1]) < 0.1 and np.abs(np.corrcoef(a, d)[0, 1]) < 0.1


def test_moments_and_bf16_rounding():
    a = W.normal(5, 9, (200000,), 0.02, "f32").astype(np.float64)
    assert abs(a.mean()) < 2e-4 and abs(a.std() - 0.02) < 2e-4
    b = W.normal(5, 9, (200000,), 0.02, "bf16")
    bf = (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    # round to nearest: |bf16 - f32| <= half a bf16 ulp (2^-8 relative)
    assert np.all(np.abs(bf - a) <= np.abs(a) * 2.0 ** -8 + 1e-30)


def test_workload_table_shapes():
    wl = W.WORKLOADS["tiny_f32"]
    inp = W.make_inputs(wl)
    assert inp["x"].shape == (64, 128) and inp["x"].dtype == np.float32
    assert inp["w_gate"].shape == (4, 128, 256) and inp["w_down"].shape == (4, 256, 128)
    z = W.zipf_bias(32)
    assert z[0] == 0.0 and abs(z[31] - 0.5 * np.log(1 / 32)) < 1e-6
