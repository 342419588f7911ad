"""Host-side checks of the FP8 input generator and of bench.py's traffic
bookkeeping (no GPU)."""
import numpy as np

from sparse_mixture_experts_aux_b200.inputs import Workload, make_fp8_weights


def test_fp8_generator_draws_only_finite_codes_covering_subnormals():
    w = Workload("gen", 4, 64, 3, 128, 1, seed=9)
    fp8 = make_fp8_weights(w, device="cpu")
    for name, shape in (("W_g", (3, 128, 64)), ("W_u", (3, 128, 64)), ("W_d", (3, 64, 128))):
        c = fp8[name].numpy()
        assert c.shape == shape and c.dtype == np.uint8
        assert not np.any((c & 0x7F) == 0x7F), "E4M3 NaN codes must never be drawn"
    allc = np.concatenate([fp8[n].numpy().ravel() for n in ("W_g", "W_u", "W_d")])
    mag = allc & 0x7F
    assert np.any((mag >= 1) & (mag <= 7)), "subnormal codes should occur"
    assert np.any(allc & 0x80) and np.any((allc & 0x80) == 0)
    sc = fp8["weight_scales"].numpy()
    assert sc.shape == (3 * 128 + 3 * 128 + 3 * 64,) and np.all(sc > 0)
    # seeded: the same workload draws the same codes
    again = make_fp8_weights(w, device="cpu")
    assert np.array_equal(again["W_g"].numpy(), fp8["W_g"].numpy())


def test_bench_reports_traffic_only_where_captured():
    import bench
    assert ("mixtral", "dtype") in bench.TRAFFIC_RATIO
    for table in (bench.TRAFFIC_RATIO, bench.DOWN_TRAFFIC_RATIO):
        for key, (ratio, case) in table.items():
            # DRAM bytes close to the algorithmic bytes: weights read about once
            assert 0.9 < ratio < 1.2, key
            assert "case" in case
    for key in (("decode", "dtype"), ("mixtral", "w8a8"), ("switch_zipf", "dtype")):
        assert key not in bench.TRAFFIC_RATIO
