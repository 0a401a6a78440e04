"""Host-side arithmetic of bench.py (no GPU)."""
import pytest

import bench


def test_awq_hbm_phase_rates():
    # AWQ layer: X 16384 x 8192 bf16 (268,435,456 B read once for mean|x|);
    # W 8192^2 fp32 read once (268,435,456 B) and 20 bf16 deltas written
    # (20 x 134,217,728 B): 2,952,790,016 B
    r = bench.hbm_phase_rates({"colstats": 0.125, "quant_delta": 2.13, "error_gemm": 30.0},
                              16384, 8192, 8192, 20, 6538.3)
    assert set(r) == {"colstats", "quant_delta"}
    assert r["colstats"]["bytes"] == 268_435_456
    assert r["colstats"]["gb_per_s"] == pytest.approx(268_435_456 / 0.125e-3 / 1e9)
    assert r["colstats"]["gb_per_s"] == pytest.approx(2147.48, rel=1e-5)
    assert r["quant_delta"]["bytes"] == 2_952_790_016
    assert r["quant_delta"]["gb_per_s"] == pytest.approx(1386.3, rel=1e-4)
    assert r["quant_delta"]["frac"] == pytest.approx(1386.3 / 6538.3, rel=1e-4)


def test_awq_hbm_phase_rates_skip_missing_phases():
    assert bench.hbm_phase_rates({}, 16, 8, 8, 1, 1000.0) == {}
