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


def test_reference_arm_line(monkeypatch, capsys):
    # the oracle arm's JSON line, with the timed oracle sample stubbed (its real
    # run takes about ten seconds a step)
    import json
    import numpy as np
    monkeypatch.setattr(bench, "make_inputs",
                        lambda rank, n=None, workload="down_proj_70b": (
                            np.zeros((8, 8), np.float32), np.zeros((4, 8), np.uint16), None))
    monkeypatch.setattr(bench, "oracle_sample", lambda *a, **k: (2.0, "stub sample"))
    assert bench.main(["--impl", "reference", "--steps", "2", "--warmup", "3"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["value"] == pytest.approx(8192 * 28672 / 2.0 / 1e6)  # the 70B down_proj layer
    assert line["higher_is_better"] is True and line["steps"] == 2 and line["warmup"] == 3
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline"]["sample"] == "stub sample"
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"],
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert "workload" in line["config"] and "model" not in line["config"]


def test_warmup_below_three_is_refused():
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2"])


def test_phase_rooflines():
    # q_proj 4096^2, 131072 samples; 1 ms per phase
    ph = {k: 1.0 for k in ("hessian", "factor", "sweep", "pack", "error")}
    r = bench.phase_rooflines(ph, 4096, 4096, 131072, 1600.0, 6500.0)
    assert r["hessian"]["achieved"] == pytest.approx(131072 * 4096 * 4097 / 1e-3 / 1e12)
    assert r["hessian"]["frac"] == pytest.approx(r["hessian"]["achieved"] / 1600.0)
    # FP64-grade products: INT8 = 2 x bf16, 15 digit products (factor and sweep)
    assert r["factor"]["peak"] == pytest.approx(3200.0 / 15)
    assert r["factor"]["achieved"] == pytest.approx(4096 ** 3 / 3 / 1e-3 / 1e12)
    assert r["sweep"]["peak"] == pytest.approx(3200.0 / 15)
    assert r["sweep"]["achieved"] == pytest.approx(4096 ** 3 / 1e-3 / 1e12)
    assert r["pack"]["achieved"] == pytest.approx(4096 * 4096 * 9.5 / 1e-3 / 1e9)
    assert r["pack"]["unit"] == "GB/s"
    assert bench.phase_rooflines({}, 8, 8, 8, 1.0, 1.0) == {}
