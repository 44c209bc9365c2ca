"""Host-side helpers of bench.py, on CPU: the roofline blocks, the DRAM-traffic
records keyed by kernel-source hash, the per-leg clock summary and the
whole-job rate. None of them touches a GPU."""

import pytest

import bench


PEAKS = {"hbm_gbs": 6543.4, "bf16_tflops": 1617.4, "bf16_tflops_sustained": 1372.7}


def test_tensor_roofline_reports_burst_and_sustained_fractions():
    r = bench.tensor_roofline(1000.0, PEAKS, "measured", "k", 1.0e9, alg_bytes=2.0e9)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["peak"] == 1617.4 and r["frac"] == pytest.approx(1000.0 / 1617.4)
    assert r["peak_sustained"] == 1372.7 and r["frac_sustained"] == pytest.approx(1000.0 / 1372.7)
    assert r["traffic"] == 1.0e9 and r["algorithmic_bytes"] == 2.0e9
    # without a sustained figure there is no sustained fraction
    r2 = bench.tensor_roofline(1000.0, {"bf16_tflops": 1590.0}, "fallback", "k", None)
    assert "frac_sustained" not in r2 and r2["traffic"] is None


def test_hbm_roofline():
    r = bench.hbm_roofline(6543.4, PEAKS, "measured", "k", None, 123)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["frac"] == pytest.approx(1.0)
    assert r["algorithmic_bytes"] == 123


def test_recorded_traffic_matches_kernel_and_hash(tmp_path, monkeypatch):
    h = bench.kernel_source_hash("attn_fwd_kernel")
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "ncu_traffic.txt").write_text(
        "# kernel workload bytes hash source\n"
        f"attn_fwd_kernel mha8k 1000 {h} x.md\n"
        "attn_fwd_kernel mha2k 2000 0000000000000000 x.md\n")
    # the records are read under ROOT; the hash is the real sources' (taken above)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda k: h)
    assert bench.recorded_traffic("attn_fwd_kernel", "mha8k") == 1000.0
    assert bench.recorded_traffic("attn_fwd_kernel", "mha2k") is None      # other sources
    assert bench.recorded_traffic("attn_fwd_kernel", "gqa32k") is None     # no record
    assert bench.recorded_traffic("attn_fwd_kernel", "mha8k", resized=True) is None


def test_clock_summary_per_leg():
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.samples = [("mha8k", 1700), ("mha8k", 1680), ("mha8k", 1690), ("decode", 1965)]
    s.reasons = 0x4
    s.max_mhz = 1965
    out = s.summary()
    assert out["sm_mhz_per_leg"] == {"mha8k": 1690, "decode": 1965}
    assert out["reasons"] == ["sw_power_cap"] and out["samples"] == 4
    assert out["scope"] == "timed regions only"


def test_whole_job_rate_uses_the_slowest_rank():
    # 2 ranks, 1e12 units each, slowest rank 2 ms -> 1e15 units/s
    assert bench.whole_job_rate(1e12, 2.0, 2) == pytest.approx(1e15)


def test_time_stats():
    st = bench.time_stats([3.0, 1.0, 2.0])
    assert st == {"mean": 2.0, "median": 2.0, "min": 1.0}
