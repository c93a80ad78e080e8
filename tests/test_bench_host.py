"""Host-side pieces of bench.py that decide what the JSON line reports, on CPU:
the clock / throttle-reason summary of the nvidia-smi samples, and the GEMM
DRAM traffic that is reported only while the recorded ncu counters belong to
the GEMM source as it is now."""
import json

import bench


def _sampler_with(tmp_path, lines):
    s = bench.ClockSampler(0)
    s.path = str(tmp_path / "clocks.csv")
    (tmp_path / "clocks.csv").write_text("".join(l + "\n" for l in lines))
    return s


def test_clock_summary_median_max_and_reasons(tmp_path):
    na = "Not Active"
    s = _sampler_with(tmp_path, [
        f"0, 1965, 1965, 700.10, 0x0000000000000000, {na}, {na}, {na}, {na}",
        f"0, 1800, 1965, 990.00, 0x0000000000000004, {na}, {na}, {na}, Active",
        f"0, 1950, 1965, 995.00, 0x0000000000000004, {na}, {na}, {na}, Active",
    ])
    r = s.summary()
    assert r["sm_mhz"] == 1950.0 and r["sm_max_mhz"] == 1965.0 and r["samples"] == 3
    assert r["reasons"] == ["sw_power_cap"]


def test_clock_summary_flags_slowdowns_and_skips_bad_rows(tmp_path):
    na = "Not Active"
    s = _sampler_with(tmp_path, [
        f"0, [N/A], 1965, 700.10, 0x0, {na}, {na}, {na}, {na}",
        f"0, 1200, 1965, 500.00, 0x0000000000000008, Active, {na}, Active, {na}",
    ])
    r = s.summary()
    assert r["sm_mhz"] == 1200.0
    assert r["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]


def test_clock_summary_without_samples(tmp_path):
    s = bench.ClockSampler(0)
    s.path = str(tmp_path / "missing.csv")
    assert s.summary() is None


def test_recorded_traffic_only_for_the_current_gemm_source(tmp_path, monkeypatch):
    orig = bench.COUNTERS
    d = json.load(open(orig))
    per = d["gemm_dram_bytes_per_launch"]["llama3_8b_qkv_o"]
    mean, names = bench.recorded_traffic("llama3_8b_qkv_o")
    if d["gemm_source_hash"] == bench.gemm_source_hash():
        assert mean == sum(per.values()) / len(per) and names == sorted(per)
    else:
        assert (mean, names) == (None, None)
    # counters taken on another source are not reported
    stale = dict(d, gemm_source_hash="0" * 16)
    p = tmp_path / "counters.json"
    p.write_text(json.dumps(stale))
    monkeypatch.setattr(bench, "COUNTERS", str(p))
    assert bench.recorded_traffic("llama3_8b_qkv_o") == (None, None)
    assert bench.recorded_tensor_pipe("llama3_8b_qkv_o") is None
    # nor a workload without a capture
    monkeypatch.setattr(bench, "COUNTERS", orig)
    assert bench.recorded_traffic("no_such_workload") == (None, None)
    assert bench.recorded_tensor_pipe("no_such_workload") is None
    if d["gemm_source_hash"] == bench.gemm_source_hash():
        pipe = bench.recorded_tensor_pipe("llama3_8b_qkv_o")
        assert set(pipe) == set(per) and all(0.0 < v <= 100.0 for v in pipe.values())
