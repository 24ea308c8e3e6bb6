"""Host-side bookkeeping of bench.py, on the CPU: the clock record taken during the timed region
(which decides whether a run is kept) and the DRAM-traffic record, which must go null once the
kernel's source has changed since its counters were taken."""
import json
import os
import shutil

import pytest

import bench


def _clock_lines(rows):
    # index, clocks.sm, clocks.max.sm, power.draw, active mask, hw_slowdown, hw_thermal, sw_thermal, sw_power_cap
    return [", ".join(str(v) for v in r) for r in rows]


def test_clock_summary_median_under_load_and_reasons():
    c = bench.ClockSampler(0)
    c.lines = _clock_lines([
        (0, 345, 1965, 120.0, "0x0", "Not Active", "Not Active", "Not Active", "Not Active"),   # idle sample
        (0, 1965, 1965, 700.0, "0x0", "Not Active", "Not Active", "Not Active", "Not Active"),
        (0, 1900, 1965, 990.0, "0x4", "Not Active", "Not Active", "Not Active", "Active"),
        (0, 1950, 1965, 980.0, "0x4", "Not Active", "Not Active", "Not Active", "Active"),
    ])
    s = c.summary()
    assert s["sm_mhz"] == 1950.0            # median of the three samples above half of max
    assert s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]
    assert s["samples"] == 4


def test_clock_summary_flags_thermal_and_survives_garbage():
    c = bench.ClockSampler(0)
    c.lines = _clock_lines([
        (0, 1500, 1965, 900.0, "0x40", "Not Active", "Active", "Not Active", "Not Active"),
    ]) + ["[N/A], garbage", ""]
    s = c.summary()
    assert s["reasons"] == ["hw_thermal_slowdown"] and s["sm_mhz"] == 1500.0
    empty = bench.ClockSampler(0)
    empty.lines = []
    assert empty.summary()["sm_mhz"] is None


def test_traffic_record_goes_null_when_the_source_changes(tmp_path, monkeypatch):
    """traffic_for returns the recorded bytes only while the sha of the kernel's sources matches
    the one recorded with the counters."""
    csrc = tmp_path / "quantized_mixture_experts_align_b200" / "csrc"
    csrc.mkdir(parents=True)
    for n in ("w4a16_mma.cu", "common.cuh"):
        shutil.copy(os.path.join(bench.ROOT, "quantized_mixture_experts_align_b200", "csrc", n), csrc / n)
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    sha = bench.src_sha("w4a16_mma.cu", "common.cuh")
    rec = {"w4a16_gate_up_decode": {"bytes_per_launch": 123456789, "src_sha": sha, "how": "test"}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    assert bench.traffic_for("w4a16_gate_up_decode", sha) == 123456789
    assert bench.traffic_for("no_such_kernel", sha) is None
    with open(csrc / "w4a16_mma.cu", "a") as f:
        f.write("\n// edited\n")
    assert bench.traffic_for("w4a16_gate_up_decode", bench.src_sha("w4a16_mma.cu", "common.cuh")) is None


def test_committed_traffic_record_is_well_formed():
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "traffic.json")))
    for key, v in rec.items():
        assert v["bytes_per_launch"] > 0 and len(v["src_sha"]) == 16 and "ncu" in v["how"], key


def test_skew_roof_is_the_sum_of_per_expert_bounds():
    """An expert costs the slower of streaming its weights and its rows' FLOPs; empty experts
    cost nothing."""
    H, I, eb = 7168, 2048, 10_000_000
    gbs, tf = 5000.0, 1000.0
    one_byte_bound = eb / (gbs * 1e9) * 1e3
    assert bench.skew_roof_ms([0, 1, 0], eb, H, I, gbs, tf) == pytest.approx(one_byte_bound)
    big = 100000
    flop_ms = bench.W.moe_flops(big, 1, H, I) / (tf * 1e12) * 1e3
    assert bench.skew_roof_ms([big, 1], eb, H, I, gbs, tf) == pytest.approx(flop_ms + one_byte_bound)
