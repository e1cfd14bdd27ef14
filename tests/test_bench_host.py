"""Host-side logic of bench.py that its JSON line rests on, without a GPU:
the peak denominators, the DRAM-traffic records and their staleness check,
and the summary of the clock samples taken during the timed region."""
from __future__ import annotations

import json
import os
import shutil

import pytest

import bench


@pytest.fixture
def tree(tmp_path, monkeypatch):
    """A scratch repository root with a copy of the kernel sources."""
    src = os.path.join(bench.ROOT, "softmax_cross_entropy_lse_b200", "csrc")
    dst = tmp_path / "softmax_cross_entropy_lse_b200" / "csrc"
    shutil.copytree(src, dst)
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    return tmp_path


def test_peaks_measured_or_fallback(tree):
    assert bench.load_peaks() == (6650.0, 1590.0, 1400.0, "fallback")
    (tree / "MEASURED_PEAKS.json").write_text(json.dumps(
        {"hbm_gbs": 6547.2, "bf16_tflops": 1630.0, "bf16_tflops_sustained": 1383.8}))
    assert bench.load_peaks() == (6547.2, 1630.0, 1383.8, "measured")


def test_traffic_record_valid_only_on_its_sources(tree):
    files = bench.PASS_SOURCES["backward"]
    rec = {"c2": {"backward": {"bytes_per_launch": 1234, "source_sha": bench.kernel_source_sha(files)},
                  "forward": {"bytes_per_launch": 99, "source_sha": "0" * 16}}}
    (tree / "profiles" / "dram_traffic.json").write_text(json.dumps(rec))
    assert bench.recorded_traffic("c2", "backward") == 1234
    assert bench.recorded_traffic("c2", "forward") is None      # taken on other sources
    assert bench.recorded_traffic("c3a", "backward") is None    # no record
    # an edit to any listed source makes the record stale
    p = tree / "softmax_cross_entropy_lse_b200" / "csrc" / "ce_rows_bwd.cu"
    p.write_text(p.read_text() + "\n// edit\n")
    assert bench.recorded_traffic("c2", "backward") is None
    # an entry naming its own sources is checked against those only
    rec["c2"]["backward"]["sources"] = ["ce_rows_kl.cu"]
    rec["c2"]["backward"]["source_sha"] = bench.kernel_source_sha(["ce_rows_kl.cu"])
    (tree / "profiles" / "dram_traffic.json").write_text(json.dumps(rec))
    assert bench.recorded_traffic("c2", "backward") == 1234


def test_committed_traffic_records_are_well_formed():
    with open(os.path.join(bench.ROOT, "profiles", "dram_traffic.json")) as f:
        d = json.load(f)
    for workload, passes in d.items():
        for kernel, e in passes.items():
            assert kernel in ("forward", "backward"), (workload, kernel)
            assert isinstance(e["bytes_per_launch"], int) and e["bytes_per_launch"] > 0
            assert len(e["source_sha"]) == 16 and "--clock-control none" in e["command"]
            for f in e.get("sources") or bench.PASS_SOURCES[kernel]:
                assert os.path.exists(os.path.join(bench.ROOT, "softmax_cross_entropy_lse_b200",
                                                   "csrc", f)), f


def clock_line(sm, power, reasons=("Not Active",) * 4):
    return f"0, {sm}, 1965, {power}, 0x0000000000000000, " + ", ".join(reasons) + "\n"


def sampler(tmp_path, lines):
    cs = bench.ClockSampler(0)
    cs.path = str(tmp_path / "clocks.csv")
    cs.proc = object()  # as if nvidia-smi had been started
    with open(cs.path, "w") as f:
        f.writelines(lines)
    return cs


def test_clock_summary_uses_loaded_samples_and_lists_reasons(tmp_path):
    lines = [clock_line(345, 120.0), clock_line(1965, 610.5), clock_line(1800, 990.0,
             ("Not Active", "Not Active", "Not Active", "Active")), clock_line(1900, 700.0),
             "garbage line\n", "0, [N/A], 1965, 300, 0x0, Not Active, Not Active, Not Active, Not Active\n"]
    s = sampler(tmp_path, lines).summary()
    # the idle sample (under 200 W) is left out of the median; malformed lines are skipped
    assert s == {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                 "samples": 4, "power_w_max": 990.0}


def test_clock_summary_reports_slowdowns_and_missing_samples(tmp_path):
    s = sampler(tmp_path, [clock_line(1200, 800.0, ("Active", "Not Active", "Active", "Not Active"))]).summary()
    assert s["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert sampler(tmp_path, ["nothing useful\n"]).summary() is None
    cs = bench.ClockSampler(0)  # nvidia-smi never started
    assert cs.summary() is None


def test_roofline_reports_measured_and_spec_fractions():
    r = bench.roofline("hbm", "backward", 6000.0, 6547.2, "measured", None, 123)
    assert r["frac"] == round(6000.0 / 6547.2, 4) and r["unit"] == "GB/s"
    assert r["spec_peak"] == 8000.0 and r["frac_of_spec"] == 0.75
    assert r["algorithmic_bytes_per_launch"] == 123
    t = bench.roofline("tensor", "forward", 1125.0, 1383.8, "measured (sustained)", 5, 7)
    assert t["unit"] == "TFLOP/s" and t["frac_of_spec"] == 0.5 and t["traffic"] == 5
    assert t["algorithmic_flop_per_launch"] == 7


def test_workload_summary_keeps_the_rates_and_evidence():
    line = {"metric": "m", "value": 1.0, "unit": "GB/s", "n_gpus": 1, "fwd_GBs": 2.0,
            "roofline": {"frac": 0.5}, "clocks": {"sm_mhz": 1965.0}, "e2e": {"value": 0.1},
            "config": {"workload": "c3a"}, "cpu_baseline": {"value": 1}}
    s = bench.workload_summary(line)
    assert set(s) == {"value", "unit", "fwd_GBs", "roofline", "clocks", "e2e", "config"}
