"""bench.py's host-side logic, on the CPU: the roofline's choice of peak, the clock
sampler (parsing, and a live run against a stand-in nvidia-smi), the DRAM-traffic lookup
keyed by the kernel sources' digest, and the flat per-config summary."""
import os
import stat
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_peak_follows_the_run():
    cap = {"reasons": ["sw_power_cap"]}
    assert bench.use_sustained_peak(2000.0, cap) == (True, True)        # long and capped
    assert bench.use_sustained_peak(13.5, cap) == (False, True)         # short: burst
    assert bench.use_sustained_peak(2000.0, {"reasons": []}) == (False, False)
    assert bench.use_sustained_peak(2000.0, {"reasons": ["unsampled"]}) == (False, False)
    assert bench.use_sustained_peak(1000.0, cap)[0]                     # the bound is inclusive


def _line(sm, active=("Not Active",) * 4):
    return f"0, {sm}, 1965, 900.0, 0x0, {active[0]}, {active[1]}, {active[2]}, {active[3]}"


def test_clock_summary_parses_samples_and_reasons():
    c = bench.ClockSampler(0)
    c.lines = [_line(1965), _line(1400, ("Not Active", "Not Active", "Not Active", "Active")), _line(1300),
               "garbage", _line("[N/A]")]
    s = c.summary()
    assert s["samples"] == 3 and s["sm_mhz"] == 1400 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]
    c.lines = [_line(1800, ("Active", "Not Active", "Not Active", "Not Active"))]
    assert c.summary()["reasons"] == ["hw_slowdown"]
    c.lines = []
    assert c.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}


def test_clock_sampler_live_against_a_stand_in(tmp_path, monkeypatch):
    """With a stand-in nvidia-smi that prints a sample every 50 ms, the sampler is live
    before the region starts and reads one more sample after it ends, even when the
    region is far shorter than the sampling period."""
    fake = tmp_path / "nvidia-smi"
    fake.write_text("#!/bin/sh\nwhile true; do echo '" + _line(1965) + "'; sleep 0.05; done\n")
    fake.chmod(fake.stat().st_mode | stat.S_IXUSR)
    monkeypatch.setenv("PATH", str(tmp_path) + os.pathsep + os.environ.get("PATH", ""))
    with bench.ClockSampler(0) as c:
        n_at_start = len(c.lines)
    s = c.summary()
    assert n_at_start >= 1
    assert s["samples"] >= n_at_start + 1 and s["sm_mhz"] == 1965 and s["reasons"] == []


def test_clock_sampler_without_nvidia_smi(tmp_path, monkeypatch):
    monkeypatch.setenv("PATH", str(tmp_path))
    with bench.ClockSampler(0) as c:
        pass
    assert c.summary()["reasons"] == ["unsampled"]


def test_traffic_lookup_is_keyed_by_the_source_digest():
    d = bench.source_digest()
    assert len(d) == 16 and all(ch in "0123456789abcdef" for ch in d)
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    tags = [l.split() for l in open(path) if l.strip() and not l.startswith("#")]
    for tag, digest, nbytes in tags:
        got = bench.profiled_traffic(tag)
        assert got == (float(nbytes) if digest == d else None), tag
    assert bench.profiled_traffic("no_such_kernel") is None


def test_config_summary_is_flat_and_skips_missing_entries():
    cfg = {"quant_sweep_e4m3": {"GB_per_s": 5092.64681, "frac_of_hbm": 0.78846},
           "decode_shapes": {"M16": {"frac_of_hbm": 0.7377}, "weight_only_M16": {"us": 108.992}},
           "linear_small": {"us_median": 13.568}}
    s = bench.config_summary(cfg)
    assert s == {"quant_sweep_e4m3_GB_s": 5092.6468, "quant_sweep_e4m3_frac_hbm": 0.7885,
                 "decode_M16_frac_hbm": 0.7377, "weight_only_M16_us": 108.992, "linear_small_us": 13.568}
    assert all(not isinstance(v, dict) for v in s.values())
