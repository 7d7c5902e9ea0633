"""Host-side helpers of bench.py, on CPU: the per-launch DRAM traffic lookup keyed by kernel
source, and the clock sampler's summary (the bench rejects runs with thermal or hardware
slowdowns, so the reasons it reports must be exact)."""
from __future__ import annotations

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _fake_tree(tmp_path, kernel_src: bytes):
    (tmp_path / "profiles").mkdir()
    k = tmp_path / "kern.cu"
    k.write_bytes(kernel_src)
    return str(k)


def test_traffic_is_read_only_for_the_captured_source(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    k = _fake_tree(tmp_path, b"kernel v1")
    sha = bench.source_sha(k)
    (tmp_path / "profiles" / "traffic.md").write_text(
        "| kern.cu | wl | %s | 1234 |\n| kern.cu | other | %s | 99 |\n" % (sha, sha))
    assert bench.recorded_traffic(k, "wl") == 1234
    assert bench.recorded_traffic(k, "other") == 99
    assert bench.recorded_traffic(k, "missing") is None
    with open(k, "ab") as f:                      # the kernel changed since the capture
        f.write(b" // edited")
    assert bench.recorded_traffic(k, "wl") is None


def test_traffic_without_a_table_is_none(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    k = tmp_path / "kern.cu"
    k.write_bytes(b"x")
    assert bench.recorded_traffic(str(k), "wl") is None


def test_committed_traffic_row_parses():
    """The committed table has a well-formed row for the GEMM on the headline workload."""
    rows = [l for l in open(os.path.join(ROOT, "profiles", "traffic.md"))
            if l.startswith("| ck_w4a4_gemm.cu")]
    assert rows
    cells = [c.strip() for c in rows[0].strip().strip("|").split("|")]
    assert cells[1] == "zimage_m8192_k3840_n3840_g64_bf16"
    assert len(cells[2]) == 16 and int(cells[3]) > 0


def test_clock_summary_reports_median_and_every_reason():
    c = bench.ClockSampler.__new__(bench.ClockSampler)
    c._nvml = object()
    c.samples = [(1965.0, 1965.0, [False, False, False, False]),
                 (1800.0, 1965.0, [False, False, False, True]),
                 (1900.0, 1965.0, [False, True, False, False])]
    s = c.summary()
    assert s["sm_mhz"] == 1900.0 and s["sm_max_mhz"] == 1965.0 and s["sm_mhz_min"] == 1800.0
    assert s["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    assert s["samples"] == 3 and s["source"] == "nvml"


def test_clock_summary_without_samples_says_unavailable():
    c = bench.ClockSampler.__new__(bench.ClockSampler)
    c._nvml = None
    c.samples = []
    assert c.summary()["reasons"] == ["unavailable"]


def test_clock_sampler_runs_without_a_gpu():
    """On a machine without a driver the sampler starts and stops cleanly."""
    with bench.ClockSampler(0) as c:
        pass
    assert isinstance(c.summary(), dict)
