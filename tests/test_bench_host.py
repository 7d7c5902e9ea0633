"""Host-side helpers of bench.py, on CPU: the per-launch DRAM traffic lookup keyed by kernel
source, the clock sampler's summary (the bench rejects runs with thermal or hardware
slowdowns, so the reasons it reports must be exact), the workload description both arms
print, the roofline bound chosen per workload, and the CPU baseline's structure."""
from __future__ import annotations

import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from rotated_w4a4_quantized_group_b200 import workloads as W  # noqa: E402


def _fake_tree(tmp_path, kernel_src: bytes):
    (tmp_path / "profiles").mkdir()
    k = tmp_path / "kern.cu"
    k.write_bytes(kernel_src)
    return str(k)


def _table(tmp_path, rows):
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"rows": rows}))


def test_traffic_is_read_only_for_the_captured_source(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    k = _fake_tree(tmp_path, b"kernel v1")
    sha = bench.source_sha(k)
    _table(tmp_path, [{"kernel_file": "kern.cu", "workload": "wl", "source_sha16": sha,
                       "dram_bytes_per_launch": 1234},
                      {"kernel_file": "kern.cu", "workload": "other", "source_sha16": sha,
                       "dram_bytes_per_launch": 99}])
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


def test_committed_traffic_rows_parse():
    """Every committed row names a kernel source file of the package and a known workload."""
    d = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    assert d["rows"]
    csrc = os.path.join(ROOT, "rotated_w4a4_quantized_group_b200", "csrc")
    for r in d["rows"]:
        assert os.path.exists(os.path.join(csrc, r["kernel_file"]))
        assert len(r["source_sha16"]) == 16 and int(r["dram_bytes_per_launch"]) > 0
        assert r["command"]


def test_both_arms_print_the_same_config():
    case = W.LINEAR_CASES[W.HEADLINE]
    assert bench.config_of(case, 1) == bench.config_of(case, 1)
    assert bench.config_of(case, 2)["parallelism"] == "replicas x2"
    assert bench.config_of(case, 1)["workload"] == case.name


def test_roofline_bound_follows_operation_intensity():
    pk = {"hbm_gbs": 6550.0, "bf16_tflops": 1640.0}
    small = W.LINEAR_CASES["zimage_m32_k3840_n3840_g64_bf16"]
    big = W.LINEAR_CASES[W.HEADLINE]
    r0 = bench.gemm_roofline(small.M, small.N, small.K, small, 0.01, pk, "measured", 1965.0, None)
    assert r0["bound"] == "hbm" and r0["unit"] == "GB/s"
    assert abs(r0["achieved"] - r0["algorithmic_bytes"] / 1e-5 / 1e9) < 1e-6 * r0["achieved"]
    r1 = bench.gemm_roofline(big.M, big.N, big.K, big, 0.1, pk, "measured", 1965.0, None)
    assert r1["bound"] == "tensor" and r1["peak"] == 3280.0
    assert abs(r1["kind_i8_rate_tops"] - 148 * 8192 * 2 * 1.965e9 / 1e12) < 1e-6


def test_cpu_baseline_reports_all_cores_pinned_core_and_stage1():
    case = W.LINEAR_CASES["zimage_m32_k3840_n3840_g64_bf16"].replace(N=64)
    inp = W.make_linear_inputs(case)
    cb = bench.cpu_baseline(case, inp, 0.2)
    assert cb["kind"] == "oracle" and cb["cores"] == len(bench.host_cores())
    assert cb["value"] > 0 and cb["single_core_pinned"]["cores"] == 1
    assert cb["stage1"]["unit"] == "GB/s" and cb["stage1"]["value"] > 0
    assert cb["cpu_model"] and cb["hardware_concurrency"] >= 1


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


def test_sets_for_cover_three_l2s():
    """Launch data is cycled through copies totalling at least three L2s (and at least 3)."""
    import bench
    l2x3 = bench.L2_COLD_FOOTPRINT
    for per_set in (1, 8 << 20, 94 << 20, 165 << 20, 485 << 20, 2 << 30):
        n = bench.sets_for(per_set, 4096)
        assert n >= 3
        assert n * per_set >= l2x3 or n == 4096
        assert (n - 1) * per_set < l2x3 or n == 3
    assert bench.sets_for(1, 64) == 64


def test_step_schedule_runs_exactly_the_asked_steps():
    """The timed replays run exactly K steps: full graphs of S steps, then one graph of the
    first K mod S steps."""
    import bench
    built = []

    def partial(r):
        built.append(r)
        return ("first", r)

    for S in (1, 3, 7, 51):
        for n in (1, 2, 3, 5, 10, 50, 200):
            built.clear()
            sched = bench.step_schedule(("full", S), S, partial, n)
            steps = sum(S if g[0] == "full" else g[1] for g in sched)
            assert steps == n
            assert built == ([n % S] if n % S else [])
            assert all(g == ("full", S) for g in sched[: n // S])


def test_kernel_sources_follow_the_workload():
    import os
    import bench
    from rotated_w4a4_quantized_group_b200 import workloads as W
    for name, case in W.LINEAR_CASES.items():
        kern, gemm_file, rq_file = bench.kernel_sources(case)
        assert os.path.exists(gemm_file) and os.path.exists(rq_file)
        assert (kern == "w4a4_splitk_kernel") == (case.M <= 64)
        assert os.path.basename(rq_file) == ("ck_rq_f32.cu" if case.dtype == "f32" else "ck_rotate_quant.cu")
