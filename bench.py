"""Benchmark of the ConvRot W4A4 linear hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ck|reference] [--workload NAME]

One step is one pass of the whole hot path over one batch of synthetic input already
resident in HBM: stage 1 (group-wise rotation + signed-INT4 row quantization, INT8
codes) then stage 2 (W4A4 GEMM with in-shared-memory weight unpack, exact INT32
accumulation and the scale/bias epilogue), through the C ABI.  The two stages are issued
as ck_rotate_quant then ck_w4a4_linear on the codes (the same kernels ck_w4a4_linear
launches from activations) so each kernel's duration is measured with CUDA events.

Rank 0 prints one JSON line.  With N > 1 (torchrun) every rank runs its own replica of
the workload (the path has no exchange step): weak scaling, max device time over ranks.
`--impl reference` times the CPU oracle (test infrastructure, plain single-threaded C) on
a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from rotated_w4a4_quantized_group_b200 import workloads as W  # noqa: E402

METRIC = "W4A4 linear TOPS at M=8192,K=3840,N=3840 (% INT8 peak); rotate-quant GB/s"
UNIT = "TOPS"
# INT8 dense tensor throughput relative to BF16 dense on B200 (4.5 vs 2.25 PFLOP/s nominal)
INT8_OVER_BF16 = 2.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 512 << 20


# ----------------------------------------------------------------------------- helpers

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_sha(path: str) -> str:
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def recorded_traffic(kernel_file: str, workload: str):
    """DRAM bytes per launch recorded (profiles/traffic.md) from an ncu capture of this exact
    kernel source; None when no row matches the current source."""
    p = os.path.join(ROOT, "profiles", "traffic.md")
    if not os.path.exists(p):
        return None
    sha = source_sha(kernel_file)
    name = os.path.basename(kernel_file)
    with open(p) as f:
        for line in f:
            cells = [c.strip() for c in line.strip().strip("|").split("|")]
            if len(cells) >= 4 and cells[0] == name and cells[1] == workload and cells[2] == sha:
                try:
                    return int(cells[3])
                except ValueError:
                    return None
    return None


class ClockSampler:
    """Samples SM clocks and throttle reasons while the timed region runs: through NVML every
    10 ms when nvidia_ml_py is importable, else through nvidia-smi every 200 ms."""

    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.samples = []     # (sm_mhz, max_mhz, [reason flags in NAMES order])
        self._stop = threading.Event()
        self._t = None
        self._nvml = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self._bits = [pynvml.nvmlClocksThrottleReasonHwSlowdown,
                          pynvml.nvmlClocksThrottleReasonHwThermalSlowdown,
                          pynvml.nvmlClocksThrottleReasonSwThermalSlowdown,
                          pynvml.nvmlClocksThrottleReasonSwPowerCap]
        except Exception:
            self._nvml = None

    def _one(self):
        try:
            if self._nvml is not None:
                n = self._nvml
                sm = n.nvmlDeviceGetClockInfo(self._h, n.NVML_CLOCK_SM)
                mx = n.nvmlDeviceGetMaxClockInfo(self._h, n.NVML_CLOCK_SM)
                r = n.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
                self.samples.append((float(sm), float(mx), [bool(r & b) for b in self._bits]))
                return
            r = subprocess.run(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                                "--format=csv,noheader,nounits"], capture_output=True, text=True,
                               timeout=5)
            vals = [v.strip() for v in r.stdout.strip().split(",")]
            if len(vals) == 6 and vals[0].replace(".", "").isdigit():
                self.samples.append((float(vals[0]), float(vals[1]),
                                     [v.lower().startswith("active") for v in vals[2:]]))
        except Exception:
            pass

    def _loop(self):
        period = 0.01 if self._nvml is not None else 0.2
        while not self._stop.is_set():
            self._one()
            self._stop.wait(period)

    def __enter__(self):
        self._t = threading.Thread(target=self._loop, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        self._t.join(timeout=10)
        self._one()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm = [s[0] for s in self.samples]
        reasons = sorted({self.NAMES[i] for s in self.samples for i in range(4) if s[2][i]})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(s[1] for s in self.samples),
                "sm_mhz_min": min(sm), "reasons": reasons, "samples": len(sm),
                "source": "nvml" if self._nvml is not None else "nvidia-smi"}


def dist_setup(backend: str = "nccl"):
    """Process group from torchrun's environment (RANK, WORLD_SIZE, LOCAL_RANK, MASTER_*),
    with a short timeout so that ranks waiting on a lost peer end with an error.  NCCL binds
    each rank to its local GPU; gloo (CPU) serves the host-side tests."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return world, rank, local


def _reduce_device():
    return "cpu" if torch.distributed.get_backend() == "gloo" else "cuda"


def max_over_ranks(v: float, world: int) -> float:
    """The largest value over all ranks (every rank receives it)."""
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=_reduce_device())
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        torch.distributed.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


# ----------------------------------------------------------------------------- oracle (CPU)

def oracle_sample(case, inp, budget_s: float):
    """Time the CPU oracle on the first rows of the workload (all N output channels), sized
    so that it takes about budget_s seconds.  Returns (ops/s, rows, seconds)."""
    import oracle  # test infrastructure: only this CPU-baseline leg uses it
    oracle.lib()
    rows = 1
    t0 = time.perf_counter()
    oracle.linear(inp["x"], inp["R"], case.g, inp["w_packed"], inp["w_scale"], inp["bias"],
                  rows=list(range(rows)))
    dt = time.perf_counter() - t0
    rows = max(1, min(case.M, int(budget_s / max(dt, 1e-6))))
    t0 = time.perf_counter()
    oracle.linear(inp["x"], inp["R"], case.g, inp["w_packed"], inp["w_scale"], inp["bias"],
                  rows=list(range(rows)))
    dt = time.perf_counter() - t0
    return 2.0 * rows * case.N * case.K / dt, rows, dt


# ----------------------------------------------------------------------------- arms

def run_reference(args, case, world, rank):
    if rank != 0:
        return None
    inp = W.make_linear_inputs(case)
    vals = []
    rows_used = 0
    per_step = max(0.05, min(args.cpu_budget, 120.0 / max(1, args.steps + args.warmup)))
    for i in range(args.warmup + args.steps):
        v, rows, dt = oracle_sample(case, inp, per_step)
        if i >= args.warmup:
            vals.append(v)
            rows_used = rows
    value = statistics.mean(vals) / 1e12
    ms = 2.0 * case.M * case.N * case.K / (value * 1e12) * 1e3
    sample = (f"oracle linear on the first {rows_used} of {case.M} rows x all {case.N} output "
              f"channels per step (stage 1 + unpack + GEMM + epilogue), single-threaded C")
    return {
        "metric": METRIC, "value": value, "unit": UNIT, "impl": "reference", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "s8", "data": "synthetic",
        "config": {"workload": case.name, "M": case.M, "K": case.K, "N": case.N, "g": case.g,
                   "x_dtype": case.dtype},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_ck(args, case, world, rank, local):
    from rotated_w4a4_quantized_group_b200 import ck

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    inp = W.make_linear_inputs(case)
    x = inp["x"].to(dev)
    R = inp["R"].to(dev)
    wp = inp["w_packed"].to(dev)
    wsc = inp["w_scale"].to(dev)
    bias = None if inp["bias"] is None else inp["bias"].to(dev)
    M, N, K, g = case.M, case.N, case.K, case.g
    out = torch.empty(M, N, dtype=W.DTYPES[case.dtype], device=dev)
    ws = torch.empty(ck.workspace_bytes(M, N, K, wp.stride(0)), dtype=torch.uint8, device=dev)
    P = ck.workspace_codes_pitch(K)
    off = ck.workspace_scales_offset(M, K)
    codes = ws[: M * P].view(torch.int8).view(M, P)[:, :K]
    scales = ws[off: off + 4 * M].view(torch.float32)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        ck.ck_rotate_quant(x, R, g, codes=codes, scales=scales, dev_status=status, stream=stream)
        ev_mid = torch.cuda.Event(enable_timing=True)
        ev_mid.record(stream)
        ck.ck_w4a4_linear(codes, None, 0, wp, wsc, bias, a_scale=scales, out=out,
                          dev_status=status, stream=stream, workspace=ws)
        return ev_mid

    for _ in range(args.warmup):
        flush.zero_()
        step()
    barrier(world)

    evs = []
    with ClockSampler(local) as clk:
        barrier(world)
        t_wall = time.perf_counter()
        for _ in range(args.steps):
            flush.zero_()                                    # L2 flush outside the events
            e0 = torch.cuda.Event(enable_timing=True)
            e2 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            e1 = step()
            e2.record(stream)
            evs.append((e0, e1, e2))
        barrier(world)
        t_wall = time.perf_counter() - t_wall
    if status.item() != 0:
        raise RuntimeError(f"device status {status.item()}")
    stage1 = [a.elapsed_time(b) for a, b, _ in evs]
    gemm = [b.elapsed_time(c) for _, b, c in evs]
    total_ms = sum(s + t for s, t in zip(stage1, gemm))
    total_ms = max_over_ranks(total_ms, world)
    ms_per_step = total_ms / args.steps
    flops = 2.0 * M * N * K
    value = flops * world / (ms_per_step * 1e-3) / 1e12

    pk, pk_kind = peaks()
    int8_peak = pk["bf16_tflops"] * INT8_OVER_BF16
    gemm_ms = statistics.mean(gemm)
    s1_ms = statistics.mean(stage1)
    achieved = flops / (gemm_ms * 1e-3) / 1e12
    s1_bytes = W.algorithmic_bytes_rotate_quant(M, K, g, case.dtype)
    s1_gbs = s1_bytes / (s1_ms * 1e-3) / 1e9
    gemm_file = os.path.join(ROOT, "rotated_w4a4_quantized_group_b200", "csrc", "ck_w4a4_gemm.cu")
    traffic = recorded_traffic(gemm_file, case.name)

    # ---- end to end through the public call with host buffers (pinned), copies timed
    xh = torch.empty_like(inp["x"], device="cpu").pin_memory() if inp["x"].is_contiguous() \
        else inp["x"].contiguous().pin_memory()
    xh.copy_(inp["x"])
    xd = torch.empty_like(xh, device=dev)
    oh = torch.empty(M, N, dtype=out.dtype).pin_memory()
    e2e_steps = max(3, min(args.steps, 20))
    for i in range(2 + e2e_steps):
        if i == 2:
            barrier(world)
            ea = torch.cuda.Event(enable_timing=True)
            ea.record(stream)
        xd.copy_(xh, non_blocking=True)
        ck.ck_w4a4_linear(xd, R, g, wp, wsc, bias, out=out, workspace=ws, dev_status=status,
                          stream=stream)
        oh.copy_(out, non_blocking=True)
    eb = torch.cuda.Event(enable_timing=True)
    eb.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(ea.elapsed_time(eb) / e2e_steps, world)
    e2e_val = flops * world / (e2e_ms * 1e-3) / 1e12

    if rank != 0:
        return None
    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "s8", "data": "synthetic",
        "config": {"workload": case.name, "M": M, "K": K, "N": N, "g": g, "x_dtype": case.dtype,
                   "rotation": case.rotation, "l2": "flushed (512 MiB write) before every step, "
                   "outside the timed events", "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "tensor", "kernel": "w4a4_gemm_kernel", "achieved": achieved,
                     "peak": int8_peak, "unit": "TOPS", "frac": achieved / int8_peak,
                     "traffic": traffic,
                     "peak_source": f"{pk_kind} bf16 burst x {INT8_OVER_BF16} (INT8:BF16 nominal)"},
        "stage1": {"kernel": "rotate_quant", "ms": s1_ms, "algorithmic_bytes": s1_bytes,
                   "gbs": s1_gbs, "hbm_peak_gbs": pk["hbm_gbs"], "frac": s1_gbs / pk["hbm_gbs"]},
        "gemm_ms": gemm_ms,
        "e2e": {"value": e2e_val, "unit": UNIT, "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": xh.numel() * xh.element_size(),
                "d2h_bytes_per_step": oh.numel() * oh.element_size()},
        "gpu_launches": 2 * args.steps,
        "clocks": clk.summary(),
        "wall_s_timed_region": t_wall,
    }
    if not args.no_cpu_baseline and world == 1:
        v, rows, dt = oracle_sample(case, inp, args.cpu_budget)
        res["cpu_baseline"] = {"value": v / 1e12, "unit": UNIT, "cores": 1, "kind": "oracle",
                               "sample": f"oracle linear on the first {rows} of {M} rows x all "
                                         f"{N} output channels ({dt:.1f} s, single-threaded C)"}
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ck", choices=["ck", "reference"])
    ap.add_argument("--workload", default=W.HEADLINE, choices=list(W.LINEAR_CASES))
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    case = W.LINEAR_CASES[args.workload]

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        res = run_reference(args, case, int(os.environ.get("WORLD_SIZE", "1")), rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    world, rank, local = dist_setup()
    try:
        res = run_ck(args, case, world, rank, local)
        if res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
