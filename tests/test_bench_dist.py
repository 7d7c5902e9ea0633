"""Host side of bench.py's multi-process path, on CPU with the gloo backend (world size 2).

The GPU path runs one replica per rank (the linear has no exchange step) and times the
step as the maximum over ranks; rank 0 alone prints the JSON line.  These tests run the
same helpers and the reference arm under torchrun without a GPU.
"""
from __future__ import annotations

import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    sys.path.insert(0, ROOT)
    import bench
    w, r, _ = bench.dist_setup("gloo")
    try:
        got = bench.max_over_ranks(10.0 * r + 1.5, w)
        bench.barrier(w)
        with open(os.path.join(out_dir, f"rank{r}.txt"), "w") as f:
            f.write(repr(got))
    finally:
        torch.distributed.destroy_process_group()


def test_max_over_ranks_and_barrier_with_gloo(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    for r in range(world):
        assert float((tmp_path / f"rank{r}.txt").read_text()) == 11.5   # max(1.5, 11.5), all ranks


def test_reference_arm_under_torchrun_prints_one_line_from_rank_0():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "1", "--warmup", "0", "--workload", "zimage_m32_k3840_n3840_g64_bf16",
           "--cpu-budget", "0.05"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
