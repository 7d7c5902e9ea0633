"""Build the CUDA library libck.so (sm_100a) in-tree, next to this file.

    python -m rotated_w4a4_quantized_group_b200.build [--force]

Compiles every csrc/*.cu with nvcc for sm_100a and links them into one shared
library exporting the C ABI declared in include/ck.h.  It also builds
libck_test_waits.so, the same sources with every role wait limited to zero cycles,
which the bounded-wait expiry test loads to drive each kernel through its timeout path.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libck.so")
# variant name -> (output library, extra nvcc flags)
VARIANTS = {
    None: (LIB, []),
    "test_waits": (os.path.join(HERE, "libck_test_waits.so"), ["-DCK_ROLE_WAIT_LIMIT_CYCLES=0"]),
}

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-I" + INCLUDE, "-I" + CSRC,
              "--expt-relaxed-constexpr", "-Xptxas", "-warn-spills"]


def nvcc() -> str:
    p = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(p):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libck.so")
    return p


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h")) + [__file__]


def needs_build(variant=None) -> bool:
    lib = VARIANTS[variant][0]
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in _deps())


def _compile(src: str, out_dir: str, extra: list) -> str:
    obj = os.path.join(out_dir, os.path.basename(src) + ".o")
    cmd = [nvcc(), *ARCH, *NVCC_FLAGS, *extra, "-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    return obj


def build(force: bool = False, variant=None) -> str:
    lib, extra = VARIANTS[variant]
    if not force and not needs_build(variant):
        return lib
    out_dir = BUILD_DIR if variant is None else os.path.join(BUILD_DIR, variant)
    os.makedirs(out_dir, exist_ok=True)
    srcs = _sources()
    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(lambda s: _compile(s, out_dir, extra), srcs))
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs, "-Xcompiler", "-fPIC"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


def build_all(force: bool = False) -> list:
    return [build(force, v) for v in VARIANTS]


if __name__ == "__main__":
    print(build_all(force="--force" in sys.argv))
