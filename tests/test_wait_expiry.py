"""Bounded-wait expiry on the GPU without a fault.

Every wait of a kernel role on its ring is bounded; when one expires the kernel records
CK_ERR_TIMEOUT in the caller's status word, stops issuing work, waits (with the normal bound)
for the copies and MMAs it already issued, frees its tensor memory and returns.  The library
build libck_test_waits.so limits every role wait to zero cycles, so each kernel below takes
that path on an ordinary input: the call must return CK_OK, the status must read
CK_ERR_TIMEOUT after a synchronise, and the context must stay usable: a normal call
afterwards gives the oracle's result.  Nothing here traps, faults or hangs the GPU.
"""
from __future__ import annotations

import os

import numpy as np
import pytest
import torch

import oracle
from rotated_w4a4_quantized_group_b200 import ck
from rotated_w4a4_quantized_group_b200 import workloads as W

pytestmark = pytest.mark.gpu

TEST_LIB = os.path.join(os.path.dirname(ck.LIB_PATH), "libck_test_waits.so")


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return ck.load_library(TEST_LIB)


def _stage1(L, x, R, g, status):
    M, K = x.shape
    codes = torch.empty(M, K, dtype=torch.int8, device="cuda")
    scales = torch.empty(M, dtype=torch.float32, device="cuda")
    return L.ck_rotate_quant(x.data_ptr(), ck.DTYPE_CODE[x.dtype], M, K, x.stride(0), x.stride(1),
                             R.data_ptr(), g, None, codes.data_ptr(), K, scales.data_ptr(),
                             status.data_ptr(), torch.cuda.current_stream().cuda_stream)


def _healthy():
    """A normal call on the same context still matches the oracle."""
    case = W.LINEAR_CASES[W.HEADLINE].replace(M=64, N=96, K=256, seed=3)
    inp = W.make_linear_inputs(case)
    out = ck.ck_w4a4_linear(inp["x"].cuda(), inp["R"].cuda(), case.g, inp["w_packed"].cuda(),
                            inp["w_scale"].cuda(), inp["bias"].cuda())
    torch.cuda.synchronize()
    ref, oc, os_ = oracle.linear(inp["x"], inp["R"], case.g, inp["w_packed"], inp["w_scale"],
                                 inp["bias"])
    err = (out.cpu().double() - ref.double()).abs()
    assert bool((err <= 1e-2 + 2e-2 * ref.double().abs()).all())


@pytest.mark.parametrize("what,dt,g,M,K,layout", [
    ("tensor-core stage 1", torch.bfloat16, 64, 512, 3840, "row"),
    ("tensor-core stage 1, split rows", torch.bfloat16, 64, 64, 10240, "row"),
    ("warp-per-row stage 1", torch.bfloat16, 16, 512, 3856, "row"),
    ("block-ring stage 1", torch.float16, 16, 64, 32768, "row"),
    ("fp32 stage 1, row-major", torch.float32, 16, 512, 3840, "row"),
    ("fp32 stage 1, column-major cluster", torch.float32, 16, 512, 3840, "col"),
    ("fp32 split-TF32 stage 1", torch.float32, 64, 512, 3840, "row"),
    ("fp32 split-TF32 stage 1, split rows", torch.float32, 64, 64, 10240, "row"),
    ("fp32 g = 256 FFMA stage 1", torch.float32, 256, 64, 3840, "row")])
def test_stage1_wait_expiry_returns_a_status(L, what, dt, g, M, K, layout):
    x = torch.randn(M, K).to(dt)
    if layout == "col":
        x = x.t().contiguous().t()
    x = x.cuda() if layout == "row" else x.t().cuda().t()
    R = W.hadamard(g).to(dt).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert _stage1(L, x, R, g, status) == ck.CK_OK
    torch.cuda.synchronize()
    assert status.item() == ck.CK_ERR_TIMEOUT, what
    _healthy()


@pytest.mark.parametrize("what,M,N,K", [("persistent GEMM", 1024, 512, 1024),
                                        ("split-K GEMM", 16, 512, 1024)])
def test_gemm_wait_expiry_returns_a_status(L, what, M, N, K):
    q = torch.randint(-8, 8, (M, K), dtype=torch.int8, device="cuda")
    wp = torch.randint(-128, 128, (N, K // 2), dtype=torch.int8, device="cuda")
    a = torch.ones(M, device="cuda")
    ws = torch.ones(N, device="cuda")
    out = torch.empty(M, N, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = L.ck_w4a4_linear(q.data_ptr(), ck.CK_I8, M, K, K, 1, None, 0, a.data_ptr(), wp.data_ptr(),
                          N, K // 2, ws.data_ptr(), ck.CK_F32, None, out.data_ptr(), ck.CK_F32, N,
                          None, 0, status.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == ck.CK_OK
    torch.cuda.synchronize()
    assert status.item() == ck.CK_ERR_TIMEOUT, what
    _healthy()
