"""ck_w4a4_linear_noalloc: the linear for callers that cannot allocate device memory (a
plugin inside a framework that owns all device memory, or a loop that must not call
cudaMalloc).  It uses the library's built-in 32 MiB scratch array instead of a workspace
and must give the same output as ck_w4a4_linear, call after call.

This file is collected last on purpose, so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process, where its first
call sets up the scratch array's address on the device.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

from rotated_w4a4_quantized_group_b200 import ck
from rotated_w4a4_quantized_group_b200 import workloads as W


def _inputs(case, dev):
    inp = W.make_linear_inputs(case)
    return {k: (None if v is None else v.to(dev)) for k, v in inp.items()}


@pytest.mark.gpu
def test_noalloc_matches_the_workspace_entry_point_on_consecutive_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda", 0)
    # the headline shape (8192 x 3840 bf16: 31.5 MB of scratch) and a second, different input
    cases = [W.LINEAR_CASES[W.HEADLINE],
             W.LINEAR_CASES[W.HEADLINE].replace(M=1000, K=1280, N=700, seed=77, rotation="hadamard")]
    for case in cases:
        inp = _inputs(case, dev)
        ref = ck.ck_w4a4_linear(inp["x"], inp["R"], case.g, inp["w_packed"], inp["w_scale"],
                                inp["bias"])
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        outs = []
        for _ in range(2):    # two calls in a row share the scratch array
            out = torch.full_like(ref, float("nan"))
            ck.ck_w4a4_linear_noalloc(inp["x"], inp["R"], case.g, inp["w_packed"], inp["w_scale"],
                                      inp["bias"], out=out, dev_status=status)
            outs.append(out)
        torch.cuda.synchronize()
        assert status.item() == 0
        for out in outs:
            # identical kernels on identical inputs: equal bit for bit (so within any tolerance)
            assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), case.name


@pytest.mark.gpu
def test_noalloc_rescratch_paths_match_bit_for_bit():
    """The two other uses of the shared array: int8 codes whose rows are not 16-byte aligned
    (re-pitched into the array) and packed weights with an odd row pitch (re-pitched after the
    codes), each compared bit for bit with ck_w4a4_linear on two calls in a row."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda", 0)
    g = torch.Generator().manual_seed(21)
    M, N, K = 300, 200, 448
    qbuf = torch.randint(-8, 8, (M, K + 5), generator=g, dtype=torch.int8).to(dev)
    q = qbuf[:, 1:1 + K]                               # row pitch K + 5, offset 1 byte
    wbuf = torch.randint(-128, 128, (N, K // 2 + 3), generator=g, dtype=torch.int8).to(dev)
    wp = wbuf[:, :K // 2]                              # row pitch K/2 + 3 bytes
    a = (torch.rand(M, generator=g) + 0.5).to(dev)
    ws = (torch.rand(N, generator=g) + 0.5).to(dev)
    b = torch.randn(N, generator=g).to(dev)
    for wts in (wp, wbuf[:, :K // 2].contiguous()):
        ref = ck.ck_w4a4_linear(q, None, 0, wts, ws, b, a_scale=a, out_dtype=torch.float32)
        for _ in range(2):
            out = torch.full_like(ref, float("nan"))
            ck.ck_w4a4_linear_noalloc(q, None, 0, wts, ws, b, out=out, a_scale=a)
            torch.cuda.synchronize()
            assert torch.equal(out.view(torch.int32), ref.view(torch.int32))
    # activations with an odd weight pitch: codes, scales and the weight copy all in the array
    case = W.LINEAR_CASES[W.HEADLINE].replace(M=257, K=640, N=190, seed=5)
    inp = _inputs(case, dev)
    wodd = torch.zeros(case.N, case.K // 2 + 7, dtype=torch.int8, device=dev)
    wodd[:, :case.K // 2] = inp["w_packed"]
    wv = wodd[:, :case.K // 2]
    ref = ck.ck_w4a4_linear(inp["x"], inp["R"], case.g, wv, inp["w_scale"], inp["bias"])
    for _ in range(2):
        out = torch.full_like(ref, float("nan"))
        ck.ck_w4a4_linear_noalloc(inp["x"], inp["R"], case.g, wv, inp["w_scale"], inp["bias"],
                                  out=out)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


@pytest.mark.gpu
def test_noalloc_at_exactly_its_limit():
    """8729 x 3840 bf16 activations need exactly 32 MiB of scratch (codes 33,519,360 bytes,
    scales 34,916 rounded up to 35,072): accepted, and equal to ck_w4a4_linear."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda", 0)
    case = W.LINEAR_CASES[W.HEADLINE].replace(M=8729, N=256, seed=9)
    assert ck.workspace_bytes(case.M, case.N, case.K, case.K // 2) == 32 << 20
    inp = _inputs(case, dev)
    ref = ck.ck_w4a4_linear(inp["x"], inp["R"], case.g, inp["w_packed"], inp["w_scale"],
                            inp["bias"])
    for _ in range(2):
        out = torch.full_like(ref, float("nan"))
        ck.ck_w4a4_linear_noalloc(inp["x"], inp["R"], case.g, inp["w_packed"], inp["w_scale"],
                                  inp["bias"], out=out)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_noalloc_refuses_one_row_past_its_limit():
    """8730 x 3840 activations need 32 MiB + 3840 bytes: refused on the host."""
    L = ck.lib()
    fake = 1 << 20
    st = L.ck_w4a4_linear_noalloc(fake, ck.CK_BF16, 8730, 3840, 3840, 1, fake, 64, None, fake,
                                  256, 1920, fake, ck.CK_BF16, None, fake, ck.CK_BF16, 256, None,
                                  None)
    assert st == ck.CK_ERR_WORKSPACE
    # misaligned int8 codes of the same size are re-pitched into the array: refused too
    st = L.ck_w4a4_linear_noalloc(fake + 1, ck.CK_I8, 8730, 3840, 3840, 1, None, 0, fake, fake,
                                  256, 1920, fake, ck.CK_BF16, None, fake, ck.CK_BF16, 256, None,
                                  None)
    assert st == ck.CK_ERR_WORKSPACE


def test_noalloc_rejects_scratch_needs_beyond_its_limit():
    """8192 x 10240 activations need 84 MB of scratch: refused on the host, nothing launched."""
    L = ck.lib()
    fake = 1 << 20
    st = L.ck_w4a4_linear_noalloc(fake, ck.CK_F16, 8192, 10240, 10240, 1, fake, 256, None, fake,
                                  3840, 5120, fake, ck.CK_F16, None, fake, ck.CK_F16, 3840, None,
                                  None)
    assert st == ck.CK_ERR_WORKSPACE
    assert "workspace" in ck.status_string(st)
