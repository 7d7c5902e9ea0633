"""GPU parity of the CUDA path (through the C ABI) against the CPU oracle.

Small cases compare every output; the full-size workloads (the four linear shapes and
the 72-case rotate+quantize sweep) compare sampled rows / columns, which the oracle
evaluates one by one, in the same launch configuration the benchmark times.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from parity_util import (assert_close, compare_stage1, oracle_on_codes, output_widening,
                         widening_for_weights,
                         sample_cols, sample_rows, to_device, workspace_stage1)
from rotated_w4a4_quantized_group_b200 import ck
from rotated_w4a4_quantized_group_b200 import workloads as W

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ck.lib()
    yield
    torch.cuda.synchronize()


def _status():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def _run_linear(inp, case, ws_extra=0):
    x = to_device(inp["x"])
    R = inp["R"].cuda()
    wp = to_device(inp["w_packed"])
    ws_ = inp["w_scale"].cuda()
    b = None if inp["bias"] is None else inp["bias"].cuda()
    nbytes = ck.workspace_bytes(case.M, case.N, case.K, wp.stride(0))
    ws = torch.empty(nbytes + ws_extra, dtype=torch.uint8, device="cuda")
    st = _status()
    out = ck.ck_w4a4_linear(x, R, case.g, wp, ws_, b, workspace=ws, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    return out, ws


def _check_linear(case, rows, cols):
    inp = W.make_linear_inputs(case)
    out, ws = _run_linear(inp, case)
    dtype = DT[case.dtype]
    gcodes, gscales = workspace_stage1(ws, case.M, case.K)
    gc = gcodes[torch.from_numpy(rows).cuda()].cpu().numpy()
    gs = gscales[torch.from_numpy(rows).cuda()].cpu().numpy()
    # full oracle on the sampled rows / columns
    ref, oc, os_ = oracle.linear(inp["x"], inp["R"], case.g, inp["w_packed"], inp["w_scale"],
                                 inp["bias"], rows=rows, cols=cols)
    compare_stage1(gc, gs, oc, os_, dtype, case.name, case.g, x=inp["x"], R=inp["R"], rows=rows)
    got = out.cpu()[torch.from_numpy(rows)][:, torch.from_numpy(cols)]
    # bit-exact: the oracle's unpack + GEMM + epilogue on the GPU's own codes and scales
    exact = oracle_on_codes(gc, gs, inp["w_packed"], case.K, cols, inp["w_scale"], inp["bias"],
                            dtype)
    assert torch.equal(got.view(torch.int16 if dtype != torch.float32 else torch.int32),
                       exact.view(torch.int16 if dtype != torch.float32 else torch.int32)), \
        f"{case.name}: output differs from oracle GEMM+epilogue on identical codes"
    # tolerance against the whole oracle path on every sampled output; a row whose codes
    # differ from the oracle's at ties, or whose scale differs within its bound, gets its bound
    # widened by exactly that difference's effect
    extra = output_widening(gc, oc, gs, os_, inp["w_packed"], case.K, cols, inp["w_scale"])
    assert_close(got, ref, dtype, case.name, extra)
    return gc, oc


# ------------------------------------------------------------------- weight unpack

@pytest.mark.parametrize("N,K,ldp,ldo", [(1, 2, 1, 2), (7, 32, 16, 32), (300, 3840, 1920, 3840),
                                         (33, 48, 24, 48), (5, 96, 53, 100), (129, 256, 128, 272)])
def test_unpack_w4_bit_exact(N, K, ldp, ldo):
    g = torch.Generator().manual_seed(N * 7 + K)
    buf = torch.randint(-128, 128, (N, ldp), generator=g, dtype=torch.int8)
    packed = buf[:, : K // 2]
    out_buf = torch.full((N, ldo), 77, dtype=torch.int8, device="cuda")
    ck.ck_unpack_w4(to_device(packed), K, out=out_buf[:, :K])
    torch.cuda.synchronize()
    ref = oracle.unpack_w4(packed, K)
    np.testing.assert_array_equal(out_buf[:, :K].cpu().numpy(), ref)
    if ldo > K:
        assert (out_buf[:, K:] == 77).all()          # guard bytes untouched


def test_unpack_w4_full_weight_shapes():
    for case in W.LINEAR_CASES.values():
        inp = W.make_linear_inputs(case.replace(M=1))
        got = ck.ck_unpack_w4(inp["w_packed"].cuda(), case.K).cpu().numpy()
        rows = sample_rows(case.N, 64)
        np.testing.assert_array_equal(got[rows], oracle.unpack_w4(inp["w_packed"][rows], case.K))


# ------------------------------------------------------------------- stage 1

def _rq_case(case: W.RotateCase, rows=None):
    inp = W.make_rotate_inputs(case)
    x = to_device(inp["x"])
    codes, scales = ck.ck_rotate_quant(x, inp["R"].cuda(), case.g)
    torch.cuda.synchronize()
    rows = sample_rows(case.M) if rows is None else rows
    oc, os_ = oracle.rotate_quant(inp["x"], inp["R"], case.g, rows=rows)
    idx = torch.from_numpy(rows).cuda()
    return compare_stage1(codes[idx].cpu().numpy(), scales[idx].cpu().numpy(), oc, os_,
                          DT[case.dtype], case.name, case.g, x=inp["x"], R=inp["R"], rows=rows)


@pytest.mark.parametrize("case", W.sweep_cases(), ids=lambda c: c.name)
def test_rotate_quant_sweep_full_size(case):
    _rq_case(case)


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("g", [16, 64, 256])
@pytest.mark.parametrize("layout", ["contiguous", "pitch2k", "colmajor"])
def test_rotate_quant_small_every_row(dt, g, layout):
    case = W.RotateCase(f"small_{dt}_{g}_{layout}", M=37, K=g * 5, g=g, dtype=dt, seed=g + 3)
    inp = W.make_rotate_inputs(case)
    x = inp["x"]
    if layout != "contiguous":
        x = W._place(x.contiguous(), layout)
    codes, scales = ck.ck_rotate_quant(to_device(x), inp["R"].cuda(), g)
    torch.cuda.synchronize()
    oc, os_ = oracle.rotate_quant(x, inp["R"], g)
    compare_stage1(codes.cpu().numpy(), scales.cpu().numpy(), oc, os_, DT[dt], case.name, g,
                   x=x, R=inp["R"])


@pytest.mark.parametrize("dt", ["f16", "bf16"])
@pytest.mark.parametrize("g,groups,M", [(64, 1, 1000), (64, 127, 200), (64, 128, 160), (64, 129, 20),
                                        (64, 131, 9), (64, 160, 301), (64, 255, 7), (64, 256, 150),
                                        (64, 257, 3), (16, 516, 11), (16, 640, 200), (16, 1024, 5),
                                        (256, 1, 1000), (256, 43, 333), (256, 128, 150),
                                        (256, 129, 3)])
def test_rotate_quant_tile_shapes(dt, g, groups, M):
    """Rows of 1 to 257 groups: a tile packs floor(128 / groups) rows, so these cover a tile of
    128 one-group rows, one row of 127 or 128 groups, a ragged last tile and more tiles than SMs
    (150 rows of 128 groups).  Rows of 129 to 256 64-channel group-rows (g = 64, and g = 16 at
    K = 64 x 129 .. 64 x 256) are split in two parts of a tile, evenly or not (131 groups: 66 +
    65), 301 rows give more tiles than SMs, and the first lengths past each kernel's limit (257
    groups at g = 64, 129 at g = 256) go to other kernels.  R is a non-symmetric orthogonal
    matrix, so R and R^T give different results.  Every output is compared."""
    case = W.RotateCase(f"tiles_{dt}_{g}_{groups}", M=M, K=g * groups, g=g, dtype=dt,
                        seed=groups + g)
    x = W.make_rotate_inputs(case)["x"]
    R = W.haar_orthogonal(g, torch.Generator().manual_seed(g + groups)).to(DT[dt]).contiguous()
    codes, scales = ck.ck_rotate_quant(to_device(x), R.cuda(), g)
    torch.cuda.synchronize()
    oc, os_ = oracle.rotate_quant(x, R, g)
    compare_stage1(codes.cpu().numpy(), scales.cpu().numpy(), oc, os_, DT[dt], case.name, g,
                   x=x, R=R)


@pytest.mark.parametrize("dt", ["f16", "bf16"])
@pytest.mark.parametrize("g,K", [(16, 16384), (16, 32768), (64, 16384), (64, 32768), (256, 16384)])
def test_rotate_quant_long_rows(dt, g, K):
    """Rows longer than the row kernel's two double-buffered rows per warp hold (K > 12800 for
    16-bit inputs at g = 16 and 64), which the block-ring kernel takes, and a g = 256 row of 64
    groups (tensor-core kernel, two rows per tile).  Every output is compared."""
    case = W.RotateCase(f"long_{dt}_{g}_{K}", M=45, K=K, g=g, dtype=dt, seed=K // g)
    x = W.make_rotate_inputs(case)["x"]
    R = W.haar_orthogonal(g, torch.Generator().manual_seed(K + g)).to(DT[dt]).contiguous()
    codes, scales = ck.ck_rotate_quant(to_device(x), R.cuda(), g)
    torch.cuda.synchronize()
    oc, os_ = oracle.rotate_quant(x, R, g)
    compare_stage1(codes.cpu().numpy(), scales.cpu().numpy(), oc, os_, DT[dt], case.name, g,
                   x=x, R=R)


@pytest.mark.parametrize("M,groups,pitch", [(710, 5, 0), (33, 1, 0), (5, 255, 0), (3, 256, 0),
                                            (1300, 60, 64), (9, 160, 0)])
def test_rotate_quant_f32_g64_blocks(M, groups, pitch):
    """fp32 rows at g = 64 (split TF32 on tensor cores): tiles of whole rows with a ragged last
    tile (710 rows of 5 groups in tiles of 25; 33 one-group rows in one tile of 128), rows of
    60 groups two to a tile with a row pitch past K, and rows split in two parts (160 groups;
    255 and 256, the longest, one part with a group past the row).  R is a non-symmetric
    orthogonal matrix.  Every output is compared."""
    g, K = 64, 64 * groups
    case = W.RotateCase(f"f32_g64_{M}_{groups}", M=M, K=K, g=g, dtype="f32", seed=M + groups)
    x = W.make_rotate_inputs(case)["x"]
    if pitch:
        buf = torch.zeros(M, K + pitch, dtype=x.dtype)
        buf[:, :K] = x
        x = buf[:, :K]
    R = W.haar_orthogonal(g, torch.Generator().manual_seed(M * groups)).float().contiguous()
    codes, scales = ck.ck_rotate_quant(to_device(x), R.cuda(), g)
    torch.cuda.synchronize()
    oc, os_ = oracle.rotate_quant(x, R, g)
    compare_stage1(codes.cpu().numpy(), scales.cpu().numpy(), oc, os_, torch.float32, case.name,
                   g, x=x, R=R)


@pytest.mark.parametrize("M,groups,pitch", [(703, 3, 0), (100, 15, 0), (300, 15, 64), (5, 40, 0),
                                            (3, 48, 0), (150, 1, 0), (1200, 15, 0), (10000, 1, 0),
                                            (300, 64, 0), (4, 80, 0)])
def test_rotate_quant_f32_g256_blocks(M, groups, pitch):
    """fp32 rows at g = 256 (the FFMA kernel: R streams through shared memory in slices of 32
    rows, the partial sums stay in registers): blocks of 5 rows with a ragged last one (703
    rows of 3 groups), one-row blocks (15, 40 and 48 groups), a row pitch past K, one-group
    rows, several four-row blocks per CTA (1200 x 15 groups), 64-row blocks (10000 x 1 group),
    the widest row a block takes (64 groups), and a wider one (80 groups) that the generic
    kernel takes.  Each value is the in-order fp32 FMA chain.  R is a non-symmetric orthogonal
    matrix.  Every output is compared."""
    g, K = 256, 256 * groups
    case = W.RotateCase(f"f32_g256_{M}_{groups}", M=M, K=K, g=g, dtype="f32", seed=M + groups)
    x = W.make_rotate_inputs(case)["x"]
    if pitch:
        buf = torch.zeros(M, K + pitch, dtype=x.dtype)
        buf[:, :K] = x
        x = buf[:, :K]
    R = W.haar_orthogonal(g, torch.Generator().manual_seed(M * groups)).float().contiguous()
    codes, scales = ck.ck_rotate_quant(to_device(x), R.cuda(), g)
    torch.cuda.synchronize()
    oc, os_ = oracle.rotate_quant(x, R, g)
    compare_stage1(codes.cpu().numpy(), scales.cpu().numpy(), oc, os_, torch.float32, case.name,
                   g, x=x, R=R)


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
def test_rotate_quant_zero_rows_and_caller_zero_scale(dt):
    x = torch.randn(20, 128, generator=torch.Generator().manual_seed(5)).to(DT[dt])
    x[3] = 0
    x[17] = 0
    R = W.hadamard(64).to(DT[dt])
    codes, scales = ck.ck_rotate_quant(x.cuda(), R.cuda(), 64)
    torch.cuda.synchronize()
    assert not codes[3].any() and not codes[17].any()
    assert scales[3].item() == np.float32(np.finfo(np.float32).tiny)
    z = torch.zeros(1, device="cuda")
    codes0, scales0 = ck.ck_rotate_quant(x.cuda(), R.cuda(), 64, scale_in=z)
    torch.cuda.synchronize()
    oc, os_ = oracle.rotate_quant(x, R, 64, scale_in=0.0)
    np.testing.assert_array_equal(scales0.cpu().numpy(), os_)
    compare_stage1(codes0.cpu().numpy(), scales0.cpu().numpy(), oc, os_, DT[dt], "zero scale", 64,
                   x=x, R=R, scale_in=0.0)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_rotate_quant_non_finite_follows_the_oracle_convention(dt):
    x = torch.randn(4, 64, generator=torch.Generator().manual_seed(6)).to(DT[dt])
    x[1, 5] = float("nan")
    x[2, 9] = float("inf")
    R = W.hadamard(16).to(DT[dt])
    codes, scales = ck.ck_rotate_quant(x.cuda(), R.cuda(), 16)
    torch.cuda.synchronize()
    oc, os_ = oracle.rotate_quant(x, R, 16)
    gs = scales.cpu().numpy()
    assert math.isnan(gs[1]) and math.isnan(os_[1])
    assert math.isinf(gs[2]) and math.isinf(os_[2])
    np.testing.assert_array_equal(codes.cpu().numpy()[1:3], oc[1:3])
    compare_stage1(codes.cpu().numpy()[[0, 3]], gs[[0, 3]], oc[[0, 3]], os_[[0, 3]], DT[dt], "", 16,
                   x=x, R=R, rows=[0, 3])


@pytest.mark.parametrize("g", [64, 256])
def test_rotate_quant_f32_non_finite_at_wide_groups(g):
    """fp32 at g = 64 (split-TF32 tensor cores) and g = 256: a NaN makes its row's scale NaN
    and codes 0, an inf makes its row's scale inf, as in the exact rotation.  R is a Hadamard
    matrix, whose entries are exact in TF32 (its low parts are all zero), so an inf in the
    high part of a split would meet zeros; other rows follow the parity rule."""
    x = torch.randn(4, 2 * g, generator=torch.Generator().manual_seed(7))
    x[1, 5] = float("nan")
    x[2, g + 9] = float("inf")
    R = W.hadamard(g).float()
    codes, scales = ck.ck_rotate_quant(x.cuda(), R.cuda(), g)
    torch.cuda.synchronize()
    oc, os_ = oracle.rotate_quant(x, R, g)
    gs = scales.cpu().numpy()
    assert math.isnan(gs[1]) and math.isnan(os_[1])
    assert math.isinf(gs[2]) and math.isinf(os_[2])
    np.testing.assert_array_equal(codes.cpu().numpy()[1:3], oc[1:3])
    compare_stage1(codes.cpu().numpy()[[0, 3]], gs[[0, 3]], oc[[0, 3]], os_[[0, 3]], torch.float32,
                   "", g, x=x, R=R, rows=[0, 3])


def test_rotate_quant_unaligned_and_strided_views():
    base = torch.randn(50, 3 * 64 + 1, generator=torch.Generator().manual_seed(7)).to(torch.bfloat16)
    x = base[:, 1:1 + 128]                       # row pitch 193, base offset by one element
    R = W.haar_orthogonal(64, torch.Generator().manual_seed(8)).to(torch.bfloat16).contiguous()
    codes_buf = torch.full((50, 136), 55, dtype=torch.int8, device="cuda")
    codes, scales = ck.ck_rotate_quant(to_device(x), R.cuda(), 64, codes=codes_buf[:, 3:131])
    torch.cuda.synchronize()
    oc, os_ = oracle.rotate_quant(x, R, 64)
    compare_stage1(codes.cpu().numpy(), scales.cpu().numpy(), oc, os_, torch.bfloat16, "", 64,
                   x=x, R=R)
    assert (codes_buf[:, :3] == 55).all() and (codes_buf[:, 131:] == 55).all()


def test_rotate_quant_is_deterministic():
    case = W.sweep_cases()[20]
    inp = W.make_rotate_inputs(case)
    x = to_device(inp["x"])
    c1, s1 = ck.ck_rotate_quant(x, inp["R"].cuda(), case.g)
    c2, s2 = ck.ck_rotate_quant(x, inp["R"].cuda(), case.g)
    torch.cuda.synchronize()
    assert torch.equal(c1, c2) and torch.equal(s1, s2)


# ------------------------------------------------------------------- stage 2 (codes in)

@pytest.mark.parametrize("M,N,K,out_dt", [(1, 1, 2, torch.float32), (200, 300, 448, torch.float32),
                                          (129, 257, 128, torch.bfloat16),
                                          (77, 513, 3840, torch.float16),
                                          (300, 100, 48, torch.float32),
                                          # several tiles per CTA with an odd number of
                                          # 128-deep K blocks per tile
                                          (4000, 2000, 384, torch.float32)])
def test_gemm_accumulators_bit_exact(M, N, K, out_dt):
    """Unit scales, no bias, fp32 out: the output is the INT32 accumulator exactly."""
    g = torch.Generator().manual_seed(M + N + K)
    q = torch.randint(-8, 8, (M, K), generator=g, dtype=torch.int8)
    wp = torch.randint(-128, 128, (N, K // 2), generator=g, dtype=torch.int8)
    ones_w = torch.ones(N, dtype=torch.float32)
    out = ck.ck_w4a4_linear(q.cuda(), None, 0, wp.cuda(), ones_w.cuda(),
                            a_scale=torch.ones(M, device="cuda"), out_dtype=torch.float32)
    torch.cuda.synchronize()
    acc = oracle.gemm_s32(q.numpy(), oracle.unpack_w4(wp, K))
    np.testing.assert_array_equal(out.cpu().numpy(), acc.astype(np.float32))
    # with scales and bias in out_dt, against the oracle epilogue
    a = torch.rand(M, generator=g) + 0.1
    ws = (torch.rand(N, generator=g) * 0.015 + 0.005).to(out_dt)
    b = torch.randn(N, generator=g).to(out_dt)
    out2 = ck.ck_w4a4_linear(q.cuda(), None, 0, wp.cuda(), ws.cuda(), b.cuda(), a_scale=a.cuda(),
                             out_dtype=out_dt)
    torch.cuda.synchronize()
    ref = oracle.epilogue(acc, a.numpy(), ws, b, out_dt)
    assert torch.equal(out2.cpu(), ref)


def test_gemm_extreme_codes_hit_the_bound():
    M, N, K = 130, 260, 4096
    q = torch.full((M, K), -8, dtype=torch.int8)
    q[1::2] = 7
    wp = torch.full((N, K // 2), -120, dtype=torch.int8)    # 0x88: both nibbles -8
    out = ck.ck_w4a4_linear(q.cuda(), None, 0, wp.cuda(), torch.ones(N, device="cuda"),
                            a_scale=torch.ones(M, device="cuda"), out_dtype=torch.float32)
    torch.cuda.synchronize()
    o = out.cpu()
    assert (o[0::2] == 64 * K).all() and (o[1::2] == -56 * K).all()


def test_gemm_unaligned_codes_and_weights_use_the_workspace():
    M, N, K = 40, 70, 48
    g = torch.Generator().manual_seed(9)
    qbuf = torch.randint(-8, 8, (M, 53), generator=g, dtype=torch.int8)
    q = qbuf[:, 1:1 + K]                           # pitch 53, offset 1: not 16-byte aligned
    wbuf = torch.randint(-128, 128, (N, 29), generator=g, dtype=torch.int8)
    wp = wbuf[:, :K // 2]                          # pitch 29
    a = torch.rand(M, generator=g) + 0.5
    ws = torch.rand(N, generator=g) + 0.5
    dq, dw = to_device(q), to_device(wp)
    nbytes = ck.workspace_bytes(M, N, K, dw.stride(0))
    work = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    out = ck.ck_w4a4_linear(dq, None, 0, dw, ws.cuda(), a_scale=a.cuda(), workspace=work,
                            out_dtype=torch.float32)
    torch.cuda.synchronize()
    acc = oracle.gemm_s32(q.contiguous().numpy(), oracle.unpack_w4(wp, K))
    ref = oracle.epilogue(acc, a.numpy(), ws, None, torch.float32)
    assert torch.equal(out.cpu(), ref)


def test_gemm_full_size_sampled():
    """The headline shape through the codes-in path: sampled outputs bit-exact."""
    M, N, K = 8192, 3840, 3840
    g = torch.Generator().manual_seed(10)
    q = torch.randint(-8, 8, (M, K), generator=g, dtype=torch.int8)
    wp = torch.randint(-128, 128, (N, K // 2), generator=g, dtype=torch.int8)
    a = torch.rand(M, generator=g) * 0.1 + 0.01
    ws = (torch.rand(N, generator=g) * 0.015 + 0.005).to(torch.bfloat16)
    b = (torch.randn(N, generator=g) * 0.1).to(torch.bfloat16)
    out = ck.ck_w4a4_linear(q.cuda(), None, 0, wp.cuda(), ws.cuda(), b.cuda(), a_scale=a.cuda(),
                            out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    rows, cols = sample_rows(M, 64), sample_cols(N, 96)
    ref = oracle_on_codes(q.numpy()[rows], a.numpy()[rows], wp, K, cols, ws, b, torch.bfloat16)
    got = out.cpu()[torch.from_numpy(rows)][:, torch.from_numpy(cols)]
    assert torch.equal(got, ref)


def test_linear_output_guard_bytes_and_pitch():
    M, N, K = 70, 300, 256
    case = W.LinearCase("guard", M=M, K=K, N=N, g=64, dtype="bf16", rotation="haar", seed=11)
    inp = W.make_linear_inputs(case)
    big = torch.full((M + 2, N + 24), 12345.0, dtype=torch.bfloat16, device="cuda")
    view = big[1:M + 1, 8:8 + N]
    ck.ck_w4a4_linear(inp["x"].cuda(), inp["R"].cuda(), 64, inp["w_packed"].cuda(),
                      inp["w_scale"].cuda(), inp["bias"].cuda(), out=view)
    torch.cuda.synchronize()
    mask = torch.ones_like(big, dtype=torch.bool)
    mask[1:M + 1, 8:8 + N] = False
    assert (big[mask] == 12345.0).all()
    ref, _, _ = oracle.linear(inp["x"], inp["R"], 64, inp["w_packed"], inp["w_scale"], inp["bias"])
    assert_close(view.cpu(), ref, torch.bfloat16, "guard")


def test_linear_empty_rows_is_a_noop():
    out = torch.full((0, 8), 1.0, device="cuda")
    x = torch.empty(0, 64, dtype=torch.float32, device="cuda")
    ck.ck_w4a4_linear(x, torch.eye(16, device="cuda"), 16, torch.zeros(8, 32, dtype=torch.int8,
                      device="cuda"), torch.ones(8, device="cuda"), out=out)
    torch.cuda.synchronize()


# ------------------------------------------------------------------- whole linear

@pytest.mark.parametrize("name", list(W.LINEAR_CASES))
def test_linear_small_every_output(name):
    """The workload recipe at a size the oracle finishes at once; several tiles and ragged
    tails in M, N and K."""
    base = W.LINEAR_CASES[name]
    K = {16: 16 * 29, 64: 64 * 7, 256: 256 * 3}[base.g]
    case = base.replace(M=197, N=301, K=K)
    _check_linear(case, np.arange(case.M), np.arange(case.N))


@pytest.mark.parametrize("name", list(W.LINEAR_CASES))
def test_linear_full_size_sampled(name):
    case = W.LINEAR_CASES[name]
    _check_linear(case, sample_rows(case.M), sample_cols(case.N))


def test_linear_tiny_shapes():
    for (M, N, K, g, dt) in [(1, 1, 16, 16, "f32"), (3, 5, 48, 16, "bf16"), (9, 17, 64, 64, "f16"),
                             (2, 300, 256, 256, "bf16")]:
        case = W.LinearCase(f"tiny{M}_{N}_{K}", M=M, K=K, N=N, g=g, dtype=dt, rotation="haar",
                            seed=M + N)
        _check_linear(case, np.arange(M), np.arange(N))


def test_linear_is_deterministic():
    case = W.LINEAR_CASES["zimage_m32_k3840_n3840_g64_bf16"]
    inp = W.make_linear_inputs(case)
    o1, _ = _run_linear(inp, case)
    o2, _ = _run_linear(inp, case)
    assert torch.equal(o1, o2)


def test_binding_rejects_a_transposed_rotation():
    R = W.haar_orthogonal(64, torch.Generator().manual_seed(8)).to(torch.bfloat16).cuda()
    x = torch.zeros(4, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        ck.ck_rotate_quant(x, R.t(), 64)
    with pytest.raises(ValueError):
        ck.ck_rotate_quant(x, R.float(), 64)


def test_gemm_at_the_overflow_guard():
    """K just under the 64*K <= INT32_MAX guard with extreme codes: the true accumulator
    (-56 K and 49 K) fits in int32 even where intermediate sums are larger."""
    K = (2 ** 31 - 1) // 64 // 128 * 128
    M, N = 2, 16
    q = torch.full((M, K), -8, dtype=torch.int8)
    q[1] = 7
    wp = torch.full((N, K // 2), 0x77, dtype=torch.int8)     # every code 7
    out = ck.ck_w4a4_linear(q.cuda(), None, 0, wp.cuda(), torch.ones(N, device="cuda"),
                            a_scale=torch.ones(M, device="cuda"), out_dtype=torch.float32)
    torch.cuda.synchronize()
    acc = np.array([-56 * K, 49 * K], dtype=np.int64)
    assert np.abs(acc).max() <= 2 ** 31 - 1
    ref = acc.astype(np.float32)[:, None].repeat(N, 1)
    np.testing.assert_array_equal(out.cpu().numpy(), ref)


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("g", [16, 64])
def test_quantizer_exact_ties_with_inexact_reciprocal(dt, g):
    """Row absmax 21 gives s = 3 exactly, whose reciprocal is inexact: y / s is an exact
    half-integer for y = 3 (k + 1/2), and only the IEEE quotient rounds those half-to-even.
    Expected codes worked by hand: 1.5/3 = 0.5 -> 0, 4.5/3 = 1.5 -> 2, 7.5/3 = 2.5 -> 2,
    10.5/3 = 3.5 -> 4, 13.5/3 = 4.5 -> 4, 16.5/3 = 5.5 -> 6, 19.5/3 = 6.5 -> 6."""
    vals = [21, 1.5, 4.5, 7.5, 10.5, 13.5, 16.5, 19.5, -1.5, -4.5, -7.5, -10.5, -13.5, -16.5,
            -19.5, -21]
    want = [7, 0, 2, 2, 4, 4, 6, 6, 0, -2, -2, -4, -4, -6, -6, -7]
    x = torch.tensor(vals * (g // 16) * 2, dtype=torch.float64).reshape(1, -1).repeat(40, 1)
    x = x.to(DT[dt])
    R = torch.eye(g, dtype=torch.float64).to(DT[dt])
    codes, scales = ck.ck_rotate_quant(x.cuda(), R.cuda(), g)
    torch.cuda.synchronize()
    assert (scales.cpu() == 3.0).all()
    np.testing.assert_array_equal(codes.cpu().numpy(), np.array(want * (g // 16) * 2)[None].repeat(40, 0))
    oc, os_ = oracle.rotate_quant(x, R, g)
    np.testing.assert_array_equal(codes.cpu().numpy(), oc)


@pytest.mark.gpu
@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("g", [16, 64, 256])
def test_quantizer_codes_bit_exact_with_identity_rotation(dt, g):
    """With R = I the rotation is exact in every path, so the codes depend on the quantizer
    alone and must equal the oracle's IEEE-division codes bit for bit, ties included: half of
    the rows are random normals with outliers, half hold multiples of 1.5 next to an absmax
    of 21 (s = 3, an inexact reciprocal, so many quotients are exact half-integers)."""
    rng = np.random.default_rng(1000 + g)
    M, K = 300, 3840
    x = rng.standard_normal((M, K))
    x[:, rng.choice(K, K // 100, replace=False)] *= 20.0
    x[M // 2:] = 1.5 * rng.integers(-14, 15, size=(M - M // 2, K))
    x[M // 2:, 0] = 21.0
    xt = torch.from_numpy(x).to(DT[dt])
    R = torch.eye(g, dtype=torch.float64).to(DT[dt])
    codes, scales = ck.ck_rotate_quant(xt.cuda(), R.cuda(), g)
    torch.cuda.synchronize()
    oc, os_ = oracle.rotate_quant(xt, R, g)
    np.testing.assert_array_equal(scales.cpu().numpy(), os_)
    np.testing.assert_array_equal(codes.cpu().numpy(), oc)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("g", [16, 64, 256])
def test_quantizer_caller_scale_extremes_with_identity_rotation(dt, g):
    """A caller's scale far from the data, R = I so that y = x exactly.  With s = 1e-10 and
    values up to 3e35, y / s overflows fp32 and every nonzero code saturates by sign; with
    s = 2^-100 (a power of two below 2^-64) and x = k/2 * 2^-100, the quotients are exact
    half-integers and the codes are their ties rounded half to even."""
    rng = np.random.default_rng(77 + g)
    M, K = 24, g * 8
    x = rng.standard_normal((M, K))
    x[1, 5] = 1e30
    x[2, 7] = -3e35
    x[3] = 1e20
    x[4] = 0.0
    xt = torch.from_numpy(x).to(DT[dt])
    R = torch.eye(g, dtype=DT[dt])
    for sc, xs in ((1e-10, xt), (2.0 ** -100, (torch.from_numpy(rng.integers(-20, 21, size=(M, K)) / 2.0)
                                             * 2.0 ** -100).to(DT[dt]))):
        scale = torch.tensor([sc], dtype=torch.float32)
        codes, scales = ck.ck_rotate_quant(xs.cuda(), R.cuda(), g, scale_in=scale.cuda())
        torch.cuda.synchronize()
        oc, os_ = oracle.rotate_quant(xs, R, g, scale_in=float(scale))
        np.testing.assert_array_equal(scales.cpu().numpy(), os_)
        np.testing.assert_array_equal(codes.cpu().numpy(), oc)


# ------------------------------------------------------------------- fp32, g = 16 (fp64 sums)

def _colmajor(x: torch.Tensor, pad: int = 0) -> torch.Tensor:
    """x (M, K) as the transposed view of a (K, M + pad) row-major buffer."""
    M, K = x.shape
    buf = torch.zeros(K, M + pad, dtype=x.dtype)
    buf[:, :M] = x.t()
    return buf[:, :M].t()


@pytest.mark.parametrize("layout,M,K,pad", [("col", 16, 80, 0), ("col", 200, 464, 0),
                                            ("col", 1000, 3840, 12), ("col", 300, 16384, 4),
                                            ("col", 4096, 16384, 0), ("row", 1, 16, 0),
                                            ("row", 37, 80, 0), ("row", 333, 3840, 0),
                                            ("row", 129, 10240, 0), ("row", 20, 16384, 0),
                                            ("row", 50, 32768, 0)])
def test_rotate_quant_f32_g16_equals_the_oracle_bit_for_bit(layout, M, K, pad):
    """fp32 input with g = 16 forms each rotated value as the in-order fp64 sum of its sixteen
    exact products, rounded once to fp32, as the oracle does: codes and scales must equal the
    oracle's exactly.  Column-major views (unit M stride, 16-byte column pitch, some padded)
    and row-major rows from one group to 32768 channels, K split over a cluster where a block
    does not fit one CTA; a non-symmetric R, outlier channels and zero rows."""
    g = torch.Generator().manual_seed(M * 7 + K)
    x = torch.randn(M, K, generator=g)
    x[:, torch.randperm(K, generator=g)[: max(1, K // 100)]] *= 20.0
    x[M // 3] = 0.0
    if layout == "col":
        x = _colmajor(x, pad)
    elif pad:
        x = torch.zeros(M, K + pad)[:, :K].copy_(x)
    R = W.haar_orthogonal(16, torch.Generator().manual_seed(K)).float().contiguous()
    codes, scales = ck.ck_rotate_quant(to_device(x), R.cuda(), 16)
    torch.cuda.synchronize()
    rows = sample_rows(M, 96) if M * K > 4_000_000 else np.arange(M)
    oc, os_ = oracle.rotate_quant(x, R, 16, rows=rows)
    idx = torch.from_numpy(rows).cuda()
    np.testing.assert_array_equal(scales[idx].cpu().numpy(), os_)
    np.testing.assert_array_equal(codes[idx].cpu().numpy(), oc)


@pytest.mark.parametrize("layout,M,K", [("row", 9472, 512), ("row", 2000, 3840),
                                         ("col", 2368, 3840), ("col", 1100, 16384)])
def test_rotate_quant_f32_g16_many_blocks_per_cta(layout, M, K):
    """Several row blocks per CTA: the blocks cycle through the CTA's tile buffers, later
    blocks' copies landing while earlier ones are rotated and quantized, and the rotation of
    one block overlaps the cluster's exchange of the previous block's maxima.  Every row's
    codes and scale equal the oracle's bit for bit."""
    g = torch.Generator().manual_seed(M + K)
    x = torch.randn(M, K, generator=g)
    x[:, torch.randperm(K, generator=g)[: K // 64]] *= 30.0
    x[torch.randperm(M, generator=g)[:7]] *= 1e-3
    if layout == "col":
        x = _colmajor(x)
    R = W.haar_orthogonal(16, torch.Generator().manual_seed(M)).float().contiguous()
    codes, scales = ck.ck_rotate_quant(to_device(x), R.cuda(), 16)
    torch.cuda.synchronize()
    oc, os_ = oracle.rotate_quant(x, R, 16)
    np.testing.assert_array_equal(scales.cpu().numpy(), os_)
    np.testing.assert_array_equal(codes.cpu().numpy(), oc)


@pytest.mark.parametrize("layout", ["col", "row"])
def test_rotate_quant_f32_g16_caller_scale_and_non_finite(layout):
    M, K = 48, 256
    g = torch.Generator().manual_seed(5)
    x = torch.randn(M, K, generator=g)
    x[2, 5] = float("nan")
    x[7, 9] = float("inf")
    xv = _colmajor(x) if layout == "col" else x
    R = W.haar_orthogonal(16, torch.Generator().manual_seed(6)).float().contiguous()
    codes, scales = ck.ck_rotate_quant(to_device(xv), R.cuda(), 16)
    torch.cuda.synchronize()
    oc, os_ = oracle.rotate_quant(xv, R, 16)
    np.testing.assert_array_equal(scales.cpu().numpy(), os_)
    np.testing.assert_array_equal(codes.cpu().numpy(), oc)
    s = torch.tensor([0.05], dtype=torch.float32)
    codes, scales = ck.ck_rotate_quant(to_device(xv), R.cuda(), 16, scale_in=s.cuda())
    torch.cuda.synchronize()
    oc, os_ = oracle.rotate_quant(xv, R, 16, scale_in=0.05)
    np.testing.assert_array_equal(scales.cpu().numpy(), os_)
    np.testing.assert_array_equal(codes.cpu().numpy(), oc)


def test_linear_f32_g16_colmajor_outputs_equal_the_oracle():
    """The column-major fp32 workload at a size with 16-byte column pitch: stage 1 equals the
    oracle exactly, so every output equals the whole oracle path bit for bit."""
    case = W.LINEAR_CASES["krea_m4096_k16384_n6144_g16_f32_colmajor"].replace(M=400, N=300,
                                                                            K=16 * 61)
    inp = W.make_linear_inputs(case)
    assert inp["x"].stride(0) == 1 and inp["x"].stride(1) % 4 == 0
    out, ws = _run_linear(inp, case)
    ref, oc, os_ = oracle.linear(inp["x"], inp["R"], case.g, inp["w_packed"], inp["w_scale"],
                                 inp["bias"])
    gcodes, gscales = workspace_stage1(ws, case.M, case.K)
    np.testing.assert_array_equal(gcodes.cpu().numpy(), oc)
    np.testing.assert_array_equal(gscales.cpu().numpy(), os_)
    assert torch.equal(out.cpu().view(torch.int32), ref.view(torch.int32))


# ------------------------------------------------------------------- few rows (split K)

@pytest.mark.parametrize("M,N,K", [(1, 1, 128), (1, 3840, 3840), (7, 200, 448), (16, 6144, 16384),
                                   (32, 3840, 3840), (33, 129, 10240), (64, 3840, 3840),
                                   (64, 300, 48), (5, 1000, 1152)])
def test_few_rows_gemm_accumulators_bit_exact(M, N, K):
    """M <= 64 takes the split-K kernel (K split over a cluster, partial INT32 accumulators
    summed through distributed shared memory): unit scales, fp32 out give the accumulator
    exactly; then scales, bias and a 16-bit output against the oracle's epilogue."""
    g = torch.Generator().manual_seed(M * 31 + N + K)
    q = torch.randint(-8, 8, (M, K), generator=g, dtype=torch.int8)
    q[0, : min(K, 64)] = -8
    wp = torch.randint(-128, 128, (N, K // 2), generator=g, dtype=torch.int8)
    wp[0] = -120                                          # every code of channel 0 is -8
    out = ck.ck_w4a4_linear(q.cuda(), None, 0, wp.cuda(), torch.ones(N, device="cuda"),
                            a_scale=torch.ones(M, device="cuda"), out_dtype=torch.float32)
    torch.cuda.synchronize()
    cols = sample_cols(N, 160)
    acc = oracle.gemm_s32(q.numpy(), oracle.unpack_w4(wp[cols], K))
    np.testing.assert_array_equal(out.cpu().numpy()[:, cols], acc.astype(np.float32))
    a = torch.rand(M, generator=g) + 0.1
    ws = (torch.rand(N, generator=g) * 0.015 + 0.005).to(torch.bfloat16)
    b = torch.randn(N, generator=g).to(torch.bfloat16)
    out2 = ck.ck_w4a4_linear(q.cuda(), None, 0, wp.cuda(), ws.cuda(), b.cuda(), a_scale=a.cuda(),
                             out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    ref = oracle.epilogue(acc, a.numpy(), ws[cols], b[cols], torch.bfloat16)
    assert torch.equal(out2.cpu()[:, torch.from_numpy(cols)], ref)


@pytest.mark.parametrize("M", [1, 8, 16, 32])
def test_few_rows_linear_every_output(M):
    """The decode-sized linear (M = 1 to 32 rows of the Z-Image recipe, K = N = 3840) through
    both stages, every output compared with the oracle."""
    case = W.LINEAR_CASES["zimage_m32_k3840_n3840_g64_bf16"].replace(M=M, seed=100 + M)
    _check_linear(case, np.arange(case.M), sample_cols(case.N, 512))


# ------------------------------------------------------------------- grouped linear

@pytest.mark.parametrize("M,groups,dt,bias", [(197, [128, 96, 200], "bf16", True),
                                             (8192, [3840, 1024, 1024], "bf16", True),
                                             (32, [3840, 3840, 3840], "bf16", True),
                                             (300, [64, 1, 130, 7, 256], "f16", False),
                                             (5, [200, 56], "f32", True)])
def test_grouped_linear_equals_each_linear_and_the_oracle(M, groups, dt, bias):
    """Q/K/V-style projections of one input: one stage 1, one GEMM over the stacked weights.
    Each group's output must equal ck_w4a4_linear with that group's weights alone, bit for
    bit, and the oracle applied to that group within the parity rule."""
    K, g = 448 if M < 8192 else 3840, 64
    base = W.LINEAR_CASES[W.HEADLINE]
    case = base.replace(M=M, K=K, N=sum(groups), dtype=dt, has_bias=bias, seed=M + len(groups))
    inp = W.make_linear_inputs(case)
    x, R = inp["x"].cuda(), inp["R"].cuda()
    parts, o = [], 0
    for n in groups:
        b = None if inp["bias"] is None else inp["bias"][o:o + n].cuda()
        parts.append((inp["w_packed"][o:o + n].cuda(), inp["w_scale"][o:o + n].cuda(), b))
        o += n
    wp, wsc, bs, gn = ck.fuse_linear_weights(parts)
    outs = ck.ck_w4a4_grouped_linear(x, R, g, wp, wsc, bs, gn)
    singles = [ck.ck_w4a4_linear(x, R, g, p[0], p[1], p[2]) for p in parts]
    torch.cuda.synchronize()
    itype = torch.int32 if dt == "f32" else torch.int16
    rows = sample_rows(M, 64)
    o = 0
    for i, n in enumerate(groups):
        assert torch.equal(outs[i].view(itype), singles[i].view(itype)), f"group {i}"
        cols = sample_cols(n, 96)
        bi = None if inp["bias"] is None else inp["bias"][o:o + n]
        ref, oc, os_ = oracle.linear(inp["x"], inp["R"], g, inp["w_packed"][o:o + n],
                                     inp["w_scale"][o:o + n], bi, rows=rows, cols=cols)
        got = outs[i].cpu()[torch.from_numpy(rows)][:, torch.from_numpy(cols)]
        # the GPU's own codes for these rows: from a stage-1 call on the same input
        gc, gs = ck.ck_rotate_quant(x, R, g)
        gc = gc[torch.from_numpy(rows).cuda()].cpu().numpy()
        gs = gs[torch.from_numpy(rows).cuda()].cpu().numpy()
        compare_stage1(gc, gs, oc, os_, DT[dt], f"group {i}", g, x=inp["x"], R=inp["R"], rows=rows)
        extra = output_widening(gc, oc, gs, os_, inp["w_packed"][o:o + n], K, cols,
                                inp["w_scale"][o:o + n])
        assert_close(got, ref, DT[dt], f"group {i}", extra)
        o += n


def test_grouped_linear_with_codes_in_and_pitched_outputs():
    """The GEMM-only path (int8 codes with row scales) into outputs that are views of wider
    buffers: guard columns stay untouched."""
    M, K, groups = 150, 384, [100, 28, 300]
    g = torch.Generator().manual_seed(4)
    q = torch.randint(-8, 8, (M, K), generator=g, dtype=torch.int8).cuda()
    a = (torch.rand(M, generator=g) + 0.1).cuda()
    N = sum(groups)
    wp = torch.randint(-128, 128, (N, K // 2), generator=g, dtype=torch.int8).cuda()
    wsc = (torch.rand(N, generator=g) + 0.5).cuda()
    bufs = [torch.full((M, n + 5), 7.0, device="cuda") for n in groups]
    outs = [b[:, 2:2 + n] for b, n in zip(bufs, groups)]
    ck.ck_w4a4_grouped_linear(q, None, 0, wp, wsc, None, groups, outs=outs, a_scale=a)
    full = ck.ck_w4a4_linear(q, None, 0, wp, wsc, a_scale=a, out_dtype=torch.float32)
    torch.cuda.synchronize()
    o = 0
    for b, out, n in zip(bufs, outs, groups):
        assert torch.equal(out, full[:, o:o + n])
        assert (b[:, :2] == 7.0).all() and (b[:, 2 + n:] == 7.0).all()
        o += n


# ------------------------------------------------------------------- W8A8 variant

W8_RATE = 5e-3   # INT8 codes of 16-bit inputs: ~ the rate at which the dtype rounding of y flips


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("g", [16, 64, 256])
def test_int8_stage1_identity_rotation_bit_exact(dt, g):
    """R = I makes y exact in every kernel: the INT8 codes and scales equal the oracle's."""
    rng = np.random.default_rng(500 + g)
    M, K = 200, 3840
    x = rng.standard_normal((M, K)) * 3
    x[:, rng.choice(K, K // 100, replace=False)] *= 20.0
    x[7] = 0
    xt = torch.from_numpy(x).to(DT[dt])
    R = torch.eye(g, dtype=DT[dt])
    codes, scales = ck.ck_rotate_quant_int8(xt.cuda(), R.cuda(), g)
    torch.cuda.synchronize()
    oc, os_ = oracle.rotate_quant_int8(xt, R, g)
    np.testing.assert_array_equal(scales.cpu().numpy(), os_)
    np.testing.assert_array_equal(codes.cpu().numpy(), oc)


@pytest.mark.parametrize("layout", ["row", "col"])
def test_int8_stage1_f32_g16_bit_exact(layout):
    g = torch.Generator().manual_seed(61)
    x = torch.randn(256, 1024, generator=g) * 4
    xv = _colmajor(x) if layout == "col" else x
    R = W.haar_orthogonal(16, torch.Generator().manual_seed(62)).float().contiguous()
    codes, scales = ck.ck_rotate_quant_int8(to_device(xv), R.cuda(), 16)
    torch.cuda.synchronize()
    oc, os_ = oracle.rotate_quant_int8(xv, R, 16)
    np.testing.assert_array_equal(scales.cpu().numpy(), os_)
    np.testing.assert_array_equal(codes.cpu().numpy(), oc)


@pytest.mark.parametrize("dt,g,M,K", [("bf16", 64, 8192, 3840), ("f16", 256, 8192, 10240),
                                      ("bf16", 16, 300, 3840), ("f16", 64, 50, 16384)])
def test_int8_stage1_general_rotation(dt, g, M, K):
    case = W.RotateCase(f"int8_{dt}_{g}", M=M, K=K, g=g, dtype=dt, seed=g + K)
    inp = W.make_rotate_inputs(case)
    R = W.haar_orthogonal(g, torch.Generator().manual_seed(K)).to(DT[dt]).contiguous()
    codes, scales = ck.ck_rotate_quant_int8(to_device(inp["x"]), R.cuda(), g)
    torch.cuda.synchronize()
    rows = sample_rows(M, 48)
    oc, os_ = oracle.rotate_quant_int8(inp["x"], R, g, rows=rows)
    idx = torch.from_numpy(rows).cuda()
    compare_stage1(codes[idx].cpu().numpy(), scales[idx].cpu().numpy(), oc, os_, DT[dt], case.name,
                   g, x=inp["x"], R=R, rows=rows, qmax=127, max_rate=W8_RATE)


@pytest.mark.parametrize("M,N,K,out_dt", [(1, 1, 128, torch.float32), (200, 300, 448, torch.float32),
                                          (4000, 2000, 384, torch.bfloat16),
                                          (8192, 3840, 3840, torch.bfloat16),
                                          (77, 513, 4096, torch.float16)])
def test_w8a8_gemm_accumulators_bit_exact(M, N, K, out_dt):
    g = torch.Generator().manual_seed(M + N + K + 8)
    q = torch.randint(-128, 128, (M, K), generator=g, dtype=torch.int8)
    w = torch.randint(-128, 128, (N, K), generator=g, dtype=torch.int8)
    q[0] = -128
    w[0] = -128                                  # acc[0, 0] = 16384 K, the bound
    out = ck.ck_w8a8_linear(q.cuda(), None, 0, w.cuda(), torch.ones(N, device="cuda"),
                            a_scale=torch.ones(M, device="cuda"), out_dtype=torch.float32)
    torch.cuda.synchronize()
    rows, cols = sample_rows(M, 64), sample_cols(N, 96)
    acc = oracle.gemm_s32(q.numpy()[rows], w.numpy()[cols])
    got = out.cpu().numpy()[rows][:, cols]
    # exact in fp32 while |acc| < 2^24; beyond, the fp32 cast of the exact INT32 value
    np.testing.assert_array_equal(got, acc.astype(np.float32))
    assert got[0, 0] == 16384 * K
    a = torch.rand(M, generator=g) * 0.01 + 0.001
    ws = (torch.rand(N, generator=g) * 0.015 + 0.005).to(out_dt)
    b = torch.randn(N, generator=g).to(out_dt)
    out2 = ck.ck_w8a8_linear(q.cuda(), None, 0, w.cuda(), ws.cuda(), b.cuda(), a_scale=a.cuda(),
                             out_dtype=out_dt)
    torch.cuda.synchronize()
    ref = oracle.epilogue(acc, a.numpy()[rows], ws[cols], b[cols], out_dt)
    assert torch.equal(out2.cpu()[torch.from_numpy(rows)][:, torch.from_numpy(cols)], ref)


@pytest.mark.parametrize("dt,M,N,K,g", [("bf16", 197, 301, 448, 64), ("f16", 300, 130, 768, 256),
                                        ("f32", 129, 260, 464, 16), ("bf16", 8192, 3840, 3840, 64)])
def test_w8a8_linear_against_the_oracle(dt, M, N, K, g):
    """The whole W8A8 path: bit-exact against the oracle's GEMM + epilogue on the GPU's own INT8
    codes, and within the parity rule against the whole oracle path (tie flips widened)."""
    gen = torch.Generator().manual_seed(M + N)
    case = W.LinearCase("w8", M=M, K=K, N=N, g=g, dtype=dt, rotation="haar", seed=M * 3 + g)
    inp = W.make_linear_inputs(case)
    w8 = torch.randint(-128, 128, (N, K), generator=gen, dtype=torch.int8)
    x, R = to_device(inp["x"]), inp["R"].cuda()
    ws = torch.empty(int(ck.lib().ck_w8a8_linear_workspace_bytes(M, N, K, K)), dtype=torch.uint8,
                     device="cuda")
    out = ck.ck_w8a8_linear(x, R, g, w8.cuda(), inp["w_scale"].cuda(), inp["bias"].cuda(),
                            workspace=ws)
    torch.cuda.synchronize()
    rows, cols = sample_rows(M, 48), sample_cols(N, 64)
    gcodes, gscales = workspace_stage1(ws, M, K)
    gc = gcodes[torch.from_numpy(rows).cuda()].cpu().numpy()
    gs = gscales[torch.from_numpy(rows).cuda()].cpu().numpy()
    ref, oc, os_ = oracle.linear_w8a8(inp["x"], inp["R"], g, w8, inp["w_scale"], inp["bias"],
                                      rows=rows, cols=cols)
    compare_stage1(gc, gs, oc, os_, DT[dt], "w8a8", g, x=inp["x"], R=inp["R"], rows=rows,
                   qmax=127, max_rate=W8_RATE)
    got = out.cpu()[torch.from_numpy(rows)][:, torch.from_numpy(cols)]
    acc = oracle.gemm_s32(gc, w8.numpy()[cols])
    exact = oracle.epilogue(acc, gs, inp["w_scale"][cols], inp["bias"][cols], DT[dt])
    itype = torch.int32 if dt == "f32" else torch.int16
    assert torch.equal(got.view(itype), exact.view(itype))
    extra = widening_for_weights(gc, oc, gs, os_, w8.numpy()[cols], inp["w_scale"][cols])
    assert_close(got, ref, DT[dt], "w8a8", extra)


# ------------------------------------------------------------------- packed quantizer

def _unpack_codes(packed: np.ndarray) -> np.ndarray:
    lo = (packed & 0xF).astype(np.int64)
    hi = (packed >> 4).astype(np.int64)
    out = np.empty((packed.shape[0], 2 * packed.shape[1]), dtype=np.int64)
    out[:, 0::2] = np.where(lo >= 8, lo - 16, lo)
    out[:, 1::2] = np.where(hi >= 8, hi - 16, hi)
    return out


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("stochastic", [False, True])
def test_packed_quantizer_identity_rotation_bit_exact(dt, stochastic):
    """R = I: y is exact on both sides, so nearest and stochastic codes (the same Philox draws,
    the same fp32 operations) and the packed bytes equal the oracle's."""
    rng = np.random.default_rng(70)
    M, K, g = 96, 1024, 64
    x = rng.standard_normal((M, K)) * 2
    x[:, rng.choice(K, 10, replace=False)] *= 20
    x[3] = 0
    xt = torch.from_numpy(x).to(DT[dt])
    R = torch.eye(g, dtype=DT[dt])
    packed, scales = ck.ck_rotate_quant_packed(xt.cuda(), R.cuda(), g, stochastic=stochastic,
                                               seed=0x1234ABCD5678, offset=99)
    torch.cuda.synchronize()
    y = oracle.rotate(xt, R, g)
    op, os_ = oracle.quantize_packed(y, np.arange(M), K, stochastic=stochastic,
                                     seed=0x1234ABCD5678, offset=99)
    np.testing.assert_array_equal(scales.cpu().numpy(), os_)
    np.testing.assert_array_equal(packed.cpu().numpy(), op)


def test_packed_quantizer_nearest_matches_stage1_codes():
    """Nearest rounding gives ck_rotate_quant's codes, packed (identity rotation: y exact)."""
    x = torch.randn(50, 512, generator=torch.Generator().manual_seed(71)).to(torch.bfloat16).cuda()
    R = torch.eye(16, dtype=torch.bfloat16).cuda()
    packed, s1 = ck.ck_rotate_quant_packed(x, R, 16)
    codes, s2 = ck.ck_rotate_quant(x, R, 16)
    torch.cuda.synchronize()
    assert torch.equal(s1, s2)
    np.testing.assert_array_equal(_unpack_codes(packed.cpu().numpy()), codes.cpu().numpy())


@pytest.mark.parametrize("dt,g,M,K,pitch", [("bf16", 64, 1000, 3840, 0), ("f16", 16, 333, 1024, 0),
                                             ("bf16", 16, 8192, 3840, 0), ("f16", 64, 129, 8192, 3),
                                             ("bf16", 256, 700, 3840, 0), ("f16", 256, 65, 10240, 5)])
def test_packed_quantizer_nearest_equals_stage1_codes_on_tensor_cores(dt, g, M, K, pitch):
    """16-bit rows of g = 16 or 64 and at most 128 64-channel groups, or g = 256 and at most 128
    groups, take the tensor-core stage-1 kernel with a packed epilogue: with round half to even its codes are stage 1's
    codes for any R, bit for bit, and the scales are equal.  A Haar R, several rows per tile
    and split tiles, an output pitch that is not a multiple of 8 bytes (byte stores)."""
    x = torch.randn(M, K, generator=torch.Generator().manual_seed(M + K)).to(DT[dt]).cuda()
    R = W.haar_orthogonal(g, torch.Generator().manual_seed(g)).to(DT[dt]).contiguous().cuda()
    buf = torch.zeros(M, K // 2 + pitch, dtype=torch.uint8, device="cuda")
    packed, s1 = ck.ck_rotate_quant_packed(x, R, g, packed=buf[:, : K // 2])
    codes, s2 = ck.ck_rotate_quant(x, R, g)
    torch.cuda.synchronize()
    assert torch.equal(s1, s2)
    np.testing.assert_array_equal(_unpack_codes(packed.cpu().numpy()), codes.cpu().numpy())
    if pitch:
        assert int(buf[:, K // 2:].abs().sum()) == 0   # nothing written past each row


@pytest.mark.parametrize("dt,g", [("bf16", 64), ("f16", 256), ("f32", 16)])
def test_packed_quantizer_stochastic_general_rotation(dt, g):
    """A general R: y may differ from the oracle's by its accumulation's rounding, so a code may
    differ only where t + u lies within that difference of an integer (the stochastic analog
    of a tie), by one step; scales follow the stage-1 rule."""
    M, K = 64, 2048
    x = torch.randn(M, K, generator=torch.Generator().manual_seed(72)).to(DT[dt])
    R = W.haar_orthogonal(g, torch.Generator().manual_seed(73)).to(DT[dt]).contiguous()
    seed, off = 2024, 5
    packed, scales = ck.ck_rotate_quant_packed(x.cuda(), R.cuda(), g, stochastic=True, seed=seed,
                                               offset=off)
    torch.cuda.synchronize()
    y = oracle.rotate(x, R, g)
    op, os_ = oracle.quantize_packed(y, np.arange(M), K, stochastic=True, seed=seed, offset=off)
    gs = scales.cpu().numpy()
    rel = np.abs(gs.astype(np.float64) - os_) / os_
    from parity_util import scale_rtol, tie_distance_bound
    assert (rel <= scale_rtol(DT[dt], g)).all()
    gq, oq = _unpack_codes(packed.cpu().numpy()), _unpack_codes(op)
    diff = gq - oq
    assert np.abs(diff).max() <= 1 and (diff != 0).mean() <= 1e-3
    for r, k in zip(*np.nonzero(diff)):
        e = r * K + k
        word = oracle.philox4x32_10([e & 0xFFFFFFFF, e >> 32, off, 0], [seed, 0])[0]
        u = float(np.float32(word >> 8) * np.float32(2.0 ** -24))
        t = y[r, k] / float(os_[r])
        xr = oracle.decode(x[r].contiguous())
        j, c = divmod(int(k), g)
        terms = np.abs(xr[j * g:(j + 1) * g]) @ np.abs(oracle.decode(R.contiguous())[:, c])
        bound = tie_distance_bound(np.array([y[r, k]]), np.array([float(os_[r])]), np.array([terms]),
                                   DT[dt], g, dynamic=True)[0] + 2.0 ** -23 * (abs(t) + 1)
        dist = abs((t + u) - round(t + u))
        assert dist <= bound, (r, k, t, u, dist, bound)


def test_packed_quantizer_seed_and_offset_change_the_draws():
    x = torch.randn(32, 1024, generator=torch.Generator().manual_seed(74)).cuda()
    R = torch.eye(16).cuda()
    a, _ = ck.ck_rotate_quant_packed(x, R, 16, stochastic=True, seed=1)
    b, _ = ck.ck_rotate_quant_packed(x, R, 16, stochastic=True, seed=1)
    c, _ = ck.ck_rotate_quant_packed(x, R, 16, stochastic=True, seed=2)
    d, _ = ck.ck_rotate_quant_packed(x, R, 16, stochastic=True, seed=1, offset=1)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and not torch.equal(a, c) and not torch.equal(a, d)


@pytest.mark.parametrize("dt", ["f16", "bf16"])
@pytest.mark.parametrize("M,K", [(300, 64), (1000, 448), (8192, 3840), (77, 8192)])
def test_rotate_quant_g16_on_tensor_cores(dt, M, K):
    """g = 16 rows of whole 64-channel groups run as a g = 64 rotation by diag(R, R, R, R) on
    the tensor-core kernel.  A non-symmetric R, so a transposed or misplaced block shows; every
    output of the sampled rows is compared."""
    case = W.RotateCase(f"g16tc_{dt}_{K}", M=M, K=K, g=16, dtype=dt, seed=K + M)
    x = W.make_rotate_inputs(case)["x"]
    R = W.haar_orthogonal(16, torch.Generator().manual_seed(K)).to(DT[dt]).contiguous()
    codes, scales = ck.ck_rotate_quant(to_device(x), R.cuda(), 16)
    torch.cuda.synchronize()
    rows = sample_rows(M, 64)
    oc, os_ = oracle.rotate_quant(x, R, 16, rows=rows)
    idx = torch.from_numpy(rows).cuda()
    compare_stage1(codes[idx].cpu().numpy(), scales[idx].cpu().numpy(), oc, os_, DT[dt], case.name,
                   16, x=x, R=R, rows=rows)
