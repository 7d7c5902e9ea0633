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
                                        (256, 1, 1000), (256, 43, 333), (256, 128, 150),
                                        (256, 129, 3)])
def test_rotate_quant_tile_shapes(dt, g, groups, M):
    """Rows of 1 to 129 groups: a tile packs floor(128 / groups) rows, so these cover a tile of
    128 one-group rows, one row of 127 or 128 groups, a ragged last tile, more tiles than SMs
    (150 rows of 128 groups), and the first row length past 128 groups, which another kernel
    takes.  R is a non-symmetric orthogonal matrix, so R and R^T give different results.
    Every output is compared."""
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
