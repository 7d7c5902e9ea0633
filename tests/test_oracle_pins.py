"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test checks one oracle step against a hand-worked fixture (tests/golden/), an
independent library routine (numpy / torch dtype casts, numpy matmul, a fast
Walsh-Hadamard transform), a closed form, or an invariant the pages fix:
  - PR #198 "Consolidate INT8, RotateQuant, RoPE and ConvRot W4A4 backends",
    "W4A4 correctness and performance scope": rotation in the input dtype, the
    signed-INT4 quantizer, INT8 unpack of W4 codes, INT32 accumulation with an
    overflow guard, cast -> activation scale -> weight scale -> bias;
  - PR #201 "Avoid activation pack/unpack in ConvRot W4A4", "Correctness and tests":
    packed and unpacked codes are equal, zeros / tiny / max-finite / NaN / Inf cases;
  - PR #155 "Add fused RotateQuant backend": orthogonal and asymmetric rotations,
    all-zero rows, caller-provided zero scales.
"""
from __future__ import annotations

import math
import os

import numpy as np
import pytest
import torch

import oracle
from rotated_w4a4_quantized_group_b200 import workloads as W

FLT_MIN = float(np.finfo(np.float32).tiny)
TORCH_DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


# ----------------------------------------------------------------------------- helpers

def _parse_cases(path):
    cases, cur = [], None
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, _, rest = line.partition(" ")
        if key == "case":
            cur = {"name": rest}
            cases.append(cur)
        else:
            cur[key] = rest
    return cases


def _shift1(g):
    r = np.zeros((g, g))
    for i in range(g):
        r[i, (i + 1) % g] = 1.0
    return r


def _bf16_via_f32(v64: np.ndarray):
    """Independent bf16 rounding through numpy fp32 then torch's fp32->bf16 cast, plus a mask
    of the elements where that two-step rounding could differ from one rounding (the fp32
    value sits exactly on a bf16 midpoint while the double does not)."""
    f32 = v64.astype(np.float32)
    bits = f32.view(np.uint32)
    unsafe = ((bits & 0xFFFF) == 0x8000) & (f32.astype(np.float64) != v64)
    b = torch.from_numpy(f32).to(torch.bfloat16).to(torch.float64).numpy()
    return b, unsafe


def _independent_round(v64: np.ndarray, dt: str):
    if dt == "f32":
        return v64.astype(np.float32).astype(np.float64), np.zeros(v64.shape, bool)
    if dt == "f16":
        return v64.astype(np.float16).astype(np.float64), np.zeros(v64.shape, bool)
    return _bf16_via_f32(v64)


def _fwht(a: np.ndarray) -> np.ndarray:
    """Unnormalised fast Walsh-Hadamard transform along the last axis (natural order)."""
    a = a.copy()
    n = a.shape[-1]
    h = 1
    while h < n:
        a = a.reshape(*a.shape[:-1], n // (2 * h), 2, h)
        u, v = a[..., 0, :].copy(), a[..., 1, :].copy()
        a[..., 0, :], a[..., 1, :] = u + v, u - v
        a = a.reshape(*a.shape[:-3], n)
        h *= 2
    return a


# ----------------------------------------------------------------------------- dtype rounding

def test_round_f32_matches_ieee_cast():
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-45, 39, 20000),
                        [0.0, -0.0, 3.4028235677973366e38, 3.402823669209385e38, 1e-46, 7e-46,
                         1.401298464324817e-45, np.inf, -np.inf]])
    with np.errstate(over="ignore"):
        ref = v.astype(np.float32).astype(np.float64)
    np.testing.assert_array_equal(oracle.round_to(v, torch.float32), ref)


def test_round_f16_matches_numpy_half():
    rng = np.random.default_rng(2)
    v = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-9, 6, 20000),
                        [65504.0, 65519.99, 65520.0, -65520.0, 2.0 ** -24, 2.0 ** -25,
                         3 * 2.0 ** -26, 2.0 ** -14 - 2.0 ** -25, 0.0, -0.0]])
    with np.errstate(over="ignore"):
        ref = v.astype(np.float16).astype(np.float64)
    np.testing.assert_array_equal(oracle.round_to(v, torch.float16), ref)


def test_round_bf16_matches_torch_cast():
    rng = np.random.default_rng(3)
    # values exactly representable in fp32, so the fp32->bf16 cast is one rounding
    v = (rng.standard_normal(20000) * 10.0 ** rng.integers(-40, 38, 20000)).astype(np.float32)
    v = np.concatenate([v, np.float32([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8),
                                       3.3895313892515355e38, 2 ** -133, 2 ** -134])])
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.round_to(v.astype(np.float64), torch.bfloat16), ref)


def test_decode_all_16bit_patterns():
    bits = np.arange(65536, dtype=np.uint16)
    t16 = torch.from_numpy(bits.view(np.int16).copy())
    f16 = oracle.decode(t16.view(torch.float16))
    ref16 = bits.view(np.float16).astype(np.float64)
    np.testing.assert_array_equal(np.isnan(f16), np.isnan(ref16))
    ok = ~np.isnan(ref16)
    np.testing.assert_array_equal(f16[ok], ref16[ok])
    bf = oracle.decode(t16.view(torch.bfloat16))
    refb = t16.view(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(np.isnan(bf), np.isnan(refb))
    ok = ~np.isnan(refb)
    np.testing.assert_array_equal(bf[ok], refb[ok])


# ----------------------------------------------------------------------------- rotation

@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
def test_rotate_identity_is_exact(dt):
    x = torch.randn(5, 64, generator=torch.Generator().manual_seed(4)).to(TORCH_DT[dt])
    R = torch.eye(16, dtype=torch.float64).to(TORCH_DT[dt])
    y = oracle.rotate(x, R, 16)
    np.testing.assert_array_equal(y, x.to(torch.float64).numpy())


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("g", [16, 64, 256])
def test_rotate_hadamard_matches_fwht(dt, g):
    gen = torch.Generator().manual_seed(5 + g)
    x = (torch.randn(6, 2 * g, generator=gen) * 3).to(TORCH_DT[dt])
    R = W.hadamard(g).to(TORCH_DT[dt])
    y = oracle.rotate(x, R, g)
    xd = x.to(torch.float64).numpy().reshape(6, 2, g)
    exact = (_fwht(xd) / math.sqrt(g)).reshape(6, 2 * g)
    ref, unsafe = _independent_round(exact, dt)
    assert unsafe.mean() < 0.01
    np.testing.assert_array_equal(y[~unsafe], ref[~unsafe])


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("g", [16, 64, 256])
def test_rotate_haar_matches_float64_matmul(dt, g):
    gen = torch.Generator().manual_seed(6 + g)
    R = W.haar_orthogonal(g, gen).to(TORCH_DT[dt])
    x = (torch.randn(7, 3 * g, generator=gen) * 2).to(TORCH_DT[dt])
    # a column-major view exercises the stride path
    xv = x.t().contiguous().t()
    y = oracle.rotate(xv, R, g)
    xd = x.to(torch.float64).numpy().reshape(7, 3, g)
    exact = (xd @ R.to(torch.float64).numpy()).reshape(7, 3 * g)
    ref, unsafe = _independent_round(exact, dt)
    mism = (y != ref) & ~unsafe
    assert mism.mean() <= 1e-6, mism.sum()


def test_rotation_convention_is_x_times_R():
    """A non-symmetric orthogonal R (cyclic shift) tells x @ R from R @ x."""
    x = torch.arange(1, 17, dtype=torch.float32).reshape(1, 16)
    R = torch.from_numpy(_shift1(16)).to(torch.float32)
    y = oracle.rotate(x, R, 16)
    np.testing.assert_array_equal(y[0], np.roll(np.arange(1, 17), 1))


@pytest.mark.parametrize("g", [16, 64, 256])
def test_generated_rotations_are_orthogonal(g):
    gen = torch.Generator().manual_seed(7)
    for R64 in (W.hadamard(g), W.haar_orthogonal(g, gen)):
        np.testing.assert_allclose(R64.T @ R64, np.eye(g), atol=1e-12)
        for dt, eps in (("f32", 2 ** -24), ("f16", 2 ** -11), ("bf16", 2 ** -8)):
            Rd = R64.to(TORCH_DT[dt]).to(torch.float64)
            err = (Rd.T @ Rd - torch.eye(g, dtype=torch.float64)).abs().max().item()
            assert err <= 4 * math.sqrt(g) * eps
    Rh = W.haar_orthogonal(g, gen)
    assert (Rh - Rh.T).abs().max().item() > 0.1      # asymmetric, as the configs ask
    np.testing.assert_array_equal(W.hadamard(g).to(torch.bfloat16).to(torch.float64),
                                  W.hadamard(g))     # +-1/sqrt(g) is exact in every dtype


def test_rotation_preserves_group_norm():
    gen = torch.Generator().manual_seed(8)
    R = W.haar_orthogonal(64, gen).to(torch.float32)
    x = torch.randn(4, 256, generator=gen)
    y = oracle.rotate(x, R, 64).reshape(4, 4, 64)
    xn = np.linalg.norm(x.numpy().reshape(4, 4, 64).astype(np.float64), axis=-1)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), xn, rtol=1e-5)


# ----------------------------------------------------------------------------- quantizer

def test_golden_quant_rows(golden_dir):
    for c in _parse_cases(os.path.join(golden_dir, "quant_rows_g16_f32.txt")):
        x = torch.tensor([float(v) for v in c["x"].split()], dtype=torch.float32).reshape(1, 16)
        R = torch.eye(16) if c["rotation"] == "identity" else torch.from_numpy(_shift1(16)).float()
        s_in = None if c["scale_in"] == "none" else float(c["scale_in"])
        codes, scales = oracle.rotate_quant(x, R, 16, scale_in=s_in)
        assert scales[0] == np.float32(float(c["scale"])), c["name"]
        assert codes[0].tolist() == [int(v) for v in c["codes"].split()], c["name"]


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
def test_zero_rows_give_zero_codes_and_flt_min(dt):
    x = torch.randn(6, 128, generator=torch.Generator().manual_seed(9)).to(TORCH_DT[dt])
    x[2] = 0
    x[5] = -0.0
    R = W.hadamard(64).to(TORCH_DT[dt])
    codes, scales = oracle.rotate_quant(x, R, 64)
    for r in (2, 5):
        assert not codes[r].any()
        assert scales[r] == np.float32(FLT_MIN)
    assert (scales > 0).all()


def test_caller_zero_scale_follows_eager_semantics():
    """A zero tensor-wise scale becomes the finite minimum: zeros stay 0, the rest saturate."""
    x = torch.randn(3, 64, generator=torch.Generator().manual_seed(10)).to(torch.bfloat16)
    x[1, ::3] = 0
    R = torch.eye(64, dtype=torch.bfloat16)
    codes, scales = oracle.rotate_quant(x, R, 64, scale_in=0.0)
    assert (scales == np.float32(FLT_MIN)).all()
    xv = x.float().numpy()
    np.testing.assert_array_equal(codes[xv == 0], 0)
    np.testing.assert_array_equal(codes[xv > 0], 7)
    np.testing.assert_array_equal(codes[xv < 0], -8)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_caller_scale_far_from_the_data(dt):
    """Closed forms for a caller's scale, with R = I so that y = x.  Below the data (s = 1e-10,
    values up to 3e35, where y / s overflows fp32) every code is the sign's saturated value.  A
    power of two (s = 2^-100) divides exactly, so the codes of x = k/2 * 2^-100 are the
    half-integers k/2 rounded half to even and clamped, computed here with Python's round()."""
    rng = np.random.default_rng(21)
    x = rng.standard_normal((6, 64))
    x[1, 5] = 1e30
    x[2, 7] = -3e35
    x[4] = 0.0
    R = torch.eye(16, dtype=TORCH_DT[dt])
    xt = torch.from_numpy(x).to(TORCH_DT[dt])
    codes, scales = oracle.rotate_quant(xt, R, 16, scale_in=1e-10)
    assert (scales == np.float32(1e-10)).all()
    xv = xt.double().numpy()
    np.testing.assert_array_equal(codes, np.where(xv > 0, 7, np.where(xv < 0, -8, 0)))

    k = rng.integers(-20, 21, size=(6, 64))
    xt = torch.from_numpy(k / 2.0 * 2.0 ** -100).to(TORCH_DT[dt])
    codes, _ = oracle.rotate_quant(xt, R, 16, scale_in=2.0 ** -100)
    want = np.vectorize(lambda v: max(-8, min(7, round(v / 2))))(k)   # round(): half to even
    np.testing.assert_array_equal(codes, want)


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
def test_dynamic_codes_reach_seven_and_never_minus_eight(dt):
    case = W.RotateCase("t", M=40, K=512, g=64, dtype=dt, seed=11)
    inp = W.make_rotate_inputs(case)
    codes, scales = oracle.rotate_quant(inp["x"], inp["R"], case.g)
    assert (np.abs(codes).max(axis=1) == 7).all()
    assert (codes >= -7).all()


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
def test_reconstruction_error_within_half_step(dt):
    case = W.RotateCase("t", M=16, K=256, g=16, dtype=dt, seed=12)
    inp = W.make_rotate_inputs(case)
    y = oracle.rotate(inp["x"], inp["R"], case.g)
    codes, scales = oracle.quantize(y)
    s = scales.astype(np.float64)[:, None]
    err = np.abs(y - codes * s)
    assert (err <= s / 2 * (1 + 2 ** -22)).all()
    # the scale is the fp32 quotient of the row absmax by 7
    amax = np.abs(y).max(axis=1)
    np.testing.assert_array_equal(scales, (amax.astype(np.float32) / np.float32(7)))


def test_non_finite_values_follow_the_stated_convention():
    x = torch.zeros(3, 32)
    x[0, 3] = float("nan")
    x[1, 4] = float("inf")
    x[1, 20] = 1.0
    x[2] = torch.arange(32) - 8.0
    H = W.hadamard(16).to(torch.float32)
    codes, scales = oracle.rotate_quant(x, H, 16)
    assert math.isnan(scales[0]) and not codes[0].any()          # NaN row: scale NaN, codes 0
    # the inf spreads to +-inf over its group; inf/inf is NaN -> 0 and finite/inf -> 0
    assert math.isinf(scales[1]) and not codes[1].any()
    codes_c, _ = oracle.rotate_quant(x[1:2], H, 16, scale_in=1.0)
    y = np.sign(H[4].numpy())                                     # row 4 of H carries the inf
    np.testing.assert_array_equal(codes_c[0, :16], np.where(y > 0, 7, -8))   # +-inf clamps
    # an identity rotation turns inf * 0 into NaN over the whole group (IEEE)
    codes_i, scales_i = oracle.rotate_quant(x[1:2], torch.eye(16), 16)
    assert math.isnan(scales_i[0])


# ----------------------------------------------------------------------------- W4 weights

def test_w4_golden_bytes(golden_dir):
    rows = [l.split() for l in open(os.path.join(golden_dir, "w4_bytes.txt"))
            if l.strip() and not l.startswith("#")]
    packed = np.array([[int(r[0], 16)] for r in rows], dtype=np.uint8).view(np.int8)
    w = oracle.unpack_w4(packed, 2)
    assert w.tolist() == [[int(r[1]), int(r[2])] for r in rows]
    np.testing.assert_array_equal(oracle.pack_w4(w), packed)


def test_all_256_bytes_round_trip():
    packed = np.arange(256, dtype=np.uint8).view(np.int8).reshape(256, 1)
    w = oracle.unpack_w4(packed, 2)
    assert w.min() == -8 and w.max() == 7
    assert len({tuple(r) for r in w.tolist()}) == 256          # a bijection onto [-8,7]^2
    np.testing.assert_array_equal(oracle.pack_w4(w), packed)


def test_packed_then_unpacked_equals_codes():
    rng = np.random.default_rng(13)
    w = rng.integers(-8, 8, (33, 96)).astype(np.int8)
    np.testing.assert_array_equal(oracle.unpack_w4(oracle.pack_w4(w), 96), w)


def test_unpack_honours_row_pitch():
    rng = np.random.default_rng(14)
    w = rng.integers(-8, 8, (5, 32)).astype(np.int8)
    p = oracle.pack_w4(w)
    wide = np.zeros((5, 40), dtype=np.int8)
    wide[:, :16] = p
    np.testing.assert_array_equal(oracle.unpack_w4(wide[:, :16], 32), w)


# ----------------------------------------------------------------------------- GEMM

def test_gemm_matches_int64_matmul():
    rng = np.random.default_rng(15)
    for M, N, K in ((1, 1, 2), (3, 9, 64), (9, 7, 48)):
        q = rng.integers(-8, 8, (M, K)).astype(np.int8)
        w = rng.integers(-8, 8, (N, K)).astype(np.int8)
        np.testing.assert_array_equal(oracle.gemm_s32(q, w), q.astype(np.int64) @ w.T.astype(np.int64))


def test_gemm_extremes():
    K = 4096
    q = np.full((2, K), -8, np.int8)
    q[1] = 7
    w = np.full((2, K), -8, np.int8)
    w[1] = 7
    acc = oracle.gemm_s32(q, w)
    assert acc.tolist() == [[64 * K, -56 * K], [-56 * K, 49 * K]]


def test_gemm_overflow_guard_at_64k():
    """|acc| <= 64 K; the guard fires exactly when that exceeds INT32_MAX."""
    K_fit = (2 ** 31 - 1) // 64 // 16 * 16
    q = np.full((1, K_fit), -8, np.int8)
    assert oracle.gemm_s32(q, q)[0, 0] == 64 * K_fit
    K_over = K_fit + 16
    q = np.full((1, K_over), -8, np.int8)
    with pytest.raises(oracle.oracle.OracleError):
        oracle.gemm_s32(q, q)


# ----------------------------------------------------------------------------- epilogue

def test_unit_scales_give_accumulator_exactly():
    rng = np.random.default_rng(16)
    acc = rng.integers(-(2 ** 20), 2 ** 20, (4, 5)).astype(np.int32)
    out = oracle.epilogue(acc, np.ones(4, np.float32), torch.ones(5), None, torch.float32)
    np.testing.assert_array_equal(out.numpy(), acc.astype(np.float32))


def test_epilogue_order_is_acc_times_a_then_w_then_bias():
    rng = np.random.default_rng(17)
    found = 0
    for _ in range(2000):
        acc = np.int32(rng.integers(-50000, 50000))
        a = np.float32(rng.uniform(0.01, 2))
        w = np.float32(rng.uniform(0.005, 0.02))
        left = (np.float32(acc) * a) * w
        right = np.float32(acc) * (a * w)
        if left == right:
            continue
        found += 1
        out = oracle.epilogue(np.array([[acc]]), np.array([a]), torch.tensor([w]), None,
                              torch.float32)
        assert out.item() == left and out.item() != right
    assert found > 50


def test_epilogue_bias_and_output_rounding():
    rng = np.random.default_rng(18)
    acc = rng.integers(-3000, 3000, (3, 8)).astype(np.int32)
    a = rng.uniform(0.1, 1, 3).astype(np.float32)
    w = torch.from_numpy(rng.uniform(0.005, 0.02, 8)).to(torch.bfloat16)
    b = torch.from_numpy(rng.normal(0, 0.1, 8)).to(torch.bfloat16)
    out = oracle.epilogue(acc, a, w, b, torch.bfloat16)
    o = (acc.astype(np.float32) * a[:, None]) * w.float().numpy()[None, :]
    o = o + b.float().numpy()[None, :]
    ref = torch.from_numpy(o.astype(np.float32)).to(torch.bfloat16)
    assert torch.equal(out, ref)


def test_fp16_output_overflows_to_inf():
    acc = np.array([[100000]], np.int32)
    out = oracle.epilogue(acc, np.ones(1, np.float32), torch.ones(1, dtype=torch.float16), None,
                          torch.float16)
    assert math.isinf(out.float().item())


# ----------------------------------------------------------------------------- composition

def test_linear_tiny_brute_force():
    """The whole path on tiny shapes against an independent numpy/torch evaluation."""
    for dt, g, rot in (("bf16", 16, "haar"), ("f16", 64, "hadamard"), ("f32", 16, "haar")):
        case = W.LinearCase("t", M=9, K=128, N=7, g=g, dtype=dt, rotation=rot, seed=19)
        inp = W.make_linear_inputs(case)
        out, codes, scales = oracle.linear(inp["x"], inp["R"], g, inp["w_packed"], inp["w_scale"],
                                           inp["bias"])
        x = inp["x"].to(torch.float64).numpy().reshape(9, 128 // g, g)
        y, unsafe = _independent_round((x @ inp["R"].to(torch.float64).numpy()).reshape(9, 128), dt)
        assert not unsafe.any()
        amax = np.abs(y).max(1).astype(np.float32)
        s = np.maximum(amax / np.float32(7), np.float32(FLT_MIN))
        np.testing.assert_array_equal(scales, s)
        q = np.clip(np.rint(y.astype(np.float32) / s[:, None]), -8, 7).astype(np.int8)
        np.testing.assert_array_equal(codes, q)
        p = inp["w_packed"].numpy().view(np.uint8)
        wl = (p & 0xF).astype(np.int16)
        wh = (p >> 4).astype(np.int16)
        wk = np.empty((7, 128), np.int16)
        wk[:, 0::2] = np.where(wl >= 8, wl - 16, wl)
        wk[:, 1::2] = np.where(wh >= 8, wh - 16, wh)
        acc = q.astype(np.int64) @ wk.T.astype(np.int64)
        o = (acc.astype(np.float32) * s[:, None]) * inp["w_scale"].float().numpy()[None, :]
        if inp["bias"] is not None:
            o = o + inp["bias"].float().numpy()[None, :]
        ref = torch.from_numpy(o.astype(np.float32)).to(TORCH_DT[dt])
        assert torch.equal(out, ref)


def test_linear_rows_cols_subset_matches_full():
    case = W.LinearCase("t", M=12, K=256, N=10, g=64, dtype="bf16", rotation="haar", seed=20)
    inp = W.make_linear_inputs(case)
    full, codes, scales = oracle.linear(inp["x"], inp["R"], 64, inp["w_packed"], inp["w_scale"],
                                        inp["bias"])
    rows, cols = [11, 0, 5], [9, 2]
    sub, c2, s2 = oracle.linear(inp["x"], inp["R"], 64, inp["w_packed"], inp["w_scale"],
                                inp["bias"], rows=rows, cols=cols)
    assert torch.equal(sub, full[rows][:, cols])
    np.testing.assert_array_equal(c2, codes[rows])
    np.testing.assert_array_equal(s2, scales[rows])


# ------------------------------------------------------------------- W8A8 variant

def _golden_int8_rows(golden_dir):
    rows = []
    for line in open(os.path.join(golden_dir, "quant_rows_int8.txt")):
        if line.startswith("#") or not line.strip():
            continue
        s_in, ys, s, qs = [c.strip() for c in line.split("|")]
        rows.append((None if s_in == "dyn" else float(s_in), [float(v) for v in ys.split()],
                     float(s), [int(v) for v in qs.split()]))
    return rows


def test_int8_quantizer_golden_rows(golden_dir):
    for s_in, ys, s, qs in _golden_int8_rows(golden_dir):
        codes, scales = oracle.quantize_int8(np.array([ys]), scale_in=s_in)
        assert scales[0] == np.float32(s), (ys, scales[0])
        np.testing.assert_array_equal(codes[0], qs)


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
def test_int8_dynamic_codes_reach_127_never_minus_128_and_reconstruct(dt):
    rng = np.random.default_rng(41)
    y = oracle.round_to(rng.standard_normal((64, 512)) * 3.0, W.DTYPES[dt])
    y[5] = 0.0
    codes, scales = oracle.quantize_int8(y)
    amax = np.abs(y).max(axis=1)
    live = amax > 0
    np.testing.assert_array_equal(scales[live], (amax[live].astype(np.float32) / np.float32(127)))
    assert (np.abs(codes[live]).max(axis=1) == 127).all()
    assert (codes != -128).all()
    # |y - q s| <= s / 2, plus the fp32 quotient's own rounding, which can move a value within
    # |t| 2^-24 of a half-integer across it (|t| <= 127)
    err = np.abs(y[live] - codes[live].astype(np.float64) * scales[live, None])
    assert (err <= scales[live, None] * (0.5 + 127 * 2.0 ** -24) * (1 + 1e-9)).all()


def test_w8a8_linear_tiny_brute_force():
    """Independent numpy/torch evaluation of the W8A8 path on tiny shapes: group rotation in
    float64 rounded to the dtype, INT8 grid, int64 matmul with INT8 weights, fp32 epilogue."""
    rng = np.random.default_rng(43)
    for dt, (M, N, K, g) in [("bf16", (5, 7, 64, 16)), ("f32", (3, 4, 128, 64)),
                             ("f16", (2, 9, 256, 256))]:
        tdt = W.DTYPES[dt]
        x = torch.from_numpy(rng.standard_normal((M, K))).to(tdt)
        R = W.haar_orthogonal(g, torch.Generator().manual_seed(g)).to(tdt)
        w = torch.from_numpy(rng.integers(-128, 128, size=(N, K), dtype=np.int8))
        ws = torch.from_numpy(rng.uniform(0.005, 0.02, N)).to(tdt)
        b = torch.from_numpy(rng.standard_normal(N) * 0.1).to(tdt)
        got, codes, scales = oracle.linear_w8a8(x, R, g, w, ws, b)
        xd = x.double().numpy().reshape(M, K // g, g)
        y = torch.from_numpy((xd @ R.double().numpy()).reshape(M, K)).to(tdt).double().numpy()
        s = (np.abs(y).max(axis=1).astype(np.float32) / np.float32(127)).astype(np.float32)
        s = np.maximum(s, np.float32(np.finfo(np.float32).tiny))
        q = np.clip(np.rint(y.astype(np.float32) / s[:, None]), -128, 127).astype(np.int64)
        np.testing.assert_array_equal(codes, q)
        np.testing.assert_array_equal(scales, s)
        acc = q @ w.numpy().astype(np.int64).T
        o = acc.astype(np.float32) * s[:, None]
        o = o * ws.float().numpy()[None, :]
        o = o + b.float().numpy()[None, :]
        assert torch.equal(got, torch.from_numpy(o).to(tdt))


# ------------------------------------------------------------------- packed quantizer

def test_philox_known_answer_vectors(golden_dir):
    n = 0
    for line in open(os.path.join(golden_dir, "philox4x32_10_kat.txt")):
        if line.startswith("#") or not line.strip():
            continue
        v = [int(t, 16) for t in line.split()]
        np.testing.assert_array_equal(oracle.philox4x32_10(v[:4], v[4:6]), v[6:10])
        n += 1
    assert n == 3


def test_packed_nearest_equals_packed_codes_of_the_quantizer():
    rng = np.random.default_rng(44)
    y = rng.standard_normal((9, 64)) * 2
    y[3] = 0
    packed, scales = oracle.quantize_packed(y, np.arange(9), 64)
    codes, s2 = oracle.quantize(y)
    np.testing.assert_array_equal(scales, s2)
    np.testing.assert_array_equal(packed.view(np.int8), oracle.pack_w4(codes))


def test_stochastic_rounding_first_draw_worked_by_hand():
    """Element 0 of a tensor with seed 0 and offset 0 draws Philox(counter 0, key 0) word 0 =
    0x6627e8d5, so u = 0x6627e8 * 2^-24 = 0.39904...; a row [2.7, 7, ...] has s = 1 and t = 2.7:
    floor(2.7 + u) = 3; with 2.5 in its place floor(2.5 + u) = 2; with -0.7, floor(-0.3) = -1."""
    u = np.float32(0x6627e8) * np.float32(2.0 ** -24)
    assert abs(float(u) - 0.399) < 1e-3
    for first, want in ((2.7, 3), (2.5, 2), (-0.7, -1)):
        y = np.array([[first, 7.0] + [0.0] * 14])
        packed, scales = oracle.quantize_packed(y, [0], 16, stochastic=True, seed=0, offset=0)
        assert scales[0] == 1.0
        lo = int(packed[0, 0]) & 0xF
        assert (lo - 16 if lo >= 8 else lo) == want


def _unpack_rows(packed):
    lo = (packed & 0xF).astype(np.int64)
    hi = (packed >> 4).astype(np.int64)
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty((packed.shape[0], packed.shape[1] * 2), dtype=np.int64)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return out


def test_stochastic_rounding_brackets_the_quotient_and_is_unbiased():
    rng = np.random.default_rng(45)
    M, K = 64, 2048
    y = rng.uniform(-6.5, 6.5, size=(M, K))
    y[:, 0] = 7.0                                   # s = 1 in every row: t = y
    y[:, 1::97] = np.round(y[:, 1::97])             # exact integers stay
    packed, scales = oracle.quantize_packed(y, np.arange(M), K, stochastic=True, seed=1234)
    assert (scales == 1.0).all()
    q = _unpack_rows(packed)
    t = y.astype(np.float32).astype(np.float64)
    assert ((q == np.floor(t)) | (q == np.floor(t) + 1)).all()
    ints = t == np.round(t)
    np.testing.assert_array_equal(q[ints], t[ints])
    frac = t - np.floor(t)
    assert abs(float((q - np.floor(t)).mean() - frac.mean())) < 0.01   # E[q] = t
    again, _ = oracle.quantize_packed(y, np.arange(M), K, stochastic=True, seed=1234)
    np.testing.assert_array_equal(packed, again)
    other, _ = oracle.quantize_packed(y, np.arange(M), K, stochastic=True, seed=1235)
    assert (packed != other).any()
    shifted, _ = oracle.quantize_packed(y, np.arange(M), K, stochastic=True, seed=1234, offset=1)
    assert (packed != shifted).any()
