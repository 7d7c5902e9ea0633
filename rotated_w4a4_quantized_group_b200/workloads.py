"""Seeded synthetic inputs for the ConvRot W4A4 linear and its rotate+quantize stage.

This module only draws random inputs in the layouts the library accepts; it holds
none of the method's arithmetic (no rotation, no quantizer, no GEMM).  It is the one
module shared by the CPU oracle's tests and the CUDA path.

The shapes follow the activation shapes the comfy-kitchen Ascend pages measure:
Z-Image tokens x channels ([32|8192] x [3840|10240], PR #155 "Add fused RotateQuant
backend", performance table) and Krea layers (K = 6144/16384, PR #201 "Avoid
activation pack/unpack in ConvRot W4A4", operator-timing table).  The pages give no
value distributions, so each case states its own recipe below.

All tensors are CPU torch tensors.  ``x`` may be a strided view (row pitch 2K, or a
column-major transpose); ``w_packed`` is (N, K/2) int8 with two signed 4-bit codes per
byte, the even-k code in the low nibble.
"""
from __future__ import annotations

import dataclasses
import math

import torch

DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
ELEM_BYTES = {"f32": 4, "f16": 2, "bf16": 2}


@dataclasses.dataclass(frozen=True)
class LinearCase:
    """One W4A4 linear workload: x (M, K) rotated with a g x g matrix, W4 weights (N, K/2)."""

    name: str
    M: int
    K: int
    N: int
    g: int
    dtype: str                    # activation, rotation, scale and output dtype
    rotation: str = "hadamard"    # "hadamard" (Sylvester H_g / sqrt(g)) or "haar" (QR of a Gaussian)
    layout: str = "contiguous"    # "contiguous", "pitch2k" (rows of a (M, 2K) buffer), "colmajor"
    x_dist: str = "normal"        # "normal" or "student_t3"
    outlier_frac: float = 0.01    # fraction of K channels scaled by outlier_scale
    outlier_scale: float = 20.0
    zero_row_frac: float = 0.0    # fraction of rows set to exactly zero
    w_extreme_row_frac: float = 0.0  # fraction of weight rows whose codes are all -8 or 7
    has_bias: bool = True
    bias_std: float = 0.1
    seed: int = 0

    def replace(self, **kw) -> "LinearCase":
        return dataclasses.replace(self, **kw)


@dataclasses.dataclass(frozen=True)
class RotateCase:
    """One rotate+quantize-only workload (x (M, K), g x g Hadamard rotation)."""

    name: str
    M: int
    K: int
    g: int
    dtype: str
    layout: str = "contiguous"    # "contiguous" or "pitch2k"
    outlier_frac: float = 0.01
    outlier_scale: float = 20.0
    seed: int = 0


# The four full linear workloads.  Sizes are the Z-Image (K = 3840 / 10240) and
# Krea (K = 16384) activation shapes; N is the layer's output width.
LINEAR_CASES = {
    "zimage_m32_k3840_n3840_g64_bf16": LinearCase(
        "zimage_m32_k3840_n3840_g64_bf16", M=32, K=3840, N=3840, g=64, dtype="bf16",
        rotation="hadamard", seed=0xC0417000),
    "zimage_m8192_k3840_n3840_g64_bf16": LinearCase(
        "zimage_m8192_k3840_n3840_g64_bf16", M=8192, K=3840, N=3840, g=64, dtype="bf16",
        rotation="haar", seed=0xC0417001),
    "zimage_m8192_k10240_n3840_g256_f16": LinearCase(
        "zimage_m8192_k10240_n3840_g256_f16", M=8192, K=10240, N=3840, g=256, dtype="f16",
        rotation="hadamard", outlier_frac=0.005, outlier_scale=50.0, zero_row_frac=0.01,
        has_bias=False, seed=0xC0417002),
    "krea_m4096_k16384_n6144_g16_f32_colmajor": LinearCase(
        "krea_m4096_k16384_n6144_g16_f32_colmajor", M=4096, K=16384, N=6144, g=16,
        dtype="f32", rotation="haar", layout="colmajor", x_dist="student_t3",
        outlier_frac=0.0, w_extreme_row_frac=0.10, bias_std=1.0, seed=0xC0417003),
}

# The headline workload the benchmark times.
HEADLINE = "zimage_m8192_k3840_n3840_g64_bf16"


def sweep_cases() -> list[RotateCase]:
    """The 72 rotate+quantize cases: M x K x g x dtype x layout."""
    out = []
    idx = 0
    for M in (32, 8192):
        for K in (3840, 10240):
            for g in (16, 64, 256):
                for dt in ("f32", "f16", "bf16"):
                    for layout in ("contiguous", "pitch2k"):
                        out.append(RotateCase(f"rq_m{M}_k{K}_g{g}_{dt}_{layout}", M=M, K=K, g=g,
                                              dtype=dt, layout=layout, seed=0xC0418000 + idx))
                        idx += 1
    return out


def _gen(seed: int) -> torch.Generator:
    gen = torch.Generator()
    gen.manual_seed(int(seed) & 0xFFFFFFFFFFFF)
    return gen


def hadamard(g: int) -> torch.Tensor:
    """Sylvester Hadamard matrix H_g / sqrt(g) in float64 (entries +-1/sqrt(g), exact in every dtype)."""
    assert g >= 1 and (g & (g - 1)) == 0
    h = torch.ones(1, 1, dtype=torch.float64)
    while h.shape[0] < g:
        h = torch.cat([torch.cat([h, h], 1), torch.cat([h, -h], 1)], 0)
    return h / math.sqrt(g)


def haar_orthogonal(g: int, gen: torch.Generator) -> torch.Tensor:
    """Random orthogonal g x g matrix (float64): QR of a Gaussian, with the diagonal of R made positive."""
    a = torch.randn(g, g, generator=gen, dtype=torch.float64)
    q, r = torch.linalg.qr(a)
    return (q * torch.sign(torch.diagonal(r)).unsqueeze(0)).contiguous()


def _activations(M: int, K: int, dist: str, outlier_frac: float, outlier_scale: float,
                 zero_row_frac: float, gen: torch.Generator) -> torch.Tensor:
    if dist == "normal":
        x = torch.randn(M, K, generator=gen, dtype=torch.float32)
    elif dist == "student_t3":
        z = torch.randn(M, K, generator=gen, dtype=torch.float32)
        c = torch.randn(3, M, K, generator=gen, dtype=torch.float32).square_().sum(0)
        x = z / torch.sqrt(c / 3.0)
    else:
        raise ValueError(dist)
    n_out = int(round(outlier_frac * K))
    if n_out:
        ch = torch.randperm(K, generator=gen)[:n_out]
        x[:, ch] *= outlier_scale
    n_zero = int(round(zero_row_frac * M))
    if n_zero:
        rows = torch.randperm(M, generator=gen)[:n_zero]
        x[rows, :] = 0.0
    return x


def _place(x: torch.Tensor, layout: str) -> torch.Tensor:
    """Return x (M, K) in the requested memory layout (values unchanged)."""
    M, K = x.shape
    if layout == "contiguous":
        return x.contiguous()
    if layout == "pitch2k":
        buf = torch.zeros(M, 2 * K, dtype=x.dtype)
        buf[:, :K] = x
        return buf[:, :K]
    if layout == "colmajor":
        return x.t().contiguous().t()
    raise ValueError(layout)


def _weights(N: int, K: int, extreme_frac: float, gen: torch.Generator) -> torch.Tensor:
    """(N, K/2) int8 bytes.  A uniform byte holds two independent uniform 4-bit codes."""
    w = torch.randint(0, 256, (N, K // 2), generator=gen, dtype=torch.int32)
    n_ext = int(round(extreme_frac * N))
    if n_ext:
        rows = torch.randperm(N, generator=gen)[:n_ext]
        # each nibble is 0x7 (code 7) or 0x8 (code -8)
        lo = torch.where(torch.rand(n_ext, K // 2, generator=gen) < 0.5, 0x7, 0x8)
        hi = torch.where(torch.rand(n_ext, K // 2, generator=gen) < 0.5, 0x7, 0x8)
        w[rows] = (lo | (hi << 4)).to(torch.int32)
    return w.to(torch.uint8).view(torch.int8)


def rotation_matrix(kind: str, g: int, dtype: str, gen: torch.Generator) -> torch.Tensor:
    r = hadamard(g) if kind == "hadamard" else haar_orthogonal(g, gen)
    return r.to(DTYPES[dtype]).contiguous()


def make_linear_inputs(case: LinearCase) -> dict:
    """Draw every input of one linear case (CPU tensors)."""
    gen = _gen(case.seed)
    R = rotation_matrix(case.rotation, case.g, case.dtype, gen)
    x32 = _activations(case.M, case.K, case.x_dist, case.outlier_frac, case.outlier_scale,
                       case.zero_row_frac, gen)
    x = _place(x32.to(DTYPES[case.dtype]), case.layout)
    w_packed = _weights(case.N, case.K, case.w_extreme_row_frac, gen)
    w_scale = (torch.rand(case.N, generator=gen, dtype=torch.float64) * 0.015 + 0.005)
    w_scale = w_scale.to(DTYPES[case.dtype])
    bias = None
    if case.has_bias:
        bias = (torch.randn(case.N, generator=gen, dtype=torch.float64) * case.bias_std)
        bias = bias.to(DTYPES[case.dtype])
    return {"x": x, "R": R, "w_packed": w_packed, "w_scale": w_scale, "bias": bias}


def make_rotate_inputs(case: RotateCase) -> dict:
    gen = _gen(case.seed)
    R = rotation_matrix("hadamard", case.g, case.dtype, gen)
    x32 = _activations(case.M, case.K, "normal", case.outlier_frac, case.outlier_scale, 0.0, gen)
    x = _place(x32.to(DTYPES[case.dtype]), case.layout)
    return {"x": x, "R": R}


def strides_of(x: torch.Tensor) -> tuple[int, int]:
    """(stride_m, stride_k) of a 2-D view, in elements."""
    return int(x.stride(0)), int(x.stride(1))


def algorithmic_bytes_rotate_quant(M: int, K: int, g: int, dtype: str) -> int:
    """Bytes a rotate+quantize pass must move: x once, codes once, scales, R once."""
    eb = ELEM_BYTES[dtype]
    return M * K * eb + M * K + 4 * M + g * g * eb


def algorithmic_bytes_gemm(M: int, K: int, N: int, dtype: str, has_bias: bool) -> int:
    """Bytes the W4A4 GEMM must move: int8 codes, packed weights, row scales, output, w_scale, bias."""
    eb = ELEM_BYTES[dtype]
    return M * K + N * K // 2 + 4 * M + M * N * eb + N * eb * (2 if has_bias else 1)
