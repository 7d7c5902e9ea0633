"""Shared helpers for the GPU parity tests: move seeded CPU inputs to the device with
their strides, read the stage-1 result out of the workspace, and compare with the oracle.

Acceptance (per the method's numeric contract):
  - unpacked weights and INT32 accumulators: bit-exact;
  - INT4 codes: differ only by +-1, at a mismatch rate <= 1e-4;
  - outputs: rtol 2e-2 / atol 1e-2 for bf16/fp16, rtol 1e-5 for fp32 against the full
    oracle, and bit-exact against the oracle's GEMM + epilogue evaluated on the GPU's own
    codes and scales.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from rotated_w4a4_quantized_group_b200 import ck

CODE_MISMATCH_MAX = 1e-4
ULP = {torch.float32: 2.0 ** -23, torch.float16: 2.0 ** -10, torch.bfloat16: 2.0 ** -7}
TOL = {torch.bfloat16: (2e-2, 1e-2), torch.float16: (2e-2, 1e-2), torch.float32: (1e-5, 0.0)}


def to_device(t: torch.Tensor | None, device="cuda") -> torch.Tensor | None:
    """Copy a CPU tensor to the device keeping its exact strides and storage offset."""
    if t is None:
        return None
    n = t.untyped_storage().nbytes() // t.element_size()
    base = torch.empty(n, dtype=t.dtype)
    base.untyped_storage().copy_(t.untyped_storage())
    dbase = base.to(device)
    return dbase.as_strided(t.shape, t.stride(), t.storage_offset())


def sample_rows(M: int, n: int = 48, seed: int = 0) -> np.ndarray:
    if M <= n:
        return np.arange(M, dtype=np.int64)
    rng = np.random.default_rng(seed)
    edge = [0, 1, 127, 128, M // 2, M - 129, M - 128, M - 2, M - 1]
    rest = rng.choice(M, size=n - len(edge), replace=False)
    return np.unique(np.concatenate([edge, rest]).clip(0, M - 1)).astype(np.int64)


def sample_cols(N: int, n: int = 64, seed: int = 1) -> np.ndarray:
    if N <= n:
        return np.arange(N, dtype=np.int64)
    rng = np.random.default_rng(seed)
    edge = [0, 1, 31, 32, 255, 256, 511, N - 257, N - 256, N - 1]
    rest = rng.choice(N, size=n - len(edge), replace=False)
    return np.unique(np.concatenate([edge, rest]).clip(0, N - 1)).astype(np.int64)


def workspace_stage1(ws: torch.Tensor, M: int, K: int):
    """(codes (M, K) int8, scales (M,) fp32) that ck_w4a4_linear left in its workspace."""
    P = ck.workspace_codes_pitch(K)
    off = ck.workspace_scales_offset(M, K)
    codes = ws[: M * P].view(torch.int8).view(M, P)[:, :K]
    scales = ws[off: off + 4 * M].view(torch.float32)
    return codes, scales


def scale_rtol(dtype, g: int) -> float:
    """How far a row scale may sit from the oracle's.  The scale is fp32(amax) / 7 with amax
    the largest |y|.  For 16-bit inputs y is rounded to the dtype, and fp32 accumulation can
    move that rounding by one dtype ulp.  For fp32 inputs y is the fp32 sum of g products,
    within (g + 2) * 2^-24 of the exactly rounded value the oracle forms in double."""
    if dtype == torch.float32:
        return (g + 2) * 2.0 ** -24
    return ULP[dtype] * 1.01


def compare_stage1(gc: np.ndarray, gs: np.ndarray, oc: np.ndarray, os_: np.ndarray, dtype,
                   what: str = "", g: int = 256):
    """GPU vs oracle codes/scales for the same rows.  Returns the code mismatch count."""
    gc = gc.astype(np.int32)
    oc = oc.astype(np.int32)
    diff = gc - oc
    assert np.abs(diff).max(initial=0) <= 1, f"{what}: a code differs by more than 1"
    rate = float((diff != 0).mean()) if diff.size else 0.0
    assert rate <= CODE_MISMATCH_MAX, f"{what}: code mismatch rate {rate:.3g}"
    finite = np.isfinite(os_)
    np.testing.assert_array_equal(np.isfinite(gs), finite, err_msg=what)
    rel = np.abs(gs[finite].astype(np.float64) - os_[finite]) / os_[finite]
    tol = scale_rtol(dtype, g)
    assert (rel <= tol).all(), f"{what}: scale relative error {rel.max():.3g} > {tol:.3g}"
    return int((diff != 0).sum())


def oracle_on_codes(codes: np.ndarray, scales: np.ndarray, w_packed_cpu: torch.Tensor, K: int,
                    cols, w_scale_cpu, bias_cpu, out_dtype) -> torch.Tensor:
    """The oracle's unpack + GEMM + epilogue evaluated on the given (GPU-produced) codes."""
    w = oracle.unpack_w4(w_packed_cpu[cols], K)
    acc = oracle.gemm_s32(codes, w)
    b = None if bias_cpu is None else bias_cpu[cols]
    return oracle.epilogue(acc, scales, w_scale_cpu[cols], b, out_dtype)


def assert_close(gpu: torch.Tensor, ref: torch.Tensor, dtype, what="", bias=None):
    """|gpu - ref| <= atol + rtol * mag.  mag is |ref|, or, with a bias, |ref - bias| + |bias|:
    the epilogue's last step adds the bias to acc * a * w, and where the two cancel the
    result's own magnitude says nothing about the rounding error of its summands."""
    rtol, atol = TOL[dtype]
    g = gpu.to(torch.float64)
    r = ref.to(torch.float64)
    mag = r.abs()
    if bias is not None:
        b = bias.to(torch.float64).reshape(1, -1)
        mag = (r - b).abs() + b.abs()
    bad = (g - r).abs() > atol + rtol * mag
    assert not bool(bad.any()), f"{what}: {int(bad.sum())} outputs outside rtol {rtol} atol {atol}"
