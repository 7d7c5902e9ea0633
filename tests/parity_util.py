"""Shared helpers for the GPU parity tests: move seeded CPU inputs to the device with
their strides, read the stage-1 result out of the workspace, and compare with the oracle.

Acceptance rule (the method's numeric contract, with the readings the design notes list):
  - unpacked weights and INT32 accumulators: bit-exact;
  - INT4 codes: a GPU code may differ from the oracle's by +-1 only, at a mismatch rate
    <= 1e-4, and only where the oracle's exact quotient y / s lies within the rounding
    distance of a half-integer (a rounding tie).  That distance follows from how far the
    GPU's rotated value and row scale may sit from the oracle's: one ulp of the input dtype
    for the rotated value of a 16-bit input (fp32 accumulation, one final rounding), the
    fp32 accumulation bound g * 2^-24 * sum |x_i R_ic| for an fp32 input, and the row-scale
    bound below;
  - row scales: within one ulp of the input dtype (16-bit inputs) or (g + 2) * 2^-24
    relative (fp32 inputs) of the oracle's;
  - outputs: bit-exact against the oracle's GEMM + epilogue evaluated on the GPU's own codes
    and scales; and against the whole oracle path |gpu - ref| <= atol + rtol * |ref| + extra,
    with rtol 2e-2 / atol 1e-2 for bf16/fp16 and rtol 1e-5 for fp32, where extra is the
    exact first-order effect of the stage-1 differences allowed above (output_widening):
    a tie flip at position k moves the output by a_scale * |w_scale| * |w[n, k]|, a row
    scale that differs by da moves it by |acc| * da * |w_scale|.  A row whose codes and
    scale equal the oracle's gets no widening at all.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from rotated_w4a4_quantized_group_b200 import ck

CODE_MISMATCH_MAX = 1e-4
ULP = {torch.float32: 2.0 ** -23, torch.float16: 2.0 ** -10, torch.bfloat16: 2.0 ** -7}
# significand bits (with the implicit one) and minimum normal exponent of each input dtype
SIG_BITS = {torch.float32: 24, torch.float16: 11, torch.bfloat16: 8}
EMIN = {torch.float32: -126, torch.float16: -14, torch.bfloat16: -126}
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


def dtype_ulp(v: np.ndarray, dtype) -> np.ndarray:
    """One ulp of `dtype` at each |v| (the subnormal quantum below the normal range)."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, EMIN[dtype])
    return np.ldexp(1.0, (e - (SIG_BITS[dtype] - 1)).astype(np.int64))


def tie_distance_bound(y: np.ndarray, s: np.ndarray, abs_terms: np.ndarray, dtype, g: int,
                       dynamic: bool) -> np.ndarray:
    """Largest |t_gpu - t_oracle| for quotients t = y / s, given the oracle's rotated values
    y, its row scales s (broadcast per element) and sum_i |x_i R_ic| per element.

    - rotated value: one dtype ulp for 16-bit inputs; for fp32 inputs the fp32 accumulation
      bound g * 2^-24 / (1 - g * 2^-24) * sum |x_i R_ic| plus the final rounding's ulp;
    - row scale: scale_rtol relative for dynamic scales, 0 for a caller's scale;
    - both quotients are fp32 divisions: 2^-24 relative each."""
    t = np.abs(y) / s
    if dtype == torch.float32:
        gam = g * 2.0 ** -24 / (1.0 - g * 2.0 ** -24)
        dy = gam * abs_terms + dtype_ulp(y, dtype)
    else:
        dy = dtype_ulp(np.abs(y) * (1 + 2.0 ** (1 - SIG_BITS[dtype])), dtype)
    rel_s = scale_rtol(dtype, g) if dynamic else 0.0
    return dy / s + t * (rel_s + 2.0 * 2.0 ** -24) * 1.01 + 1e-12


def _abs_terms(x_rows: np.ndarray, R: np.ndarray, g: int, ks: np.ndarray, r_idx: np.ndarray):
    """sum_i |x[m, jg+i]| |R[i, c]| for the listed (row, channel) pairs (k = jg + c)."""
    out = np.empty(ks.size)
    for e, (r, k) in enumerate(zip(r_idx, ks)):
        j, c = divmod(int(k), g)
        out[e] = np.abs(x_rows[r, j * g:(j + 1) * g]) @ np.abs(R[:, c])
    return out


def compare_stage1(gc: np.ndarray, gs: np.ndarray, oc: np.ndarray, os_: np.ndarray, dtype,
                   what: str = "", g: int = 256, *, x: torch.Tensor | None = None,
                   R: torch.Tensor | None = None, rows=None, scale_in: float | None = None,
                   qmax: int = 7, max_rate: float = CODE_MISMATCH_MAX):
    """GPU vs oracle codes/scales for the same rows; returns the code mismatch count.

    qmax 127 (the W8A8 variant's INT8 grid) keeps every bound; only the mismatch rate limit,
    max_rate, is the caller's: with 16-bit inputs one dtype ulp of y moves the INT8 quotient
    by up to 127 * 2^-7 ~ 1, so the rate follows the rotation's rounding flips.

    Every mismatched code must sit at a rounding tie: x and R (the inputs, CPU) and rows
    (which rows of x the arrays hold; all rows when None) let the check recompute the
    oracle's rotated values there.  A call that finds a mismatch without them fails."""
    gc = gc.astype(np.int32)
    oc = oc.astype(np.int32)
    diff = gc - oc
    assert np.abs(diff).max(initial=0) <= 1, f"{what}: a code differs by more than 1"
    rate = float((diff != 0).mean()) if diff.size else 0.0
    assert rate <= max_rate, f"{what}: code mismatch rate {rate:.3g}"
    finite = np.isfinite(os_)
    np.testing.assert_array_equal(np.isfinite(gs), finite, err_msg=what)
    rel = np.abs(gs[finite].astype(np.float64) - os_[finite]) / os_[finite]
    tol = scale_rtol(dtype, g)
    if scale_in is not None:
        tol = 0.0
    assert (rel <= tol).all(), f"{what}: scale relative error {rel.max():.3g} > {tol:.3g}"
    n_mis = int((diff != 0).sum())
    if n_mis:
        assert x is not None and R is not None, f"{what}: mismatches but no inputs to check ties"
        r_idx, ks = np.nonzero(diff)
        ur, inv = np.unique(r_idx, return_inverse=True)
        src_rows = ur if rows is None else np.asarray(rows)[ur]
        y = oracle.rotate(x, R, g, rows=src_rows)                  # (len(ur), K) float64
        xr = oracle.decode(x[torch.from_numpy(np.asarray(src_rows))].contiguous())
        Rd = oracle.decode(R.contiguous())
        ye = y[inv, ks]
        se = os_[r_idx].astype(np.float64)
        terms = _abs_terms(xr, Rd, g, ks, inv)
        bound = tie_distance_bound(ye, se, terms, dtype, g, dynamic=scale_in is None)
        t = ye / se
        dist = np.abs(t - (np.floor(t) + 0.5))
        far = dist > bound
        assert not far.any(), (
            f"{what}: {int(far.sum())} mismatched codes are not at a rounding tie "
            f"(distance {dist[far].min():.3g} > bound {bound[far].min():.3g})")
    return n_mis


def oracle_on_codes(codes: np.ndarray, scales: np.ndarray, w_packed_cpu: torch.Tensor, K: int,
                    cols, w_scale_cpu, bias_cpu, out_dtype) -> torch.Tensor:
    """The oracle's unpack + GEMM + epilogue evaluated on the given (GPU-produced) codes."""
    w = oracle.unpack_w4(w_packed_cpu[cols], K)
    acc = oracle.gemm_s32(codes, w)
    b = None if bias_cpu is None else bias_cpu[cols]
    return oracle.epilogue(acc, scales, w_scale_cpu[cols], b, out_dtype)


def output_widening(gc: np.ndarray, oc: np.ndarray, gs: np.ndarray, os_: np.ndarray,
                    w_packed_cpu: torch.Tensor, K: int, cols, w_scale_cpu) -> np.ndarray:
    w = oracle.unpack_w4(w_packed_cpu[cols], K).astype(np.int64)
    return widening_for_weights(gc, oc, gs, os_, w, w_scale_cpu[torch.as_tensor(cols)])


def widening_for_weights(gc: np.ndarray, oc: np.ndarray, gs: np.ndarray, os_: np.ndarray,
                         w: np.ndarray, w_scale_cols) -> np.ndarray:
    """(rows, cols) bound on |out_gpu - out_oracle| that the stage-1 differences the parity
    rule allows can cause, beyond the output rounding that rtol covers.

    With acc = q . w the epilogue gives fp32(fp32(acc * a) * ws) (+ bias, rounded last):
      - each code that differs (at a tie) moves acc by |w[n, k]|: |dacc| <= sum_mis |w[n, k]|;
      - a row scale that differs moves the output by |acc| * |a_gpu - a_oracle| * |ws|;
      - and where either differs, the two products are rounded from different values:
        up to 2 * 2^-24 relative to |acc * a * ws| on each side.
    A row whose codes and scale both equal the oracle's gives an identical output (0)."""
    g32 = gc.astype(np.int32)
    o32 = oc.astype(np.int32)
    mis = (g32 != o32).astype(np.int64) * np.abs(g32 - o32)
    w = np.asarray(w, dtype=np.int64)
    dacc = (mis @ np.abs(w).T).astype(np.float64)
    acc = np.abs((o32.astype(np.int64) @ w.T).astype(np.float64))
    ag = np.abs(gs.astype(np.float64))
    ao = np.abs(os_.astype(np.float64))
    amax = np.maximum(ag, ao)[:, None]
    da = np.abs(gs.astype(np.float64) - os_.astype(np.float64))[:, None]
    differs = (mis.any(axis=1) | (gs != os_))[:, None]
    ws = np.abs(torch.as_tensor(w_scale_cols).to(torch.float64).numpy())[None, :]
    extra = ws * (dacc * amax + acc * da + differs * 4.0 * 2.0 ** -24 * (acc + dacc) * amax)
    return extra * 1.01


def assert_close(gpu: torch.Tensor, ref: torch.Tensor, dtype, what="", extra=None):
    """|gpu - ref| <= atol + rtol * |ref| + extra, element by element (extra: the per-output
    widening for mismatched codes, or None)."""
    rtol, atol = TOL[dtype]
    g = gpu.to(torch.float64)
    r = ref.to(torch.float64)
    lim = atol + rtol * r.abs()
    if extra is not None:
        lim = lim + torch.as_tensor(extra, dtype=torch.float64)
    bad = (g - r).abs() > lim
    assert not bool(bad.any()), f"{what}: {int(bad.sum())} outputs outside rtol {rtol} atol {atol}"
