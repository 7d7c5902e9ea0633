/*
 * ck.h -- C ABI of the ConvRot W4A4 quantized linear for NVIDIA B200 (sm_100a).
 *
 * The operation (comfy-kitchen PR #198 "Consolidate INT8, RotateQuant, RoPE and
 * ConvRot W4A4 backends", section "W4A4 correctness and performance scope"; PR #201
 * "Avoid activation pack/unpack in ConvRot W4A4", section "Summary"):
 *
 *   stage 1  y[m, j*g + c] = sum_i x[m, j*g + i] * R[i, c]     (rotation per K-group,
 *                                                               result in x's dtype)
 *            s[m] = max(fp32(max_k |y[m, k]|) / 7, FLT_MIN)    (per-row scale)
 *            q[m, k] = clamp(round_half_even(y[m, k] / s[m]), -8, 7)   (INT8 storage)
 *   stage 2  acc[m, n] = sum_k q[m, k] * w[n, k]               (exact INT32)
 *            out[m, n] = cvt(((fp32(acc) * s[m]) * w_scale[n]) + bias[n])
 *
 * where w[n, k] are signed 4-bit weight codes packed two per byte, (N, K/2), the
 * even k in the low nibble (comfy_kitchen/tensor/svdquant_w4a4.py module docstring
 * for the (N, K // 2) layout).
 *
 * Conventions for every entry point:
 *   - All data pointers are DEVICE pointers owned by the caller; the library
 *     allocates no memory and keeps no state between calls (except cached kernel
 *     attributes and a per-process table of driver entry points).
 *   - Work is enqueued on `stream`; the call returns before the GPU finishes.
 *   - Arguments are validated on the host before anything is launched; an invalid
 *     call returns an error and touches no memory.
 *   - Strides and leading dimensions are in ELEMENTS of the tensor they describe
 *     (bytes for int8 tensors).
 *   - M == 0 is a successful no-op ("empty rows").
 *   - dev_status, when not NULL, is a device int that a kernel sets to
 *     CK_ERR_TIMEOUT if one of its bounded internal waits expires (the kernel then
 *     exits early and its outputs are undefined).  The caller clears it and reads
 *     it after synchronising the stream.
 */
#ifndef CK_H
#define CK_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    CK_OK = 0,
    CK_ERR_INVALID_ARG = 1,   /* null pointer, bad size, bad dtype, bad group size        */
    CK_ERR_UNSUPPORTED = 2,   /* a valid call this library does not implement             */
    CK_ERR_OVERFLOW = 3,      /* 64 * K > INT32_MAX: the INT32 accumulator could overflow */
    CK_ERR_WORKSPACE = 4,     /* workspace missing or smaller than required               */
    CK_ERR_CUDA = 5,          /* a CUDA runtime/driver call or a launch failed            */
    CK_ERR_TIMEOUT = 6        /* written to *dev_status by a kernel whose wait expired    */
} ck_status;

typedef enum { CK_F32 = 0, CK_F16 = 1, CK_BF16 = 2, CK_I8 = 3 } ck_dtype;

/*
 * Stage 1: group-wise rotation, then row-wise signed-INT4 quantization with codes
 * kept in INT8 storage (PR #198 "W4A4 correctness and performance scope": rotation
 * keeps the FP32/FP16/BF16 input dtype, the reference signed-INT4 quantizer; PR #201
 * "Summary": codes are never packed; PR #155 "Add fused RotateQuant backend": group
 * sizes 16/64/256, batched / non-contiguous inputs, asymmetric rotations, zero-scale
 * handling).
 *
 *   x        (M, K) activations of x_dtype (CK_F32, CK_F16 or CK_BF16), element
 *            (m, k) at x[m*stride_m + k*stride_k]; any strides (row pitch, transposed
 *            views).  A batched (..., K) tensor is passed as its flattened 2-D view.
 *   R        (g, g) row-major rotation in x_dtype; y_group = x_group @ R.
 *   g        16, 64 or 256; K must be a positive multiple of g (and so even).
 *   scale_in NULL: dynamic per-row scales.  Otherwise a device pointer to ONE fp32
 *            tensor-wise scale used for every row after the same lower clamp at
 *            FLT_MIN (a zero scale becomes FLT_MIN, as the eager path does).
 *   codes    (M, K) int8 output, row pitch ldq >= K bytes; values in [-8, 7].
 *   scales   (M,) fp32 output, the scale each row was divided by (always written).
 *
 * The rotated value is the sum rounded once to x_dtype before the absmax.  For fp32 input
 * at g = 16 the sum is formed exactly (fp64 products and sums) and matches an exact
 * evaluation bit for bit; otherwise it accumulates in fp32, so a code may differ by one
 * from an exact-arithmetic evaluation where y / s lies within rounding of a half-integer.
 * Errors: CK_ERR_INVALID_ARG (null x/R/codes/scales, M < 0, K <= 0, K % g != 0,
 * bad g or dtype, ldq < K, R not 16-byte aligned), CK_ERR_UNSUPPORTED (a shape no kernel of
 * this library takes: an fp32 row of more than about 56,000 channels, unless g = 16 and x is
 * row-major or column-major with a 16-byte-aligned pitch), CK_ERR_CUDA (launch failure).
 */
ck_status ck_rotate_quant(const void* x, ck_dtype x_dtype, int64_t M, int64_t K,
                          int64_t stride_m, int64_t stride_k, const void* R, int g,
                          const float* scale_in, int8_t* codes, int64_t ldq, float* scales,
                          int* dev_status, cudaStream_t stream);

/*
 * The whole W4A4 linear (PR #198 "W4A4 correctness and performance scope": INT8
 * codes contracted with npu_quant_matmul-style INT32 accumulation at unit scale,
 * then cast, activation scale, weight scale and bias in eager's order, with an
 * INT32 overflow guard).
 *
 *   x, x_dtype, M, K, stride_m, stride_k, R, g
 *            as in ck_rotate_quant when x_dtype is CK_F32/CK_F16/CK_BF16: stage 1
 *            runs into the workspace, then stage 2.
 *            When x_dtype == CK_I8, x already holds (M, K) int8 codes with row pitch
 *            stride_m (stride_k must be 1), a_scale holds their (M,) fp32 row scales,
 *            and R/g are ignored: the GEMM-only path.
 *   a_scale  (M,) fp32 row scales for CK_I8 input; ignored (may be NULL) otherwise.
 *   w_packed (N, K/2) int8, row pitch w_ld >= K/2 bytes, two signed 4-bit codes per
 *            byte, code of k = 2i in the low nibble of byte i.
 *   w_scale  (N,) per-output-channel weight scale, scale_dtype (CK_F32/F16/BF16).
 *   bias     (N,) of scale_dtype, or NULL.
 *   out      (M, N) of out_dtype (CK_F32/F16/BF16), row pitch ldo >= N.
 *   workspace, workspace_bytes
 *            caller-owned device scratch of at least
 *            ck_w4a4_linear_workspace_bytes(M, N, K, w_ld) bytes, 256-byte aligned.
 *            After a floating-point-input call it holds the stage-1 result: int8
 *            codes (M, K) with row pitch ck_workspace_codes_pitch(K) at offset 0,
 *            then fp32 row scales (M,) at offset ck_workspace_scales_offset(M, K).
 *
 * Errors: CK_ERR_INVALID_ARG, CK_ERR_OVERFLOW (64*K > 2^31 - 1, the bound
 * |acc| <= 8*8*K), CK_ERR_WORKSPACE, CK_ERR_CUDA.
 */
ck_status ck_w4a4_linear(const void* x, ck_dtype x_dtype, int64_t M, int64_t K,
                         int64_t stride_m, int64_t stride_k, const void* R, int g,
                         const float* a_scale, const int8_t* w_packed, int64_t N, int64_t w_ld,
                         const void* w_scale, ck_dtype scale_dtype, const void* bias,
                         void* out, ck_dtype out_dtype, int64_t ldo,
                         void* workspace, size_t workspace_bytes, int* dev_status,
                         cudaStream_t stream);

/*
 * Several linears that read the same activations, as one call (comfy_kitchen/tensor/
 * svdquant_w4a4.py: svdquant_w4a4_grouped_linear runs the projections that share one input,
 * such as attention's Q, K and V, as one linear over their weights fused along N by
 * svdquant_w4a4_fuse_linear_weights, and splits the result per projection).  Stage 1 runs
 * once on x; one stage-2 GEMM covers the stacked weights; the channels of group i go to
 * outs[i].
 *
 *   w_packed  (N, K/2) int8, the n_groups weights stacked along N in group order (row pitch
 *             w_ld), N = group_n[0] + ... + group_n[n_groups - 1]
 *   w_scale   (N,) stacked the same way; bias (N,) stacked, or NULL for no bias in any group
 *   n_groups  1 to 8
 *   group_n   host array: channels of each group (>= 0)
 *   outs      host array of device pointers: group i's output (M, group_n[i]) of out_dtype
 *   ldos      host array: group i's row pitch, >= group_n[i]
 * Every other argument, the workspace size (for the stacked N) and the errors are those of
 * ck_w4a4_linear, plus CK_ERR_INVALID_ARG for a bad n_groups, group_n or ldos, or a NULL
 * outs[i] for a non-empty group.  Group i's output equals ck_w4a4_linear's with group i's
 * weights, scales and bias alone, bit for bit: the same stage 1 and, per channel, the same
 * arithmetic.
 */
ck_status ck_w4a4_grouped_linear(const void* x, ck_dtype x_dtype, int64_t M, int64_t K,
                                 int64_t stride_m, int64_t stride_k, const void* R, int g,
                                 const float* a_scale, const int8_t* w_packed, int64_t w_ld,
                                 const void* w_scale, ck_dtype scale_dtype, const void* bias,
                                 int n_groups, const int64_t* group_n, void* const* outs,
                                 const int64_t* ldos, ck_dtype out_dtype, void* workspace,
                                 size_t workspace_bytes, int* dev_status, cudaStream_t stream);

/* Workspace ck_w4a4_linear needs for these sizes: the stage-1 codes and scales (also
 * used to re-pitch CK_I8 codes whose rows are not 16-byte aligned) and, when w_ld is
 * not a multiple of 16, a 16-byte-pitched copy of the packed weights.  Assumes a
 * 16-byte aligned w_packed.  Returns 0 for invalid sizes. */
size_t ck_w4a4_linear_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t w_ld);

/* Layout of the stage-1 result inside the workspace (see ck_w4a4_linear). */
int64_t ck_workspace_codes_pitch(int64_t K);
size_t ck_workspace_scales_offset(int64_t M, int64_t K);

/*
 * Weight unpack (PR #198: the W4 codes are unpacked to INT8; PR #201: only weights
 * are unpacked): packed (N, K/2) int8 with row pitch ld_packed bytes ->
 * out (N, K) int8 sign-extended codes in [-8, 7], row pitch ld_out bytes.
 * Bit-exact.  Errors: CK_ERR_INVALID_ARG (null pointers, N < 0, K <= 0 or odd,
 * ld_packed < K/2, ld_out < K), CK_ERR_CUDA.
 */
ck_status ck_unpack_w4(const int8_t* packed, int64_t N, int64_t K, int64_t ld_packed,
                       int8_t* out, int64_t ld_out, cudaStream_t stream);

/*
 * The whole linear without a caller-provided workspace, for callers that cannot allocate
 * device memory (a plugin inside a host framework that owns all device memory and offers no
 * allocation hook, or a latency-critical loop that must not call cudaMalloc, which may
 * synchronise the device).  This entry point has no counterpart on the pages: it is a
 * deployment convenience around ck_w4a4_linear, with the same arguments, results and errors
 * except workspace / workspace_bytes.
 *
 * Scratch memory comes from an array compiled into the library: 32 MiB of device memory
 * that every GPU which loads the library holds until the process exits.  The call allocates
 * nothing (no cudaMalloc, cudaFree or allocating library routine).
 *   - Limit: calls whose scratch need exceeds 32 MiB return CK_ERR_WORKSPACE and launch
 *     nothing (e.g. 8192 x 3840 activations fit, 8192 x 10240 do not).  The need is the
 *     scratch ck_w4a4_linear uses for this call: the stage-1 codes and scales of
 *     floating-point input (ck_workspace_scales_offset(M, K) + 4 M, rounded up to 256), the
 *     same for int8 codes whose rows are not 16-byte aligned (0 for aligned ones), plus a
 *     16-byte-pitched weight copy when w_packed is not 16-byte aligned and pitched.
 *   - The first call on each device looks up the array's device address (with that device
 *     current) and caches it; after a device reset, which ends the context and may move the
 *     array, the next call looks it up again.  Make the first call on a device before any
 *     stream capture.
 *   - Every pointer must refer to memory of the calling thread's current device (the array
 *     used is the current device's).
 *   - Every call on a device shares the one array and nothing in it needs clearing between
 *     calls; calls whose GPU work overlaps in time (different streams) race on it.
 */
ck_status ck_w4a4_linear_noalloc(const void* x, ck_dtype x_dtype, int64_t M, int64_t K,
                                 int64_t stride_m, int64_t stride_k, const void* R, int g,
                                 const float* a_scale, const int8_t* w_packed, int64_t N,
                                 int64_t w_ld, const void* w_scale, ck_dtype scale_dtype,
                                 const void* bias, void* out, ck_dtype out_dtype, int64_t ldo,
                                 int* dev_status, cudaStream_t stream);

/*
 * The W8A8 variant (comfy-kitchen PR #155 "Add fused RotateQuant backend": the fused rotation
 * and quantization emitting INT8 codes with per-row scales; PR #198 "Consolidate INT8,
 * RotateQuant, RoPE and ConvRot W4A4 backends": the INT8 linear).  The same rotation, the INT8
 * grid instead of INT4:
 *   s[m] = max(fp32(max_k |y[m, k]|) / 127, FLT_MIN)   (or the caller's scale, clamped the same way)
 *   q[m, k] = clamp(round_half_even(y[m, k] / s[m]), -128, 127)
 * ck_rotate_quant_int8 takes and returns what ck_rotate_quant does.
 */
ck_status ck_rotate_quant_int8(const void* x, ck_dtype x_dtype, int64_t M, int64_t K,
                               int64_t stride_m, int64_t stride_k, const void* R, int g,
                               const float* scale_in, int8_t* codes, int64_t ldq, float* scales,
                               int* dev_status, cudaStream_t stream);

/*
 * The W8A8 linear: ck_rotate_quant_int8 (or INT8 codes given with x_dtype == CK_I8 and their
 * row scales in a_scale), then acc[m, n] = sum_k q[m, k] * w[n, k] in exact INT32 over INT8
 * weights w (N, K) with row pitch w_ld >= K bytes (no unpack), and ck_w4a4_linear's epilogue.
 * Every argument but w / w_ld means what it does for ck_w4a4_linear; the workspace is
 * ck_w8a8_linear_workspace_bytes(M, N, K, w_ld).  CK_ERR_OVERFLOW when 128 * 128 * K > 2^31 - 1
 * (K > 131071), the bound of |acc| on this grid.
 */
ck_status ck_w8a8_linear(const void* x, ck_dtype x_dtype, int64_t M, int64_t K,
                         int64_t stride_m, int64_t stride_k, const void* R, int g,
                         const float* a_scale, const int8_t* w, int64_t N, int64_t w_ld,
                         const void* w_scale, ck_dtype scale_dtype, const void* bias,
                         void* out, ck_dtype out_dtype, int64_t ldo,
                         void* workspace, size_t workspace_bytes, int* dev_status,
                         cudaStream_t stream);
size_t ck_w8a8_linear_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t w_ld);

/*
 * The public packed-activation quantizer (comfy-kitchen PR #201 "Avoid activation pack/unpack
 * in ConvRot W4A4", "Summary": the W4A4 path no longer packs activations, while the public
 * packed quantizer keeps its signature, scales and stochastic rounding; "Correctness and
 * tests": odd widths are rejected).  The rotation and row scale of ck_rotate_quant, then with
 * t = y / s (the IEEE fp32 quotient):
 *   stochastic == 0:  q = clamp(round_half_even(t), -8, 7)
 *   stochastic == 1:  q = clamp(floor(t + u), -8, 7) with the sum rounded to fp32 and
 *                     u = (r >> 8) * 2^-24, r = word 0 of Philox4x32-10 (Salmon et al., SC 2011)
 *                     of counter {e, e >> 32, offset, offset >> 32} under key {seed, seed >> 32},
 *                     e = m * K + k the element's index: the same (seed, offset) gives the same
 *                     codes, and E[q] = t inside the grid.
 * (NaN quotients give 0.)  The pages give no random-number specification; this one is the
 * library's.
 *   packed   (M, K / 2) bytes, row pitch ld_packed >= K / 2: byte k / 2 holds code k (even k) in
 *            its low nibble and code k + 1 in its high nibble.
 *   scales   (M,) fp32, as ck_rotate_quant.
 * Errors: CK_ERR_INVALID_ARG (as ck_rotate_quant, plus odd K, ld_packed < K / 2, stochastic
 * not 0 or 1), CK_ERR_UNSUPPORTED (rows whose fp32 copy and R exceed shared memory, about
 * 56,000 channels), CK_ERR_CUDA.
 */
ck_status ck_rotate_quant_packed(const void* x, ck_dtype x_dtype, int64_t M, int64_t K,
                                 int64_t stride_m, int64_t stride_k, const void* R, int g,
                                 const float* scale_in, int stochastic, uint64_t seed,
                                 uint64_t offset, uint8_t* packed, int64_t ld_packed,
                                 float* scales, cudaStream_t stream);

/* Static description of a status code (never NULL). */
const char* ck_status_string(ck_status status);

#ifdef __cplusplus
}
#endif

#endif /* CK_H */
