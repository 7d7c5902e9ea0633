/*
 * ck_oracle.h -- plain single-threaded CPU oracle of the ConvRot W4A4 linear.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code, header,
 * table or helper with the CUDA path, and the CUDA path never calls it.
 *
 * Sources (comfy-kitchen pages):
 *   - PR #198 "Consolidate INT8, RotateQuant, RoPE and ConvRot W4A4 backends",
 *     section "W4A4 correctness and performance scope": rotation keeps the
 *     FP32/FP16/BF16 input dtype; the reference signed-INT4 quantizer; codes
 *     unpacked to INT8 and accumulated in INT32 at unit scale; cast, then
 *     activation scale, then weight scale, then bias; INT32 overflow guard.
 *   - PR #201 "Avoid activation pack/unpack in ConvRot W4A4", section "Summary":
 *     activation codes stay in INT8 storage, only weights are unpacked.
 *   - PR #155 "Add fused RotateQuant backend", backend list and review comment:
 *     deterministic rounding, caller-provided zero scales replaced by the eager
 *     path's finite minimum before division.
 *   - comfy_kitchen/tensor/svdquant_w4a4.py, module docstring: (N, K // 2) int8
 *     packed W4 weight layout.
 *
 * dtype codes: 0 = fp32, 1 = fp16, 2 = bf16 (16-bit values are passed as raw bits).
 * Every function returns 0 on success and a negative number on a bad argument or
 * an accumulator that does not fit in int32.
 */
#ifndef CK_ORACLE_H
#define CK_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
/* ---------------------------------------------------------------- W8A8 variant
 * The same rotation with INT8 codes (PR #155 "Add fused RotateQuant backend": the fused
 * rotate-and-quantize operator emits INT8 codes with per-row scales; PR #198: the INT8
 * linear): s = max(fp32(amax|y|) / 127, FLT_MIN) per row (or the caller's scale, clamped the
 * same way), q = clamp(round_half_even(fp32(y) / s), -128, 127). */
int ck_oracle_quantize_int8(const double* y, int64_t nrows, int64_t K, const float* scale_in,
                            int8_t* codes, float* scales);

int ck_oracle_rotate_quant_int8(const void* x, int dtype, int64_t M, int64_t K,
                                int64_t stride_m, int64_t stride_k, const void* R, int g,
                                const float* scale_in, const int64_t* rows, int64_t nrows,
                                int8_t* codes, float* scales);

/* W8A8 linear on the listed rows / cols: INT8 stage 1, INT8 weights w (N, K) with row pitch
 * w_ld, exact INT32 GEMM, the same epilogue. */
int ck_oracle_linear_w8a8(const void* x, int dtype, int64_t M, int64_t K, int64_t stride_m,
                          int64_t stride_k, const void* R, int g, const int8_t* w, int64_t N,
                          int64_t w_ld, const void* w_scale, const void* bias, int scale_dtype,
                          int out_dtype, const int64_t* rows, int64_t nrows, const int64_t* cols,
                          int64_t ncols, void* out, int8_t* codes, float* scales);

/* ---------------------------------------------------------------- packed quantizer
 * Philox4x32-10 (J. K. Salmon, M. A. Moraes, R. O. Dror, D. E. Shaw, "Parallel random
 * numbers: as easy as 1, 2, 3", SC 2011): out = bijection of the 128-bit counter ctr under
 * the 64-bit key, ten rounds. */
int ck_oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]);

/* The public signed-INT4 quantizer with nibble-packed output (PR #201 "Summary": the public
 * packed quantizer keeps its signature, scales and stochastic rounding).  Scales as in
 * ck_oracle_quantize.  t = fp32(y) / s (IEEE), then
 *   rounding 0: q = clamp(round_half_even(t), -8, 7)
 *   rounding 1: q = clamp(floor(fp32(t + u)), -8, 7), u = (r >> 8) * 2^-24 with r word 0 of
 *               Philox4x32-10(counter {e, e >> 32, offset, offset >> 32}, key {seed, seed >> 32})
 *               and e = rows[i] * K + k, the element's index in the (M, K) tensor
 * (a NaN t gives 0).  packed (nrows, K / 2): byte k / 2 holds code k (even) in its low nibble
 * and code k + 1 in its high nibble.  K must be even. */
int ck_oracle_quantize_packed(const double* y, int64_t nrows, int64_t K, const float* scale_in,
                              int rounding, uint64_t seed, uint64_t offset, const int64_t* rows,
                              uint8_t* packed, float* scales);

#endif

/* Round each v[i] to the nearest value of the dtype (ties to even, IEEE overflow to inf). */
int ck_oracle_round(double* v, int64_t n, int dtype);

/* Decode n dtype elements (raw storage) to double. */
int ck_oracle_decode(const void* src, int dtype, int64_t n, double* dst);

/* Encode n doubles that are exact dtype values to raw storage (fp32 or 16-bit bits). */
int ck_oracle_encode(const double* src, int dtype, int64_t n, void* dst);

/* Group-wise rotation of the rows listed in rows[0..nrows):
 * y[r, j*g + c] = round_dtype( sum_i x[rows[r], j*g + i] * R[i, c] ), summed in double.
 * x is read through (stride_m, stride_k) in elements; R is g*g row-major in the same dtype.
 * y is (nrows, K) double. */
int ck_oracle_rotate(const void* x, int dtype, int64_t M, int64_t K, int64_t stride_m,
                     int64_t stride_k, const void* R, int g, const int64_t* rows, int64_t nrows,
                     double* y);

/* Row-wise signed-INT4 quantization of already rotated rows y (nrows, K) (values of the dtype).
 * scale_in == NULL: s = max(fp32(amax|y|) / 7, FLT_MIN) per row (a NaN in the row gives NaN);
 * else s = max(*scale_in, FLT_MIN) for every row.
 * q = clamp(round_half_even(fp32(y) / s), -8, 7) (a NaN quotient gives 0).  codes (nrows, K). */
int ck_oracle_quantize(const double* y, int64_t nrows, int64_t K, const float* scale_in,
                       int8_t* codes, float* scales);

/* Stage 1 for the listed rows: rotate then quantize. codes (nrows, K), scales (nrows). */
int ck_oracle_rotate_quant(const void* x, int dtype, int64_t M, int64_t K, int64_t stride_m,
                           int64_t stride_k, const void* R, int g, const float* scale_in,
                           const int64_t* rows, int64_t nrows, int8_t* codes, float* scales);

/* Pack (N, K) codes in [-8, 7] to (N, K/2) bytes, even k in the low nibble. */
int ck_oracle_pack_w4(const int8_t* w, int64_t N, int64_t K, int8_t* packed);

/* Unpack (N, K/2) bytes (row pitch ld bytes) to (N, K) sign-extended codes. */
int ck_oracle_unpack_w4(const int8_t* packed, int64_t N, int64_t K, int64_t ld, int8_t* w);

/* acc[i, j] = sum_k q[i, k] * w[j, k] in int64; fails (-2) if any |acc| exceeds int32.
 * q is (Mq, K), w is (Nw, K) unpacked codes. */
int ck_oracle_gemm_s32(const int8_t* q, int64_t Mq, const int8_t* w, int64_t Nw, int64_t K,
                       int32_t* acc);

/* out[i, j] = cvt( ((fp32(acc[i, j]) * a_scale[i]) * fp32(w_scale[j])) + fp32(bias[j]) ),
 * each step one IEEE fp32 operation, one final rounding to out_dtype.
 * w_scale and bias are in scale_dtype; bias may be NULL.  out holds out_dtype storage. */
int ck_oracle_epilogue(const int32_t* acc, int64_t Mq, int64_t Nw, const float* a_scale,
                       const void* w_scale, const void* bias, int scale_dtype, void* out,
                       int out_dtype);

/* The whole linear on the listed rows and columns (cols index output channels):
 * stage 1 on rows, unpack of the listed weight rows, GEMM, epilogue.
 * out (nrows, ncols) in out_dtype storage; codes (nrows, K) and scales (nrows) may be NULL. */
int ck_oracle_linear(const void* x, int dtype, int64_t M, int64_t K, int64_t stride_m,
                     int64_t stride_k, const void* R, int g, const int8_t* w_packed, int64_t N,
                     int64_t w_ld, const void* w_scale, const void* bias, int scale_dtype,
                     int out_dtype, const int64_t* rows, int64_t nrows, const int64_t* cols,
                     int64_t ncols, void* out, int8_t* codes, float* scales);

#ifdef __cplusplus
}
/* ---------------------------------------------------------------- W8A8 variant
 * The same rotation with INT8 codes (PR #155 "Add fused RotateQuant backend": the fused
 * rotate-and-quantize operator emits INT8 codes with per-row scales; PR #198: the INT8
 * linear): s = max(fp32(amax|y|) / 127, FLT_MIN) per row (or the caller's scale, clamped the
 * same way), q = clamp(round_half_even(fp32(y) / s), -128, 127). */
int ck_oracle_quantize_int8(const double* y, int64_t nrows, int64_t K, const float* scale_in,
                            int8_t* codes, float* scales);

int ck_oracle_rotate_quant_int8(const void* x, int dtype, int64_t M, int64_t K,
                                int64_t stride_m, int64_t stride_k, const void* R, int g,
                                const float* scale_in, const int64_t* rows, int64_t nrows,
                                int8_t* codes, float* scales);

/* W8A8 linear on the listed rows / cols: INT8 stage 1, INT8 weights w (N, K) with row pitch
 * w_ld, exact INT32 GEMM, the same epilogue. */
int ck_oracle_linear_w8a8(const void* x, int dtype, int64_t M, int64_t K, int64_t stride_m,
                          int64_t stride_k, const void* R, int g, const int8_t* w, int64_t N,
                          int64_t w_ld, const void* w_scale, const void* bias, int scale_dtype,
                          int out_dtype, const int64_t* rows, int64_t nrows, const int64_t* cols,
                          int64_t ncols, void* out, int8_t* codes, float* scales);

/* ---------------------------------------------------------------- packed quantizer
 * Philox4x32-10 (J. K. Salmon, M. A. Moraes, R. O. Dror, D. E. Shaw, "Parallel random
 * numbers: as easy as 1, 2, 3", SC 2011): out = bijection of the 128-bit counter ctr under
 * the 64-bit key, ten rounds. */
int ck_oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]);

/* The public signed-INT4 quantizer with nibble-packed output (PR #201 "Summary": the public
 * packed quantizer keeps its signature, scales and stochastic rounding).  Scales as in
 * ck_oracle_quantize.  t = fp32(y) / s (IEEE), then
 *   rounding 0: q = clamp(round_half_even(t), -8, 7)
 *   rounding 1: q = clamp(floor(fp32(t + u)), -8, 7), u = (r >> 8) * 2^-24 with r word 0 of
 *               Philox4x32-10(counter {e, e >> 32, offset, offset >> 32}, key {seed, seed >> 32})
 *               and e = rows[i] * K + k, the element's index in the (M, K) tensor
 * (a NaN t gives 0).  packed (nrows, K / 2): byte k / 2 holds code k (even) in its low nibble
 * and code k + 1 in its high nibble.  K must be even. */
int ck_oracle_quantize_packed(const double* y, int64_t nrows, int64_t K, const float* scale_in,
                              int rounding, uint64_t seed, uint64_t offset, const int64_t* rows,
                              uint8_t* packed, float* scales);

#endif
/* ---------------------------------------------------------------- W8A8 variant
 * The same rotation with INT8 codes (PR #155 "Add fused RotateQuant backend": the fused
 * rotate-and-quantize operator emits INT8 codes with per-row scales; PR #198: the INT8
 * linear): s = max(fp32(amax|y|) / 127, FLT_MIN) per row (or the caller's scale, clamped the
 * same way), q = clamp(round_half_even(fp32(y) / s), -128, 127). */
int ck_oracle_quantize_int8(const double* y, int64_t nrows, int64_t K, const float* scale_in,
                            int8_t* codes, float* scales);

int ck_oracle_rotate_quant_int8(const void* x, int dtype, int64_t M, int64_t K,
                                int64_t stride_m, int64_t stride_k, const void* R, int g,
                                const float* scale_in, const int64_t* rows, int64_t nrows,
                                int8_t* codes, float* scales);

/* W8A8 linear on the listed rows / cols: INT8 stage 1, INT8 weights w (N, K) with row pitch
 * w_ld, exact INT32 GEMM, the same epilogue. */
int ck_oracle_linear_w8a8(const void* x, int dtype, int64_t M, int64_t K, int64_t stride_m,
                          int64_t stride_k, const void* R, int g, const int8_t* w, int64_t N,
                          int64_t w_ld, const void* w_scale, const void* bias, int scale_dtype,
                          int out_dtype, const int64_t* rows, int64_t nrows, const int64_t* cols,
                          int64_t ncols, void* out, int8_t* codes, float* scales);

/* ---------------------------------------------------------------- packed quantizer
 * Philox4x32-10 (J. K. Salmon, M. A. Moraes, R. O. Dror, D. E. Shaw, "Parallel random
 * numbers: as easy as 1, 2, 3", SC 2011): out = bijection of the 128-bit counter ctr under
 * the 64-bit key, ten rounds. */
int ck_oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]);

/* The public signed-INT4 quantizer with nibble-packed output (PR #201 "Summary": the public
 * packed quantizer keeps its signature, scales and stochastic rounding).  Scales as in
 * ck_oracle_quantize.  t = fp32(y) / s (IEEE), then
 *   rounding 0: q = clamp(round_half_even(t), -8, 7)
 *   rounding 1: q = clamp(floor(fp32(t + u)), -8, 7), u = (r >> 8) * 2^-24 with r word 0 of
 *               Philox4x32-10(counter {e, e >> 32, offset, offset >> 32}, key {seed, seed >> 32})
 *               and e = rows[i] * K + k, the element's index in the (M, K) tensor
 * (a NaN t gives 0).  packed (nrows, K / 2): byte k / 2 holds code k (even) in its low nibble
 * and code k + 1 in its high nibble.  K must be even. */
int ck_oracle_quantize_packed(const double* y, int64_t nrows, int64_t K, const float* scale_in,
                              int rounding, uint64_t seed, uint64_t offset, const int64_t* rows,
                              uint8_t* packed, float* scales);

#endif
