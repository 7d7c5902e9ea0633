/*
 * ck_oracle.c -- plain single-threaded CPU oracle of the ConvRot W4A4 linear.
 *
 * TEST INFRASTRUCTURE ONLY: loaded by the tests, the package smoke check and the
 * benchmark's CPU-baseline leg, never by the product path.  Shares no code with
 * the CUDA library.  Build with -ffp-contract=off and without fast-math so every
 * fp32 step below is one IEEE operation with round-to-nearest-even.
 *
 * The computation, as the comfy-kitchen pages state it (see ck_oracle.h for the
 * page list):
 *   1. rotate each activation row group-wise along K with a g x g orthogonal
 *      matrix, in the input dtype (PR #198, "W4A4 correctness and performance scope");
 *   2. quantize each row to signed INT4 codes with one positive scale per row,
 *      deterministic rounding, codes kept in INT8 storage (PR #198 same section;
 *      PR #201 "Summary"; PR #155 backend list);
 *   3. unpack the (N, K/2) W4 weight bytes to INT8 (PR #198; svdquant_w4a4.py
 *      module docstring for the (N, K // 2) layout);
 *   4. exact integer contraction with INT32 accumulation at unit scale, guarded
 *      against INT32 overflow (PR #198);
 *   5. cast to fp32, times activation scale, times weight scale, plus bias, in
 *      that order (PR #198).
 *
 * Readings where the pages are silent (each one is listed with its reason in the
 * design notes of the repository):
 *   - rotation is x_group @ R (row vector times R), summed exactly in double and
 *     rounded once to the dtype;
 *   - the quantizer's grid is the symmetric signed-INT4 one: s = amax / 7 in fp32,
 *     q = clamp(round_half_even(y / s), -8, 7);
 *   - the "finite minimum" that replaces a zero scale is FLT_MIN (2^-126), applied
 *     as a lower clamp; NaN propagates;
 *   - the low nibble of a weight byte holds the even k;
 *   - a NaN quotient y / s gives code 0.
 */
#include "ck_oracle.h"

#include <float.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>

enum { OR_F32 = 0, OR_F16 = 1, OR_BF16 = 2 };

/* ---------------------------------------------------------------- dtype helpers */

/* binary16: 10 stored mantissa bits, normal exponents from -14, max finite 65504. */
static double dec_f16(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 31;
    int m = h & 1023;
    double v;
    if (e == 0) {
        v = ldexp((double)m, -24);
    } else if (e == 31) {
        v = m ? NAN : INFINITY;
    } else {
        v = ldexp((double)(1024 + m), e - 25);
    }
    return sign ? -v : v;
}

/* bfloat16 is the high half of an IEEE binary32. */
static double dec_bf16(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static double dec_f32(const void* p) {
    float f;
    memcpy(&f, p, 4);
    return (double)f;
}

static double load_elem(const void* base, int dtype, int64_t idx) {
    if (dtype == OR_F32) return dec_f32((const char*)base + 4 * idx);
    uint16_t h;
    memcpy(&h, (const char*)base + 2 * idx, 2);
    return dtype == OR_F16 ? dec_f16(h) : dec_bf16(h);
}

/* Round v to the nearest number with `mant` stored mantissa bits and minimum normal
 * exponent `emin` (subnormals below it), ties to even; beyond `maxv` it becomes inf. */
static double round_format(double v, int mant, int emin, double maxv) {
    if (isnan(v) || isinf(v) || v == 0.0) return v;
    int e;
    frexp(fabs(v), &e);          /* |v| = f * 2^e, f in [0.5, 1): leading bit at 2^(e-1) */
    int lead = e - 1;
    if (lead < emin) lead = emin;
    double quantum = ldexp(1.0, lead - mant);
    double r = nearbyint(v / quantum) * quantum;   /* default rounding mode: ties to even */
    if (fabs(r) > maxv) r = copysign(INFINITY, v);
    return r;
}

static double round_dtype(double v, int dtype) {
    switch (dtype) {
        case OR_F32: return round_format(v, 23, -126, (double)FLT_MAX);
        case OR_F16: return round_format(v, 10, -14, 65504.0);
        default:     return round_format(v, 7, -126, ldexp(255.0, 120)); /* (2 - 2^-7) * 2^127 */
    }
}

static uint16_t enc_f16(double r) {
    uint16_t sign = signbit(r) ? 0x8000 : 0;
    double a = fabs(r);
    if (isnan(r)) return 0x7E00;
    if (isinf(r)) return sign | 0x7C00;
    if (a == 0.0) return sign;
    if (a < ldexp(1.0, -14)) return sign | (uint16_t)(a / ldexp(1.0, -24));
    int e;
    double f = frexp(a, &e);     /* a = f * 2^e, leading bit 2^(e-1) */
    int be = e - 1 + 15;
    uint16_t m = (uint16_t)((f * 2.0 - 1.0) * 1024.0);
    return sign | (uint16_t)(be << 10) | m;
}

static void store_elem(void* base, int dtype, int64_t idx, double r) {
    if (dtype == OR_F32) {
        float f = (float)r;
        memcpy((char*)base + 4 * idx, &f, 4);
    } else if (dtype == OR_F16) {
        uint16_t h = enc_f16(r);
        memcpy((char*)base + 2 * idx, &h, 2);
    } else {
        float f = (float)r;      /* r is a bf16 value: exact in fp32, low 16 bits zero */
        uint32_t u;
        memcpy(&u, &f, 4);
        uint16_t h = (uint16_t)(u >> 16);
        if (isnan(r)) h = 0x7FC0;
        memcpy((char*)base + 2 * idx, &h, 2);
    }
}

static int bad_dtype(int d) { return d != OR_F32 && d != OR_F16 && d != OR_BF16; }

int ck_oracle_round(double* v, int64_t n, int dtype) {
    if (bad_dtype(dtype) || n < 0 || (n && !v)) return -1;
    for (int64_t i = 0; i < n; ++i) v[i] = round_dtype(v[i], dtype);
    return 0;
}

int ck_oracle_decode(const void* src, int dtype, int64_t n, double* dst) {
    if (bad_dtype(dtype) || n < 0) return -1;
    for (int64_t i = 0; i < n; ++i) dst[i] = load_elem(src, dtype, i);
    return 0;
}

int ck_oracle_encode(const double* src, int dtype, int64_t n, void* dst) {
    if (bad_dtype(dtype) || n < 0) return -1;
    for (int64_t i = 0; i < n; ++i) store_elem(dst, dtype, i, src[i]);
    return 0;
}

/* ---------------------------------------------------------------- stage 1 */

/* Rotation in the input dtype (PR #198, "W4A4 correctness and performance scope":
 * the FP32/FP16/BF16 activation dtype is kept during rotation; PR #155: the rotation
 * matrix may be asymmetric).  Each group of g consecutive channels of a row is
 * multiplied on the right by R; the exact sum is formed in double and rounded once. */
int ck_oracle_rotate(const void* x, int dtype, int64_t M, int64_t K, int64_t stride_m,
                     int64_t stride_k, const void* R, int g, const int64_t* rows, int64_t nrows,
                     double* y) {
    if (bad_dtype(dtype) || M < 0 || K <= 0 || g <= 0 || K % g != 0 || nrows < 0) return -1;
    double* rd = (double*)malloc(sizeof(double) * (size_t)g * (size_t)g);
    if (!rd) return -3;
    for (int64_t i = 0; i < (int64_t)g * g; ++i) rd[i] = load_elem(R, dtype, i);
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t m = rows[r];
        if (m < 0 || m >= M) { free(rd); return -1; }
        for (int64_t j = 0; j < K / g; ++j) {
            for (int c = 0; c < g; ++c) {
                double acc = 0.0;
                for (int i = 0; i < g; ++i) {
                    double xv = load_elem(x, dtype, m * stride_m + (j * g + i) * stride_k);
                    acc += xv * rd[(int64_t)i * g + c];
                }
                y[r * K + j * g + c] = round_dtype(acc, dtype);
            }
        }
    }
    free(rd);
    return 0;
}

/* Reference signed-INT4 row-wise quantizer (PR #198 "W4A4 correctness and performance
 * scope"; PR #155: deterministic rounding, positive scales, caller-provided zero scale
 * replaced by the eager path's finite minimum before division). */
int ck_oracle_quantize(const double* y, int64_t nrows, int64_t K, const float* scale_in,
                       int8_t* codes, float* scales) {
    if (nrows < 0 || K <= 0) return -1;
    for (int64_t r = 0; r < nrows; ++r) {
        const double* row = y + r * K;
        float s;
        if (scale_in) {
            s = *scale_in;
        } else {
            double amax = 0.0;
            int has_nan = 0;
            for (int64_t k = 0; k < K; ++k) {
                if (isnan(row[k])) has_nan = 1;
                else if (fabs(row[k]) > amax) amax = fabs(row[k]);
            }
            s = has_nan ? NAN : (float)amax / 7.0f;
        }
        if (s < FLT_MIN) s = FLT_MIN;      /* lower clamp; NaN compares false and stays */
        scales[r] = s;
        for (int64_t k = 0; k < K; ++k) {
            float t = (float)row[k] / s;
            int8_t q;
            if (isnan(t)) {
                q = 0;
            } else {
                t = rintf(t);                   /* ties to even */
                if (t > 7.0f) t = 7.0f;
                if (t < -8.0f) t = -8.0f;
                q = (int8_t)t;
            }
            codes[r * K + k] = q;
        }
    }
    return 0;
}

int ck_oracle_rotate_quant(const void* x, int dtype, int64_t M, int64_t K, int64_t stride_m,
                           int64_t stride_k, const void* R, int g, const float* scale_in,
                           const int64_t* rows, int64_t nrows, int8_t* codes, float* scales) {
    if (nrows < 0 || K <= 0) return -1;
    if (nrows == 0) return 0;
    double* y = (double*)malloc(sizeof(double) * (size_t)nrows * (size_t)K);
    if (!y) return -3;
    int rc = ck_oracle_rotate(x, dtype, M, K, stride_m, stride_k, R, g, rows, nrows, y);
    if (rc == 0) rc = ck_oracle_quantize(y, nrows, K, scale_in, codes, scales);
    free(y);
    return rc;
}

/* ---------------------------------------------------------------- weights */

/* W4 packing: (N, K/2) bytes (svdquant_w4a4.py module docstring), the code of the even
 * k in the low nibble. */
int ck_oracle_pack_w4(const int8_t* w, int64_t N, int64_t K, int8_t* packed) {
    if (N < 0 || K <= 0 || K % 2) return -1;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t i = 0; i < K / 2; ++i) {
            int lo = w[n * K + 2 * i] & 0xF;
            int hi = w[n * K + 2 * i + 1] & 0xF;
            packed[n * (K / 2) + i] = (int8_t)(uint8_t)(lo | (hi << 4));
        }
    return 0;
}

/* Weight unpack to INT8 (PR #198: the same W4 codes are unpacked to INT8 before the
 * integer matmul; PR #201: only weights are unpacked).  Each nibble is a 4-bit two's
 * complement code. */
int ck_oracle_unpack_w4(const int8_t* packed, int64_t N, int64_t K, int64_t ld, int8_t* w) {
    if (N < 0 || K <= 0 || K % 2 || ld < K / 2) return -1;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t i = 0; i < K / 2; ++i) {
            int b = (uint8_t)packed[n * ld + i];
            int lo = b & 0xF, hi = (b >> 4) & 0xF;
            w[n * K + 2 * i] = (int8_t)(lo >= 8 ? lo - 16 : lo);
            w[n * K + 2 * i + 1] = (int8_t)(hi >= 8 ? hi - 16 : hi);
        }
    return 0;
}

/* ---------------------------------------------------------------- stage 2 */

/* Integer contraction at unit scale with INT32 accumulation (PR #198); the sum is formed
 * in int64 and must fit in int32 (the overflow guard). */
int ck_oracle_gemm_s32(const int8_t* q, int64_t Mq, const int8_t* w, int64_t Nw, int64_t K,
                       int32_t* acc) {
    if (Mq < 0 || Nw < 0 || K <= 0) return -1;
    for (int64_t i = 0; i < Mq; ++i)
        for (int64_t j = 0; j < Nw; ++j) {
            int64_t s = 0;
            for (int64_t k = 0; k < K; ++k) s += (int64_t)q[i * K + k] * (int64_t)w[j * K + k];
            if (s > INT32_MAX || s < INT32_MIN) return -2;
            acc[i * Nw + j] = (int32_t)s;
        }
    return 0;
}

/* Cast, activation scale, weight scale, bias, in that order (PR #198), each an fp32
 * operation; the result is rounded once to the output dtype. */
int ck_oracle_epilogue(const int32_t* acc, int64_t Mq, int64_t Nw, const float* a_scale,
                       const void* w_scale, const void* bias, int scale_dtype, void* out,
                       int out_dtype) {
    if (bad_dtype(scale_dtype) || bad_dtype(out_dtype) || Mq < 0 || Nw < 0) return -1;
    for (int64_t i = 0; i < Mq; ++i)
        for (int64_t j = 0; j < Nw; ++j) {
            float o = (float)acc[i * Nw + j];
            o = o * a_scale[i];
            o = o * (float)load_elem(w_scale, scale_dtype, j);
            if (bias) o = o + (float)load_elem(bias, scale_dtype, j);
            store_elem(out, out_dtype, i * Nw + j, round_dtype((double)o, out_dtype));
        }
    return 0;
}

int ck_oracle_linear(const void* x, int dtype, int64_t M, int64_t K, int64_t stride_m,
                     int64_t stride_k, const void* R, int g, const int8_t* w_packed, int64_t N,
                     int64_t w_ld, const void* w_scale, const void* bias, int scale_dtype,
                     int out_dtype, const int64_t* rows, int64_t nrows, const int64_t* cols,
                     int64_t ncols, void* out, int8_t* codes, float* scales) {
    if (nrows < 0 || ncols < 0 || K <= 0 || K % 2 || w_ld < K / 2) return -1;
    int rc = 0;
    int8_t* q = (int8_t*)malloc((size_t)(nrows ? nrows : 1) * (size_t)K);
    float* s = (float*)malloc(sizeof(float) * (size_t)(nrows ? nrows : 1));
    int8_t* wsel = (int8_t*)malloc((size_t)(ncols ? ncols : 1) * (size_t)K);
    int32_t* acc = (int32_t*)malloc(sizeof(int32_t) * (size_t)(nrows ? nrows : 1) *
                                    (size_t)(ncols ? ncols : 1));
    unsigned char* wsc = (unsigned char*)malloc(4 * (size_t)(ncols ? ncols : 1));
    unsigned char* bsel = (unsigned char*)malloc(4 * (size_t)(ncols ? ncols : 1));
    if (!q || !s || !wsel || !acc || !wsc || !bsel) { rc = -3; goto done; }
    rc = ck_oracle_rotate_quant(x, dtype, M, K, stride_m, stride_k, R, g, NULL, rows, nrows,
                                q, s);
    if (rc) goto done;
    int eb = scale_dtype == OR_F32 ? 4 : 2;
    for (int64_t c = 0; c < ncols; ++c) {
        int64_t n = cols[c];
        if (n < 0 || n >= N) { rc = -1; goto done; }
        rc = ck_oracle_unpack_w4(w_packed + n * w_ld, 1, K, w_ld, wsel + c * K);
        if (rc) goto done;
        memcpy(wsc + c * eb, (const char*)w_scale + n * eb, (size_t)eb);
        if (bias) memcpy(bsel + c * eb, (const char*)bias + n * eb, (size_t)eb);
    }
    rc = ck_oracle_gemm_s32(q, nrows, wsel, ncols, K, acc);
    if (rc) goto done;
    rc = ck_oracle_epilogue(acc, nrows, ncols, s, wsc, bias ? bsel : NULL, scale_dtype, out,
                            out_dtype);
    if (rc) goto done;
    if (codes) memcpy(codes, q, (size_t)nrows * (size_t)K);
    if (scales) memcpy(scales, s, sizeof(float) * (size_t)nrows);
done:
    free(q); free(s); free(wsel); free(acc); free(wsc); free(bsel);
    return rc;
}

/* ---------------------------------------------------------------- W8A8 variant */

/* INT8 row-wise quantizer: the same steps as ck_oracle_quantize with the INT8 grid, qmax 127
 * (PR #155, fused RotateQuant emitting INT8 codes). */
int ck_oracle_quantize_int8(const double* y, int64_t nrows, int64_t K, const float* scale_in,
                            int8_t* codes, float* scales) {
    if (nrows < 0 || K <= 0) return -1;
    for (int64_t r = 0; r < nrows; ++r) {
        const double* row = y + r * K;
        float s;
        if (scale_in) {
            s = *scale_in;
        } else {
            double amax = 0.0;
            int has_nan = 0;
            for (int64_t k = 0; k < K; ++k) {
                if (isnan(row[k])) has_nan = 1;
                else if (fabs(row[k]) > amax) amax = fabs(row[k]);
            }
            s = has_nan ? NAN : (float)amax / 127.0f;
        }
        if (s < FLT_MIN) s = FLT_MIN;
        scales[r] = s;
        for (int64_t k = 0; k < K; ++k) {
            float t = (float)row[k] / s;
            int8_t q;
            if (isnan(t)) {
                q = 0;
            } else {
                t = rintf(t);
                if (t > 127.0f) t = 127.0f;
                if (t < -128.0f) t = -128.0f;
                q = (int8_t)t;
            }
            codes[r * K + k] = q;
        }
    }
    return 0;
}

int ck_oracle_rotate_quant_int8(const void* x, int dtype, int64_t M, int64_t K,
                                int64_t stride_m, int64_t stride_k, const void* R, int g,
                                const float* scale_in, const int64_t* rows, int64_t nrows,
                                int8_t* codes, float* scales) {
    if (nrows < 0 || K <= 0) return -1;
    if (nrows == 0) return 0;
    double* y = (double*)malloc(sizeof(double) * (size_t)nrows * (size_t)K);
    if (!y) return -3;
    int rc = ck_oracle_rotate(x, dtype, M, K, stride_m, stride_k, R, g, rows, nrows, y);
    if (rc == 0) rc = ck_oracle_quantize_int8(y, nrows, K, scale_in, codes, scales);
    free(y);
    return rc;
}

int ck_oracle_linear_w8a8(const void* x, int dtype, int64_t M, int64_t K, int64_t stride_m,
                          int64_t stride_k, const void* R, int g, const int8_t* w, int64_t N,
                          int64_t w_ld, const void* w_scale, const void* bias, int scale_dtype,
                          int out_dtype, const int64_t* rows, int64_t nrows, const int64_t* cols,
                          int64_t ncols, void* out, int8_t* codes, float* scales) {
    if (nrows < 0 || ncols < 0 || K <= 0 || w_ld < K) return -1;
    int rc = 0;
    int8_t* q = (int8_t*)malloc((size_t)(nrows ? nrows : 1) * (size_t)K);
    float* s = (float*)malloc(sizeof(float) * (size_t)(nrows ? nrows : 1));
    int8_t* wsel = (int8_t*)malloc((size_t)(ncols ? ncols : 1) * (size_t)K);
    int32_t* acc = (int32_t*)malloc(sizeof(int32_t) * (size_t)(nrows ? nrows : 1) *
                                    (size_t)(ncols ? ncols : 1));
    unsigned char* wsc = (unsigned char*)malloc(4 * (size_t)(ncols ? ncols : 1));
    unsigned char* bsel = (unsigned char*)malloc(4 * (size_t)(ncols ? ncols : 1));
    if (!q || !s || !wsel || !acc || !wsc || !bsel) { rc = -3; goto done; }
    rc = ck_oracle_rotate_quant_int8(x, dtype, M, K, stride_m, stride_k, R, g, NULL, rows,
                                     nrows, q, s);
    if (rc) goto done;
    int eb = scale_dtype == OR_F32 ? 4 : 2;
    for (int64_t c = 0; c < ncols; ++c) {
        int64_t n = cols[c];
        if (n < 0 || n >= N) { rc = -1; goto done; }
        memcpy(wsel + c * K, w + n * w_ld, (size_t)K);
        memcpy(wsc + c * eb, (const char*)w_scale + n * eb, (size_t)eb);
        if (bias) memcpy(bsel + c * eb, (const char*)bias + n * eb, (size_t)eb);
    }
    rc = ck_oracle_gemm_s32(q, nrows, wsel, ncols, K, acc);
    if (rc) goto done;
    rc = ck_oracle_epilogue(acc, nrows, ncols, s, wsc, bias ? bsel : NULL, scale_dtype, out,
                            out_dtype);
    if (rc) goto done;
    if (codes) memcpy(codes, q, (size_t)nrows * (size_t)K);
    if (scales) memcpy(scales, s, sizeof(float) * (size_t)nrows);
done:
    free(q); free(s); free(wsel); free(acc); free(wsc); free(bsel);
    return rc;
}

/* ---------------------------------------------------------------- packed quantizer */

/* Philox4x32-10 as published (Salmon et al., SC 2011): each round multiplies two counter
 * words by the constants 0xD2511F53 and 0xCD9E8D57 into 64-bit products and mixes their high
 * halves with the other two words and the key; the key is bumped by the Weyl constants
 * 0x9E3779B9 and 0xBB67AE85 between rounds. */
int ck_oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        const uint64_t p0 = (uint64_t)0xD2511F53u * c0;
        const uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
        const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        const uint32_t n0 = hi1 ^ c1 ^ k0;
        const uint32_t n1 = lo1;
        const uint32_t n2 = hi0 ^ c3 ^ k1;
        const uint32_t n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
    return 0;
}

int ck_oracle_quantize_packed(const double* y, int64_t nrows, int64_t K, const float* scale_in,
                              int rounding, uint64_t seed, uint64_t offset, const int64_t* rows,
                              uint8_t* packed, float* scales) {
    if (nrows < 0 || K <= 0 || K % 2 || (rounding != 0 && rounding != 1) || !rows) return -1;
    int8_t* q = (int8_t*)malloc((size_t)(K ? K : 1));
    if (!q) return -3;
    const uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    for (int64_t r = 0; r < nrows; ++r) {
        const double* row = y + r * K;
        float s;
        if (scale_in) {
            s = *scale_in;
        } else {
            double amax = 0.0;
            int has_nan = 0;
            for (int64_t k = 0; k < K; ++k) {
                if (isnan(row[k])) has_nan = 1;
                else if (fabs(row[k]) > amax) amax = fabs(row[k]);
            }
            s = has_nan ? NAN : (float)amax / 7.0f;
        }
        if (s < FLT_MIN) s = FLT_MIN;
        scales[r] = s;
        for (int64_t k = 0; k < K; ++k) {
            float t = (float)row[k] / s;
            if (isnan(t)) {
                q[k] = 0;
                continue;
            }
            if (rounding == 0) {
                t = rintf(t);
            } else {
                const uint64_t e = (uint64_t)rows[r] * (uint64_t)K + (uint64_t)k;
                const uint32_t ctr[4] = {(uint32_t)e, (uint32_t)(e >> 32), (uint32_t)offset,
                                         (uint32_t)(offset >> 32)};
                uint32_t rnd[4];
                ck_oracle_philox4x32_10(ctr, key, rnd);
                const float u = (float)(rnd[0] >> 8) * 0x1p-24f;
                t = floorf(t + u);
            }
            if (t > 7.0f) t = 7.0f;
            if (t < -8.0f) t = -8.0f;
            q[k] = (int8_t)t;
        }
        for (int64_t i = 0; i < K / 2; ++i)
            packed[r * (K / 2) + i] =
                (uint8_t)(((uint8_t)q[2 * i] & 0xF) | (((uint8_t)q[2 * i + 1] & 0xF) << 4));
    }
    free(q);
    return 0;
}
