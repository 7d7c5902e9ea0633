// ck_api.cu -- the extern "C" boundary declared in include/ck.h: argument validation,
// workspace layout, TMA descriptor encoding and dispatch to the kernels.
#include <cuda.h>
#include <cuda_runtime_api.h>
#include <stdint.h>

#include <mutex>

#include "ck.h"
#include "ck_internal.h"

namespace ck {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

ck_status encode_tma(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base,
                     const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                     CUtensorMapSwizzle swizzle) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return CK_ERR_CUDA;
    cuuint64_t d[5], s[4];
    cuuint32_t b[5], e[5];
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        b[i] = box[i];
        e[i] = 1;
        if (i + 1 < rank) s[i] = strides_bytes[i];
    }
    CUresult r = fn(map, dtype, (cuuint32_t)rank, const_cast<void*>(base), d, s, b, e,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? CK_OK : CK_ERR_CUDA;
}

int num_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        return 148;
    return n;
}

static bool float_dtype(ck_dtype d) { return d == CK_F32 || d == CK_F16 || d == CK_BF16; }
static bool group_ok(int g) { return g == 16 || g == 64 || g == 256; }
static int64_t round_up(int64_t v, int64_t a) { return (v + a - 1) / a * a; }

// The largest K for which |acc| <= 8 * 8 * K fits in int32 (INT4 codes), and the same for
// INT8 codes and weights (|acc| <= 128 * 128 * K).
static constexpr int64_t kMaxK = 2147483647LL / 64;
static constexpr int64_t kMaxK8 = 2147483647LL / (128 * 128);

size_t linear_scratch_need(const void* x, ck_dtype x_dtype, int64_t M, int64_t K,
                           int64_t stride_m, const int8_t* w_packed, int64_t N, int64_t w_ld,
                           bool w8) {
    const bool codes_in = x_dtype == CK_I8;
    const bool codes_aligned = codes_in && aligned(x, 16) && stride_m % 16 == 0;
    const bool w_aligned = aligned(w_packed, 16) && w_ld % 16 == 0;
    const int64_t P = K <= 0 ? 0 : round_up(K, 16);
    const size_t scales_off = (size_t)round_up(M * P, 256);
    const size_t wcopy_off = scales_off + (size_t)round_up(4 * M, 256);
    size_t need = 0;
    if (!codes_in || !codes_aligned) need = wcopy_off;
    if (!w_aligned) need = wcopy_off + (size_t)round_up(N * round_up(w8 ? K : K / 2, 16), 256);
    return need;
}

}  // namespace ck

using namespace ck;

extern "C" {

const char* ck_status_string(ck_status s) {
    switch (s) {
        case CK_OK: return "ok";
        case CK_ERR_INVALID_ARG: return "invalid argument";
        case CK_ERR_UNSUPPORTED: return "unsupported configuration";
        case CK_ERR_OVERFLOW: return "64*K exceeds INT32_MAX: INT32 accumulator could overflow";
        case CK_ERR_WORKSPACE: return "workspace missing or too small";
        case CK_ERR_CUDA: return "CUDA error";
        case CK_ERR_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

int64_t ck_workspace_codes_pitch(int64_t K) { return K <= 0 ? 0 : round_up(K, 16); }

size_t ck_workspace_scales_offset(int64_t M, int64_t K) {
    if (M < 0 || K <= 0) return 0;
    return (size_t)round_up(M * ck_workspace_codes_pitch(K), 256);
}

size_t ck_w8a8_linear_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t w_ld) {
    if (M < 0 || N < 0 || K <= 0 || K % 2 != 0 || w_ld < K) return 0;
    size_t bytes = ck_workspace_scales_offset(M, K) + (size_t)round_up(4 * M, 256);
    if (w_ld % 16 != 0) bytes += (size_t)round_up(N * round_up(K, 16), 256);
    return bytes;
}

size_t ck_w4a4_linear_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t w_ld) {
    if (M < 0 || N < 0 || K <= 0 || K % 2 != 0 || w_ld < K / 2) return 0;
    size_t bytes = ck_workspace_scales_offset(M, K) + (size_t)round_up(4 * M, 256);
    if (w_ld % 16 != 0) bytes += (size_t)round_up(N * round_up(K / 2, 16), 256);
    return bytes;
}

static ck_status rotate_quant_checked(const void* x, ck_dtype x_dtype, int64_t M, int64_t K,
                                      int64_t stride_m, int64_t stride_k, const void* R, int g,
                                      const float* scale_in, int8_t* codes, int64_t ldq,
                                      float* scales, int qmax, int* dev_status,
                                      cudaStream_t stream) {
    if (!float_dtype(x_dtype) || !group_ok(g) || M < 0 || K <= 0 || K % g != 0 || ldq < K)
        return CK_ERR_INVALID_ARG;
    if (M == 0) return CK_OK;
    if (!x || !R || !codes || !scales) return CK_ERR_INVALID_ARG;
    if (!aligned(R, 16)) return CK_ERR_INVALID_ARG;
    return launch_rotate_quant(x, x_dtype, M, K, stride_m, stride_k, R, g, scale_in, codes, ldq,
                               scales, qmax, dev_status, stream);
}

ck_status ck_rotate_quant(const void* x, ck_dtype x_dtype, int64_t M, int64_t K,
                          int64_t stride_m, int64_t stride_k, const void* R, int g,
                          const float* scale_in, int8_t* codes, int64_t ldq, float* scales,
                          int* dev_status, cudaStream_t stream) {
    return rotate_quant_checked(x, x_dtype, M, K, stride_m, stride_k, R, g, scale_in, codes, ldq,
                                scales, 7, dev_status, stream);
}

ck_status ck_rotate_quant_int8(const void* x, ck_dtype x_dtype, int64_t M, int64_t K,
                               int64_t stride_m, int64_t stride_k, const void* R, int g,
                               const float* scale_in, int8_t* codes, int64_t ldq, float* scales,
                               int* dev_status, cudaStream_t stream) {
    return rotate_quant_checked(x, x_dtype, M, K, stride_m, stride_k, R, g, scale_in, codes, ldq,
                                scales, 127, dev_status, stream);
}

ck_status ck_rotate_quant_packed(const void* x, ck_dtype x_dtype, int64_t M, int64_t K,
                                 int64_t stride_m, int64_t stride_k, const void* R, int g,
                                 const float* scale_in, int stochastic, uint64_t seed,
                                 uint64_t offset, uint8_t* packed, int64_t ld_packed,
                                 float* scales, cudaStream_t stream) {
    if (!float_dtype(x_dtype) || !group_ok(g) || M < 0 || K <= 0 || K % 2 != 0 || K % g != 0 ||
        ld_packed < K / 2 || (stochastic != 0 && stochastic != 1))
        return CK_ERR_INVALID_ARG;
    if (M == 0) return CK_OK;
    if (!x || !R || !packed || !scales) return CK_ERR_INVALID_ARG;
    return launch_rotate_quant_packed(x, x_dtype, M, K, stride_m, stride_k, R, g, scale_in,
                                      stochastic != 0, seed, offset, packed, ld_packed, scales,
                                      stream);
}

ck_status ck_unpack_w4(const int8_t* packed, int64_t N, int64_t K, int64_t ld_packed,
                       int8_t* out, int64_t ld_out, cudaStream_t stream) {
    if (N < 0 || K <= 0 || K % 2 != 0 || ld_packed < K / 2 || ld_out < K)
        return CK_ERR_INVALID_ARG;
    if (N == 0) return CK_OK;
    if (!packed || !out) return CK_ERR_INVALID_ARG;
    return launch_unpack_w4(packed, N, K, ld_packed, out, ld_out, stream);
}

}  // extern "C"

namespace ck {

// The linear once its outputs' places are known (one segment, or one per group); every
// argument check but the outputs' is here.
static ck_status linear_impl(const void* x, ck_dtype x_dtype, int64_t M, int64_t K,
                             int64_t stride_m, int64_t stride_k, const void* R, int g,
                             const float* a_scale, const int8_t* w_packed, int64_t N, int64_t w_ld,
                             const void* w_scale, ck_dtype scale_dtype, const void* bias,
                             const OutSegs& segs, ck_dtype out_dtype, void* workspace,
                             size_t workspace_bytes, bool w8, int* dev_status,
                             cudaStream_t stream) {
    const bool codes_in = x_dtype == CK_I8;
    if (!(codes_in || float_dtype(x_dtype)) || !float_dtype(scale_dtype) ||
        !float_dtype(out_dtype))
        return CK_ERR_INVALID_ARG;
    if (M < 0 || N < 0 || K <= 0 || K % 2 != 0 || w_ld < (w8 ? K : K / 2))
        return CK_ERR_INVALID_ARG;
    if (codes_in) {
        if (stride_k != 1 || stride_m < K) return CK_ERR_INVALID_ARG;
    } else {
        if (!group_ok(g) || K % g != 0) return CK_ERR_INVALID_ARG;
    }
    if (K > (w8 ? kMaxK8 : kMaxK)) return CK_ERR_OVERFLOW;
    if (M == 0 || N == 0) return CK_OK;
    if (!x || !w_packed || !w_scale) return CK_ERR_INVALID_ARG;
    for (int s = 0; s < segs.n; ++s)
        if (segs.start[s + 1] > segs.start[s] && !segs.ptr[s]) return CK_ERR_INVALID_ARG;
    if (codes_in ? !a_scale : (!R || !aligned(R, 16))) return CK_ERR_INVALID_ARG;
    if (M >= (1LL << 31) || N >= (1LL << 31)) return CK_ERR_UNSUPPORTED;

    unsigned char* ws = static_cast<unsigned char*>(workspace);
    const int64_t P = ck_workspace_codes_pitch(K);
    const size_t scales_off = ck_workspace_scales_offset(M, K);
    const size_t wcopy_off = scales_off + (size_t)round_up(4 * M, 256);
    const bool codes_aligned = codes_in && aligned(x, 16) && stride_m % 16 == 0;
    const bool w_aligned = aligned(w_packed, 16) && w_ld % 16 == 0;
    const size_t need = linear_scratch_need(x, x_dtype, M, K, stride_m, w_packed, N, w_ld, w8);
    if (need) {
        if (!ws || workspace_bytes < need || !aligned(ws, 256)) return CK_ERR_WORKSPACE;
    }

    const int8_t* codes;
    int64_t ldq;
    const float* row_scale;
    ck_status st = CK_OK;
    if (codes_in) {
        if (codes_aligned) {
            codes = static_cast<const int8_t*>(x);
            ldq = stride_m;
        } else {
            st = launch_copy_rows(static_cast<const int8_t*>(x), stride_m,
                                  reinterpret_cast<int8_t*>(ws), P, M, K, stream);
            if (st != CK_OK) return st;
            codes = reinterpret_cast<const int8_t*>(ws);
            ldq = P;
        }
        row_scale = a_scale;
    } else {
        int8_t* wcodes = reinterpret_cast<int8_t*>(ws);
        float* wscales = reinterpret_cast<float*>(ws + scales_off);
        st = launch_rotate_quant(x, x_dtype, M, K, stride_m, stride_k, R, g, nullptr, wcodes, P,
                                 wscales, w8 ? 127 : 7, dev_status, stream);
        if (st != CK_OK) return st;
        codes = wcodes;
        ldq = P;
        row_scale = wscales;
    }
    const int8_t* wp = w_packed;
    int64_t wld = w_ld;
    if (!w_aligned) {
        const int64_t wrow = w8 ? K : K / 2;
        const int64_t wp_pitch = round_up(wrow, 16);
        int8_t* dst = reinterpret_cast<int8_t*>(ws + wcopy_off);
        st = launch_copy_rows(w_packed, w_ld, dst, wp_pitch, N, wrow, stream);
        if (st != CK_OK) return st;
        wp = dst;
        wld = wp_pitch;
    }
    // the GEMM overlaps stage 1's tail when stage 1 is the kernel right before it
    const bool after_stage1 = !codes_in && w_aligned;
    if (w8)
        return launch_w8a8_gemm(codes, ldq, row_scale, M, K, wp, wld, N, w_scale, scale_dtype,
                                bias, segs, out_dtype, after_stage1, dev_status, stream);
    return launch_w4a4_gemm(codes, ldq, row_scale, M, K, wp, wld, N, w_scale, scale_dtype, bias,
                            segs, out_dtype, after_stage1, dev_status, stream);
}

}  // namespace ck

extern "C" {

ck_status ck_w4a4_linear(const void* x, ck_dtype x_dtype, int64_t M, int64_t K,
                         int64_t stride_m, int64_t stride_k, const void* R, int g,
                         const float* a_scale, const int8_t* w_packed, int64_t N, int64_t w_ld,
                         const void* w_scale, ck_dtype scale_dtype, const void* bias,
                         void* out, ck_dtype out_dtype, int64_t ldo, void* workspace,
                         size_t workspace_bytes, int* dev_status, cudaStream_t stream) {
    if (ldo < N) return CK_ERR_INVALID_ARG;
    if (M > 0 && N > 0 && !out) return CK_ERR_INVALID_ARG;
    return linear_impl(x, x_dtype, M, K, stride_m, stride_k, R, g, a_scale, w_packed, N, w_ld,
                       w_scale, scale_dtype, bias, single_segment(out, N, ldo), out_dtype,
                       workspace, workspace_bytes, false, dev_status, stream);
}

ck_status ck_w8a8_linear(const void* x, ck_dtype x_dtype, int64_t M, int64_t K,
                         int64_t stride_m, int64_t stride_k, const void* R, int g,
                         const float* a_scale, const int8_t* w, int64_t N, int64_t w_ld,
                         const void* w_scale, ck_dtype scale_dtype, const void* bias,
                         void* out, ck_dtype out_dtype, int64_t ldo, void* workspace,
                         size_t workspace_bytes, int* dev_status, cudaStream_t stream) {
    if (ldo < N) return CK_ERR_INVALID_ARG;
    if (M > 0 && N > 0 && !out) return CK_ERR_INVALID_ARG;
    return linear_impl(x, x_dtype, M, K, stride_m, stride_k, R, g, a_scale, w, N, w_ld, w_scale,
                       scale_dtype, bias, single_segment(out, N, ldo), out_dtype, workspace,
                       workspace_bytes, true, dev_status, stream);
}

ck_status ck_w4a4_grouped_linear(const void* x, ck_dtype x_dtype, int64_t M, int64_t K,
                                 int64_t stride_m, int64_t stride_k, const void* R, int g,
                                 const float* a_scale, const int8_t* w_packed, int64_t w_ld,
                                 const void* w_scale, ck_dtype scale_dtype, const void* bias,
                                 int n_groups, const int64_t* group_n, void* const* outs,
                                 const int64_t* ldos, ck_dtype out_dtype, void* workspace,
                                 size_t workspace_bytes, int* dev_status, cudaStream_t stream) {
    if (n_groups < 1 || n_groups > kMaxOutSegs || !group_n || !outs || !ldos)
        return CK_ERR_INVALID_ARG;
    OutSegs segs = {};
    segs.n = n_groups;
    int64_t N = 0;
    for (int i = 0; i < n_groups; ++i) {
        if (group_n[i] < 0 || ldos[i] < group_n[i]) return CK_ERR_INVALID_ARG;
        segs.start[i] = N;
        segs.ptr[i] = outs[i];
        segs.ldo[i] = ldos[i];
        N += group_n[i];
    }
    segs.start[n_groups] = N;
    return linear_impl(x, x_dtype, M, K, stride_m, stride_k, R, g, a_scale, w_packed, N, w_ld,
                       w_scale, scale_dtype, bias, segs, out_dtype, workspace, workspace_bytes,
                       false, dev_status, stream);
}

}  // extern "C"
