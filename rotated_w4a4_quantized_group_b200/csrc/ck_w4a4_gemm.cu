// ck_w4a4_gemm.cu -- stage 2: INT4 x INT4 GEMM with exact INT32 accumulation and the
// cast -> x a_scale[m] -> x w_scale[n] -> + bias[n] epilogue.
//
// Operation (comfy-kitchen PR #198 "Consolidate INT8, RotateQuant, RoPE and ConvRot W4A4
// backends", "W4A4 correctness and performance scope": the same A4/W4 codes unpacked to
// INT8 and accumulated into INT32 at unit scale, then cast and scaled in eager's order;
// PR #201 "Avoid activation pack/unpack in ConvRot W4A4": activation codes arrive as INT8,
// only the weights are unpacked):
//   acc[m, n] = sum_k q[m, k] * w[n, k]
//   out[m, n] = cvt(((fp32(acc) * a_scale[m]) * w_scale[n]) + bias[n])
//
// One CTA computes a 128 x 256 output tile on one SM:
//   warp 0      TMA producer: A codes (128 x 128 bytes, 128-byte swizzle) and packed W
//               (256 rows x 64 bytes) into a 3-stage shared-memory ring;
//   warp 1      TMEM allocation and the single MMA-issuing thread
//               (tcgen05.mma.cta_group::1.kind::i8, 128 x 256 x 32 per instruction);
//   warps 4-7   unpack each W stage from nibbles to sign-extended INT8 in the
//               128-byte-swizzled K-major layout the MMA reads, then, after the K loop,
//               the epilogue: tcgen05.ld of the INT32 accumulators, scales, bias, store.
// Out-of-range rows/columns arrive as zeros from TMA and are masked at the store, so any
// M, N and K (K a multiple of 2) work.  Every wait is bounded (see ck_device.cuh).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "ck_device.cuh"
#include "ck_internal.h"

namespace ck {

namespace gemm {
constexpr int BM = 128;                 // rows of A (activation rows) per tile
constexpr int BN = 256;                 // rows of W (output channels) per tile
constexpr int BK = 128;                 // K elements (bytes of A) per stage
constexpr int STAGES = 3;
constexpr int A_BYTES = BM * BK;        // 16 KB
constexpr int WP_BYTES = BN * BK / 2;   // 16 KB packed weights
constexpr int B_BYTES = BN * BK;        // 32 KB unpacked weights
constexpr int STAGE_BYTES = A_BYTES + WP_BYTES + B_BYTES;
constexpr int THREADS = 256;
constexpr uint32_t TMEM_COLS = 256;     // one 128 x 256 int32 accumulator
constexpr int UNPACK_WARP0 = 4;         // warps 4..7
constexpr size_t SMEM_BYTES = (size_t)STAGES * STAGE_BYTES + 1024;
}  // namespace gemm

struct GemmParams {
    int64_t M, N, ldo;
    int num_kb;
    int vec_out;
    const float* a_scale;
    const void* w_scale;
    const void* bias;
    void* out;
    int* dev_status;
};

// 8 packed bytes' worth of nibbles in one 32-bit word -> 8 sign-extended INT8 codes,
// in k order (low nibble of byte i is k = 2i).  Each nibble is flipped to an unsigned
// offset u = v ^ 8, then (u + 0x78) ^ 0x80 = u - 8 per byte without cross-byte carries.
__device__ __forceinline__ void unpack_word(uint32_t w, uint32_t& o0, uint32_t& o1) {
    const uint32_t x = w ^ 0x88888888u;
    uint32_t lo = x & 0x0F0F0F0Fu;
    uint32_t hi = (x >> 4) & 0x0F0F0F0Fu;
    lo = (lo + 0x78787878u) ^ 0x80808080u;
    hi = (hi + 0x78787878u) ^ 0x80808080u;
    o0 = __byte_perm(lo, hi, 0x5140);   // k0 k1 k2 k3
    o1 = __byte_perm(lo, hi, 0x7362);   // k4 k5 k6 k7
}

template <typename T> __device__ __forceinline__ float load_scale(const void* p, int64_t i);
template <> __device__ __forceinline__ float load_scale<float>(const void* p, int64_t i) {
    return static_cast<const float*>(p)[i];
}
template <> __device__ __forceinline__ float load_scale<__half>(const void* p, int64_t i) {
    return __half2float(static_cast<const __half*>(p)[i]);
}
template <> __device__ __forceinline__ float load_scale<__nv_bfloat16>(const void* p, int64_t i) {
    return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
}

template <typename OutT> struct OutStore;
template <> struct OutStore<float> {
    static constexpr int kPerVec = 4;
    __device__ static __forceinline__ void vec(float* dst, const float* v) {
        for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
    }
    __device__ static __forceinline__ void one(float* dst, float v) { *dst = v; }
};
template <> struct OutStore<__nv_bfloat16> {
    __device__ static __forceinline__ void vec(__nv_bfloat16* dst, const float* v) {
        for (int i = 0; i < 32; i += 8) {
            uint32_t u[4];
            for (int j = 0; j < 4; ++j) {
                __nv_bfloat162 h = __floats2bfloat162_rn(v[i + 2 * j], v[i + 2 * j + 1]);
                u[j] = *reinterpret_cast<uint32_t*>(&h);
            }
            *reinterpret_cast<uint4*>(dst + i) = make_uint4(u[0], u[1], u[2], u[3]);
        }
    }
    __device__ static __forceinline__ void one(__nv_bfloat16* dst, float v) {
        *dst = __float2bfloat16_rn(v);
    }
};
template <> struct OutStore<__half> {
    __device__ static __forceinline__ void vec(__half* dst, const float* v) {
        for (int i = 0; i < 32; i += 8) {
            uint32_t u[4];
            for (int j = 0; j < 4; ++j) {
                __half2 h = __floats2half2_rn(v[i + 2 * j], v[i + 2 * j + 1]);
                u[j] = *reinterpret_cast<uint32_t*>(&h);
            }
            *reinterpret_cast<uint4*>(dst + i) = make_uint4(u[0], u[1], u[2], u[3]);
        }
    }
    __device__ static __forceinline__ void one(__half* dst, float v) { *dst = __float2half_rn(v); }
};

template <typename OutT, typename ScaleT>
__global__ void __launch_bounds__(gemm::THREADS, 1)
    w4a4_gemm_kernel(const __grid_constant__ CUtensorMap amap,
                     const __grid_constant__ CUtensorMap wmap, GemmParams p) {
    using namespace gemm;
    extern __shared__ __align__(1024) unsigned char gemm_smem[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(gemm_smem) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t full_bar[STAGES], unpacked_bar[STAGES], empty_bar[STAGES];
    __shared__ __align__(8) uint64_t accum_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_flag;
    __shared__ float ws_sh[BN], bias_sh[BN];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t n0 = (int64_t)blockIdx.x * BN;
    const int64_t m0 = (int64_t)blockIdx.y * BM;
    auto A_st = [&](int s) { return smem + (size_t)s * STAGE_BYTES; };
    auto WP_st = [&](int s) { return smem + (size_t)s * STAGE_BYTES + A_BYTES; };
    auto B_st = [&](int s) { return smem + (size_t)s * STAGE_BYTES + A_BYTES + WP_BYTES; };

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&unpacked_bar[s], 4);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(&accum_bar, 1);
        abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&amap);
        tma_prefetch_desc(&wmap);
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_sh, TMEM_COLS);
        tmem_relinquish();
    }
    if (warp >= UNPACK_WARP0) {
        for (int i = tid - UNPACK_WARP0 * 32; i < BN; i += 128) {
            const int64_t n = n0 + i;
            ws_sh[i] = n < p.N ? load_scale<ScaleT>(p.w_scale, n) : 0.f;
            bias_sh[i] = (p.bias && n < p.N) ? load_scale<ScaleT>(p.bias, n) : 0.f;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_sh;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int issued = 0;
            for (int kb = 0; kb < p.num_kb; ++kb) {
                const int s = kb % STAGES;
                const uint32_t round = (uint32_t)(kb / STAGES);
                if (kb >= STAGES &&
                    !mbar_wait(&empty_bar[s], (round - 1) & 1u, &abort_flag, p.dev_status))
                    break;
                mbar_arrive_expect_tx(&full_bar[s], A_BYTES + WP_BYTES);
                tma_load_2d(A_st(s), &amap, &full_bar[s], kb * BK, (int32_t)m0);
                tma_load_2d(WP_st(s), &wmap, &full_bar[s], kb * (BK / 2), (int32_t)n0);
                ++issued;
            }
            if (abort_flag) {
                // let copies already in flight land before the CTA exits
                for (int kb = issued > STAGES ? issued - STAGES : 0; kb < issued; ++kb)
                    mbar_wait(&full_bar[kb % STAGES], (uint32_t)(kb / STAGES) & 1u, nullptr, nullptr);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_i8(BM, BN);
            for (int kb = 0; kb < p.num_kb; ++kb) {
                const int s = kb % STAGES;
                const uint32_t par = (uint32_t)(kb / STAGES) & 1u;
                if (!mbar_wait(&full_bar[s], par, &abort_flag, p.dev_status)) break;
                if (!mbar_wait(&unpacked_bar[s], par, &abort_flag, p.dev_status)) break;
                tc_fence_after();
                const uint64_t adesc = smem_desc_k_sw128(smem_u32(A_st(s)));
                const uint64_t bdesc = smem_desc_k_sw128(smem_u32(B_st(s)));
#pragma unroll
                for (int kk = 0; kk < BK / 32; ++kk) {
                    // advance 32 bytes (one MMA K step) inside the 128-byte swizzled row
                    tc_mma_i8(tmem_base, adesc + (uint64_t)(kk * 2), bdesc + (uint64_t)(kk * 2),
                              idesc, (kb | kk) != 0 ? 1u : 0u);
                }
                tc_commit(&empty_bar[s]);
            }
            tc_commit(&accum_bar);
            // drain: every MMA issued above has completed once accum_bar flips
            mbar_wait(&accum_bar, 0, nullptr, p.dev_status);
        }
    } else if (warp >= UNPACK_WARP0) {
        // ------------------------------------------------------------ unpack, then epilogue
        const int ut = tid - UNPACK_WARP0 * 32;
        for (int kb = 0; kb < p.num_kb; ++kb) {
            const int s = kb % STAGES;
            const uint32_t par = (uint32_t)(kb / STAGES) & 1u;
            if (!mbar_wait(&full_bar[s], par, &abort_flag, p.dev_status)) break;
            const unsigned char* wp = WP_st(s);
            unsigned char* bdst = B_st(s);
#pragma unroll 4
            for (int it = 0; it < (BN * 8) / 128; ++it) {
                const int task = it * 128 + ut;
                const int row = task >> 3, ch = task & 7;
                const uint2 v = *reinterpret_cast<const uint2*>(wp + row * 64 + ch * 8);
                uint4 o;
                unpack_word(v.x, o.x, o.y);
                unpack_word(v.y, o.z, o.w);
                *reinterpret_cast<uint4*>(bdst + (row >> 3) * 1024 + (row & 7) * 128 +
                                          ((ch ^ (row & 7)) << 4)) = o;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&unpacked_bar[s]);
        }

        if (mbar_wait(&accum_bar, 0, &abort_flag, p.dev_status)) {
            tc_fence_after();
            const int q = warp & 3;
            const int64_t row = m0 + q * 32 + lane;
            const bool row_ok = row < p.M;
            const float a_s = row_ok ? p.a_scale[row] : 0.f;
            OutT* orow = static_cast<OutT*>(p.out) + (row_ok ? row : 0) * p.ldo + n0;
            for (int c0 = 0; c0 < BN; c0 += 32) {
                if (n0 + c0 >= p.N) break;
                uint32_t r[32];
                tc_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)c0, r);
                tc_wait_ld();
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    float o = __int2float_rn((int)r[i]);
                    o = __fmul_rn(o, a_s);
                    o = __fmul_rn(o, ws_sh[c0 + i]);
                    if (p.bias) o = __fadd_rn(o, bias_sh[c0 + i]);
                    v[i] = o;
                }
                if (!row_ok) continue;
                if (p.vec_out && n0 + c0 + 32 <= p.N) {
                    OutStore<OutT>::vec(orow + c0, v);
                } else {
                    for (int i = 0; i < 32; ++i)
                        if (n0 + c0 + i < p.N) OutStore<OutT>::one(orow + c0 + i, v[i]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

template <typename OutT, typename ScaleT>
static ck_status launch_typed(const CUtensorMap& amap, const CUtensorMap& wmap,
                              const GemmParams& p, dim3 grid, cudaStream_t stream) {
    auto kern = w4a4_gemm_kernel<OutT, ScaleT>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)gemm::SMEM_BYTES) != cudaSuccess)
        return CK_ERR_CUDA;
    kern<<<grid, gemm::THREADS, gemm::SMEM_BYTES, stream>>>(amap, wmap, p);
    return cudaGetLastError() == cudaSuccess ? CK_OK : CK_ERR_CUDA;
}

template <typename OutT>
static ck_status launch_out(const CUtensorMap& amap, const CUtensorMap& wmap, const GemmParams& p,
                            dim3 grid, ck_dtype scale_dt, cudaStream_t stream) {
    switch (scale_dt) {
        case CK_F32: return launch_typed<OutT, float>(amap, wmap, p, grid, stream);
        case CK_F16: return launch_typed<OutT, __half>(amap, wmap, p, grid, stream);
        case CK_BF16: return launch_typed<OutT, __nv_bfloat16>(amap, wmap, p, grid, stream);
        default: return CK_ERR_INVALID_ARG;
    }
}

ck_status launch_w4a4_gemm(const int8_t* codes, int64_t ldq, const float* a_scale, int64_t M,
                           int64_t K, const int8_t* w_packed, int64_t w_ld, int64_t N,
                           const void* w_scale, ck_dtype scale_dt, const void* bias, void* out,
                           ck_dtype out_dt, int64_t ldo, int* dev_status, cudaStream_t stream) {
    using namespace gemm;
    if (M == 0 || N == 0) return CK_OK;
    CUtensorMap amap, wmap;
    {
        const uint64_t dims[2] = {(uint64_t)K, (uint64_t)M};
        const uint64_t strides[1] = {(uint64_t)ldq};
        const uint32_t box[2] = {BK, BM};
        ck_status st = encode_tma(&amap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, codes, dims, strides,
                                  box, CU_TENSOR_MAP_SWIZZLE_128B);
        if (st != CK_OK) return st;
    }
    {
        const uint64_t dims[2] = {(uint64_t)(K / 2), (uint64_t)N};
        const uint64_t strides[1] = {(uint64_t)w_ld};
        const uint32_t box[2] = {BK / 2, BN};
        ck_status st = encode_tma(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, w_packed, dims, strides,
                                  box, CU_TENSOR_MAP_SWIZZLE_NONE);
        if (st != CK_OK) return st;
    }
    GemmParams p;
    p.M = M;
    p.N = N;
    p.ldo = ldo;
    p.num_kb = (int)((K + BK - 1) / BK);
    const size_t osz = out_dt == CK_F32 ? 4 : 2;
    p.vec_out = (aligned(out, 16) && (ldo * (int64_t)osz) % 16 == 0) ? 1 : 0;
    p.a_scale = a_scale;
    p.w_scale = w_scale;
    p.bias = bias;
    p.out = out;
    p.dev_status = dev_status;
    dim3 grid((unsigned)((N + BN - 1) / BN), (unsigned)((M + BM - 1) / BM));
    switch (out_dt) {
        case CK_F32: return launch_out<float>(amap, wmap, p, grid, scale_dt, stream);
        case CK_F16: return launch_out<__half>(amap, wmap, p, grid, scale_dt, stream);
        case CK_BF16: return launch_out<__nv_bfloat16>(amap, wmap, p, grid, scale_dt, stream);
        default: return CK_ERR_INVALID_ARG;
    }
}

}  // namespace ck
