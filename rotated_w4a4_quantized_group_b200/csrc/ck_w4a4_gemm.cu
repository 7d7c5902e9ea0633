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
// Persistent, warp-specialised, one CTA per SM, 128 x BN output tiles (BN <= 240):
//   warp 0      TMA producer of the A codes (128 rows x 128 bytes, 128-byte swizzle), 4-stage ring
//   warp 2      TMA producer of the packed weights (BN rows x 64 bytes), 3-stage ring
//   warps 8-17  unpack each packed stage into the unpacked-weight ring (3 stages) in the
//               128-byte-swizzled K-major layout the tensor core reads
//   warp 1      TMEM allocation and the single MMA-issuing thread:
//               tcgen05.mma.cta_group::1.kind::i8, 128 x (BN + 16) x 32 per instruction,
//               into one of two TMEM accumulators (2 x 256 columns)
//   warps 4-7   epilogue: tcgen05.ld of the finished accumulator, fp32 scale/bias, store,
//               overlapped with the MMAs of the next tile
//
// Unsigned weight operand.  Each 4-bit code v in [-8, 7] is expanded to u = v + 8 in
// [0, 15] (one LOP3 per 8 nibbles: (w & 0x0F) ^ 0x08 per byte) and the MMA runs signed A x
// unsigned B, giving sum_k q*u = acc + 8 * sum_k q.  Sixteen extra B rows of constant 1 sit
// after the BN weight rows of every stage (written once), so accumulator column BN holds
// sum_k q[m, k] and the epilogue recovers acc = sum q*u - 8 * sum q exactly (mod 2^32, and
// the true acc fits in int32 under the 64*K guard).
//
// Every wait is bounded (ck_device.cuh); out-of-range rows/columns arrive as zeros from TMA
// and are masked at the store.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "ck_device.cuh"
#include "ck_internal.h"

namespace ck {

namespace gemm {
constexpr int BM = 128;                  // activation rows per tile (MMA M)
constexpr int BK = 128;                  // K elements (bytes of A) per stage
constexpr int BN_MAX = 240;              // weight rows per tile; MMA N = BN + 16 <= 256
constexpr int ONES = 16;                 // constant-one B rows that produce the row sums
constexpr int A_ST = 4, WP_ST = 3, B_ST = 3;
constexpr int A_BYTES = BM * BK;         // 16 KB
constexpr int WARP_TMA_A = 0, WARP_MMA = 1, WARP_TMA_W = 2;
constexpr int EPI_WARP0 = 4;             // warps 4..7 own TMEM lanes 0..127
constexpr int UNP_WARP0 = 8, UNP_WARPS = 10;
constexpr int UNP_THREADS = UNP_WARPS * 32;
constexpr int THREADS = UNP_WARP0 * 32 + UNP_THREADS;
// unpack task = (row, quarter): 16 packed bytes -> 32 codes.  Thread ut takes tasks
// ut + UNP_THREADS * j, i.e. rows (ut / 4) + UNP_ROW_STEP * j with the same quarter.
constexpr int UNP_ROW_STEP = UNP_THREADS / 4;
constexpr int UNP_MAX_J = (BN_MAX * 4 + UNP_THREADS - 1) / UNP_THREADS;
static_assert(UNP_ROW_STEP % 8 == 0, "row step must keep the swizzle phase");
constexpr uint32_t TMEM_COLS = 512;      // two accumulators of 256 columns
constexpr uint32_t ACC_COLS = 256;

__host__ __device__ constexpr uint32_t wp_stage_bytes(int bn) { return (uint32_t)bn * (BK / 2); }
__host__ __device__ constexpr uint32_t b_stage_bytes(int bn) { return (uint32_t)(bn + ONES) * BK; }
__host__ __device__ constexpr size_t smem_bytes(int bn) {
    return (size_t)A_ST * A_BYTES + (size_t)WP_ST * wp_stage_bytes(bn) +
           (size_t)B_ST * b_stage_bytes(bn) + 1024;
}
}  // namespace gemm

struct GemmParams {
    int64_t M, N, ldo;
    int num_kb;        // K blocks of BK
    int BN;            // weight rows per tile (multiple of 16, <= BN_MAX)
    int tiles_n;       // tiles along N
    int tiles;         // total tiles
    uint32_t idesc;    // MMA instruction descriptor for 128 x (BN + 16)
    int vec_out;
    const float* a_scale;
    const void* w_scale;
    const void* bias;
    void* out;
    int* dev_status;
};

// Eight 4-bit codes of one packed word -> eight unsigned u = v + 8 bytes in k order
// (the low nibble of byte i is k = 2i).
__device__ __forceinline__ void unpack_word_u(uint32_t w, uint32_t& o0, uint32_t& o1) {
    const uint32_t lo = (w & 0x0F0F0F0Fu) ^ 0x08080808u;          // k = 0, 2, 4, 6
    const uint32_t hi = ((w >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;   // k = 1, 3, 5, 7
    o0 = __byte_perm(lo, hi, 0x5140);                             // k0 k1 k2 k3
    o1 = __byte_perm(lo, hi, 0x7362);                             // k4 k5 k6 k7
}

template <typename T> __device__ __forceinline__ float load_scale(const void* p, int64_t i);
template <> __device__ __forceinline__ float load_scale<float>(const void* p, int64_t i) {
    return __ldg(static_cast<const float*>(p) + i);
}
template <> __device__ __forceinline__ float load_scale<__half>(const void* p, int64_t i) {
    return __half2float(__ldg(static_cast<const __half*>(p) + i));
}
template <> __device__ __forceinline__ float load_scale<__nv_bfloat16>(const void* p, int64_t i) {
    return __bfloat162float(__ldg(static_cast<const __nv_bfloat16*>(p) + i));
}

template <typename OutT> struct OutStore;
template <> struct OutStore<float> {
    __device__ static __forceinline__ void vec16(float* dst, const float* v) {
#pragma unroll
        for (int i = 0; i < 16; i += 4)
            *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
    }
    __device__ static __forceinline__ void one(float* dst, float v) { *dst = v; }
};
template <> struct OutStore<__nv_bfloat16> {
    __device__ static __forceinline__ void vec16(__nv_bfloat16* dst, const float* v) {
#pragma unroll
        for (int i = 0; i < 16; i += 8) {
            uint32_t u[4];
#pragma unroll
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
    __device__ static __forceinline__ void vec16(__half* dst, const float* v) {
#pragma unroll
        for (int i = 0; i < 16; i += 8) {
            uint32_t u[4];
#pragma unroll
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
    const uint32_t wp_bytes = wp_stage_bytes(p.BN);
    const uint32_t b_bytes = b_stage_bytes(p.BN);
    unsigned char* a_ring = smem;
    unsigned char* wp_ring = a_ring + (size_t)A_ST * A_BYTES;
    unsigned char* b_ring = wp_ring + (size_t)WP_ST * wp_bytes;

    __shared__ __align__(8) uint64_t a_full[A_ST], a_empty[A_ST];
    __shared__ __align__(8) uint64_t wp_full[WP_ST], wp_empty[WP_ST];
    __shared__ __align__(8) uint64_t b_full[B_ST], b_empty[B_ST];
    __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2], drain_bar, vec_ready[2];
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_flag;
    __shared__ __align__(16) float ws_sh[2][BN_MAX], bias_sh[2][BN_MAX];   // per-tile epilogue vectors

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < A_ST; ++s) { mbar_init(&a_full[s], 1); mbar_init(&a_empty[s], 1); }
        for (int s = 0; s < WP_ST; ++s) {
            mbar_init(&wp_full[s], 1);
            mbar_init(&wp_empty[s], UNP_WARPS);
        }
        for (int s = 0; s < B_ST; ++s) {
            mbar_init(&b_full[s], UNP_WARPS);
            mbar_init(&b_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&acc_full[s], 1);
            mbar_init(&acc_empty[s], 4);
            mbar_init(&vec_ready[s], 4);
        }
        mbar_init(&drain_bar, 1);
        abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&amap);
        tma_prefetch_desc(&wmap);
    }
    if (warp == WARP_MMA) {
        tmem_alloc(&tmem_base_sh, TMEM_COLS);
        tmem_relinquish();
    }
    if (warp >= UNP_WARP0) {
        // the constant-one rows after the weight rows of every unpacked stage
        const int ut = tid - UNP_WARP0 * 32;
        for (int s = 0; s < B_ST; ++s) {
            unsigned char* ones = b_ring + (size_t)s * b_bytes + (size_t)p.BN * BK;
            for (int i = ut; i < ONES * BK / 16; i += UNP_THREADS)
                reinterpret_cast<uint4*>(ones)[i] = make_uint4(0x01010101u, 0x01010101u,
                                                              0x01010101u, 0x01010101u);
        }
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_sh;

    if (warp == WARP_TMA_A) {
        // ---------------------------------------------------------------- A codes producer
        if (lane == 0) {
            uint32_t it = 0, issued = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < p.tiles; t += gridDim.x) {
                const int32_t m0 = (t / p.tiles_n) * BM;
                for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
                    const uint32_t s = it % A_ST, r = it / A_ST;
                    if (it >= (uint32_t)A_ST &&
                        !mbar_wait(&a_empty[s], (r - 1) & 1u, &abort_flag, p.dev_status)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&a_full[s], A_BYTES);
                    tma_load_2d(a_ring + (size_t)s * A_BYTES, &amap, &a_full[s], kb * BK, m0);
                    ++issued;
                }
            }
            if (!ok)
                for (uint32_t j = issued > A_ST ? issued - A_ST : 0; j < issued; ++j)
                    mbar_wait(&a_full[j % A_ST], (j / A_ST) & 1u, nullptr, nullptr);
        }
    } else if (warp == WARP_TMA_W) {
        // ---------------------------------------------------------------- packed W producer
        if (lane == 0) {
            uint32_t it = 0, issued = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < p.tiles; t += gridDim.x) {
                const int32_t n0 = (t % p.tiles_n) * p.BN;
                for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
                    const uint32_t s = it % WP_ST, r = it / WP_ST;
                    if (it >= (uint32_t)WP_ST &&
                        !mbar_wait(&wp_empty[s], (r - 1) & 1u, &abort_flag, p.dev_status)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&wp_full[s], wp_bytes);
                    tma_load_2d(wp_ring + (size_t)s * wp_bytes, &wmap, &wp_full[s], kb * (BK / 2),
                                n0);
                    ++issued;
                }
            }
            if (!ok)
                for (uint32_t j = issued > WP_ST ? issued - WP_ST : 0; j < issued; ++j)
                    mbar_wait(&wp_full[j % WP_ST], (j / WP_ST) & 1u, nullptr, nullptr);
        }
    } else if (warp == WARP_MMA) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            uint32_t it = 0, lt = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < p.tiles; t += gridDim.x, ++lt) {
                const uint32_t acc = lt & 1u;
                if (lt >= 2 && !mbar_wait(&acc_empty[acc], ((lt >> 1) - 1) & 1u, &abort_flag,
                                          p.dev_status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * ACC_COLS;
                for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
                    const uint32_t sa = it % A_ST, sb = it % B_ST;
                    if (!mbar_wait(&a_full[sa], (it / A_ST) & 1u, &abort_flag, p.dev_status) ||
                        !mbar_wait(&b_full[sb], (it / B_ST) & 1u, &abort_flag, p.dev_status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t adesc = smem_desc_k_sw128(smem_u32(a_ring + (size_t)sa * A_BYTES));
                    const uint64_t bdesc = smem_desc_k_sw128(smem_u32(b_ring + (size_t)sb * b_bytes));
#pragma unroll
                    for (int kk = 0; kk < BK / 32; ++kk) {
                        // advance 32 bytes (one MMA K step) inside the 128-byte swizzled row
                        tc_mma_i8(d_tmem, adesc + (uint64_t)(kk * 2), bdesc + (uint64_t)(kk * 2),
                                  p.idesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    tc_commit(&a_empty[sa]);
                    tc_commit(&b_empty[sb]);
                }
                if (ok) tc_commit(&acc_full[acc]);
            }
            // every MMA issued above has completed once drain_bar flips
            tc_commit(&drain_bar);
            mbar_wait(&drain_bar, 0, nullptr, p.dev_status);
        }
    } else if (warp >= UNP_WARP0) {
        // ---------------------------------------------------------------- unpack
        constexpr int ROW_STEP = UNP_ROW_STEP;
        const int ut = tid - UNP_WARP0 * 32;
        const int row0 = ut >> 2, q = ut & 3;
        const int n_j = (p.BN * 4 - ut + UNP_THREADS - 1) / UNP_THREADS;   // 0..UNP_MAX_J
        const uint32_t ld_off = (uint32_t)(row0 * 64 + q * 16);
        const uint32_t st_base = (uint32_t)((row0 >> 3) * 1024 + (row0 & 7) * 128);
        const uint32_t st_off0 = st_base + (uint32_t)(((2 * q) ^ (row0 & 7)) << 4);
        const uint32_t st_off1 = st_base + (uint32_t)(((2 * q + 1) ^ (row0 & 7)) << 4);
        uint32_t it = 0;
        bool ok = true;
        for (int t = blockIdx.x; ok && t < p.tiles; t += gridDim.x) {
            for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
                const uint32_t sw = it % WP_ST, sb = it % B_ST;
                if (!mbar_wait(&wp_full[sw], (it / WP_ST) & 1u, &abort_flag, p.dev_status) ||
                    (it >= (uint32_t)B_ST &&
                     !mbar_wait(&b_empty[sb], ((it / B_ST) - 1) & 1u, &abort_flag, p.dev_status))) {
                    ok = false;
                    break;
                }
                const unsigned char* wp = wp_ring + (size_t)sw * wp_bytes + ld_off;
                unsigned char* bdst = b_ring + (size_t)sb * b_bytes;
                // all loads first (row step j: ROW_STEP * 64 packed bytes further, and
                // ROW_STEP / 8 swizzle atoms of ROW_STEP * 128 bytes in the unpacked tile)
                uint4 v[UNP_MAX_J];
#pragma unroll
                for (int j = 0; j < UNP_MAX_J; ++j)
                    v[j] = *reinterpret_cast<const uint4*>(wp + (j < n_j ? j : 0) * ROW_STEP * 64);
#pragma unroll
                for (int j = 0; j < UNP_MAX_J; ++j) {
                    uint4 o0, o1;
                    unpack_word_u(v[j].x, o0.x, o0.y);
                    unpack_word_u(v[j].y, o0.z, o0.w);
                    unpack_word_u(v[j].z, o1.x, o1.y);
                    unpack_word_u(v[j].w, o1.z, o1.w);
                    if (j < n_j) {
                        *reinterpret_cast<uint4*>(bdst + st_off0 + j * (ROW_STEP * BK)) = o0;
                        *reinterpret_cast<uint4*>(bdst + st_off1 + j * (ROW_STEP * BK)) = o1;
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&wp_empty[sw]);
                    mbar_arrive(&b_full[sb]);
                }
            }
        }
    } else if (warp >= EPI_WARP0 && warp < EPI_WARP0 + 4) {
        // ---------------------------------------------------------------- epilogue
        const int qd = warp & 3;   // TMEM lanes 32*qd .. 32*qd + 31
        const int et = tid - EPI_WARP0 * 32;
        uint32_t lt = 0;
        for (int t = blockIdx.x; t < p.tiles; t += gridDim.x, ++lt) {
            const uint32_t acc = lt & 1u;
            const int64_t m0 = (int64_t)(t / p.tiles_n) * BM;
            const int64_t n0 = (int64_t)(t % p.tiles_n) * p.BN;
            // this tile's weight scales and bias, once, into the buffer of its parity; each
            // epilogue warp arrives on vec_ready after its share.  A warp rewrites a buffer
            // only after the previous tile's vec_ready phase, for which every warp arrived
            // after finishing the tile that last read it.
            float* ws_t = ws_sh[acc];
            float* bs_t = bias_sh[acc];
            for (int i = et; i < p.BN; i += 128) {
                const int64_t n = n0 + i;
                ws_t[i] = n < p.N ? load_scale<ScaleT>(p.w_scale, n) : 0.f;
                bs_t[i] = (p.bias && n < p.N) ? load_scale<ScaleT>(p.bias, n) : 0.f;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&vec_ready[acc]);
            if (!mbar_wait(&vec_ready[acc], (lt >> 1) & 1u, &abort_flag, p.dev_status)) break;
            if (!mbar_wait(&acc_full[acc], (lt >> 1) & 1u, &abort_flag, p.dev_status)) break;
            tc_fence_after();
            const int64_t row = m0 + qd * 32 + lane;
            const bool row_ok = row < p.M;
            const float a_s = row_ok ? __ldg(p.a_scale + row) : 0.f;
            const uint32_t tbase = tmem_base + acc * ACC_COLS + ((uint32_t)(qd * 32) << 16);
            uint32_t rs[16];
            tc_ld_32x32b_x16(tbase + (uint32_t)p.BN, rs);   // sum_k q[row, k] (16 copies)
            tc_wait_ld();
            const uint32_t corr = rs[0] * 8u;
            OutT* orow = static_cast<OutT*>(p.out) + (row_ok ? row : 0) * p.ldo;
            for (int c0 = 0; c0 < p.BN; c0 += 16) {
                uint32_t r[16];
                tc_ld_32x32b_x16(tbase + (uint32_t)c0, r);
                tc_wait_ld();
                const int64_t nb = n0 + c0;
                float v[16], wsv[16];
#pragma unroll
                for (int i = 0; i < 16; i += 4)
                    *reinterpret_cast<float4*>(&wsv[i]) = *reinterpret_cast<const float4*>(ws_t + c0 + i);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float o = __int2float_rn((int)(r[i] - corr));
                    o = __fmul_rn(o, a_s);
                    v[i] = __fmul_rn(o, wsv[i]);
                }
                if (p.bias) {
                    float bv[16];
#pragma unroll
                    for (int i = 0; i < 16; i += 4)
                        *reinterpret_cast<float4*>(&bv[i]) =
                            *reinterpret_cast<const float4*>(bs_t + c0 + i);
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = __fadd_rn(v[i], bv[i]);
                }
                if (row_ok && nb < p.N) {
                    if (p.vec_out && nb + 16 <= p.N) {
                        OutStore<OutT>::vec16(orow + nb, v);
                    } else {
                        for (int i = 0; i < 16; ++i)
                            if (nb + i < p.N) OutStore<OutT>::one(orow + nb + i, v[i]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[acc]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

template <typename OutT, typename ScaleT>
static ck_status launch_typed(const CUtensorMap& amap, const CUtensorMap& wmap,
                              const GemmParams& p, int grid, cudaStream_t stream) {
    auto kern = w4a4_gemm_kernel<OutT, ScaleT>;
    const size_t smem = gemm::smem_bytes(p.BN);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return CK_ERR_CUDA;
    kern<<<grid, gemm::THREADS, smem, stream>>>(amap, wmap, p);
    return cudaGetLastError() == cudaSuccess ? CK_OK : CK_ERR_CUDA;
}

template <typename OutT>
static ck_status launch_out(const CUtensorMap& amap, const CUtensorMap& wmap, const GemmParams& p,
                            int grid, ck_dtype scale_dt, cudaStream_t stream) {
    switch (scale_dt) {
        case CK_F32: return launch_typed<OutT, float>(amap, wmap, p, grid, stream);
        case CK_F16: return launch_typed<OutT, __half>(amap, wmap, p, grid, stream);
        case CK_BF16: return launch_typed<OutT, __nv_bfloat16>(amap, wmap, p, grid, stream);
        default: return CK_ERR_INVALID_ARG;
    }
}

// Tile width along N: the multiple of 16 (<= 240) that minimises the persistent schedule's
// length, (waves of 128 x BN tiles over the SMs) x BN, preferring wider tiles on ties.
static int choose_bn(int64_t M, int64_t N, int sms) {
    const int64_t tiles_m = (M + gemm::BM - 1) / gemm::BM;
    int best = gemm::BN_MAX;
    int64_t best_cost = -1;
    for (int bn = gemm::BN_MAX; bn >= 64; bn -= 16) {
        const int64_t tiles = tiles_m * ((N + bn - 1) / bn);
        const int64_t waves = (tiles + sms - 1) / sms;
        const int64_t cost = waves * (bn + gemm::ONES);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = bn;
        }
    }
    return best;
}

ck_status launch_w4a4_gemm(const int8_t* codes, int64_t ldq, const float* a_scale, int64_t M,
                           int64_t K, const int8_t* w_packed, int64_t w_ld, int64_t N,
                           const void* w_scale, ck_dtype scale_dt, const void* bias, void* out,
                           ck_dtype out_dt, int64_t ldo, int* dev_status, cudaStream_t stream) {
    using namespace gemm;
    if (M == 0 || N == 0) return CK_OK;
    const int sms = num_sms();
    const int BN = choose_bn(M, N, sms);
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
        const uint32_t box[2] = {BK / 2, (uint32_t)BN};
        ck_status st = encode_tma(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, w_packed, dims, strides,
                                  box, CU_TENSOR_MAP_SWIZZLE_NONE);
        if (st != CK_OK) return st;
    }
    GemmParams p;
    p.M = M;
    p.N = N;
    p.ldo = ldo;
    p.num_kb = (int)((K + BK - 1) / BK);
    p.BN = BN;
    p.tiles_n = (int)((N + BN - 1) / BN);
    const int64_t tiles = (int64_t)p.tiles_n * ((M + BM - 1) / BM);
    if (tiles >= (1LL << 31)) return CK_ERR_UNSUPPORTED;
    p.tiles = (int)tiles;
    // signed 8-bit A, unsigned 8-bit B, s32 accumulator, 128 x (BN + 16)
    p.idesc = (2u << 4) | (1u << 7) | (0u << 10) | ((uint32_t)((BN + ONES) >> 3) << 17) |
              ((uint32_t)(BM >> 4) << 24);
    const size_t osz = out_dt == CK_F32 ? 4 : 2;
    p.vec_out = (aligned(out, 16) && (ldo * (int64_t)osz) % 16 == 0) ? 1 : 0;
    p.a_scale = a_scale;
    p.w_scale = w_scale;
    p.bias = bias;
    p.out = out;
    p.dev_status = dev_status;
    const int grid = (int)(p.tiles < sms ? p.tiles : sms);
    switch (out_dt) {
        case CK_F32: return launch_out<float>(amap, wmap, p, grid, scale_dt, stream);
        case CK_F16: return launch_out<__half>(amap, wmap, p, grid, scale_dt, stream);
        case CK_BF16: return launch_out<__nv_bfloat16>(amap, wmap, p, grid, scale_dt, stream);
        default: return CK_ERR_INVALID_ARG;
    }
}

}  // namespace ck
