// ck_rotate_quant.cu -- stage 1: group-wise rotation in the input dtype, then row-wise
// signed-INT4 quantization with the codes kept in INT8 storage.
//
// Operation (comfy-kitchen PR #198 "Consolidate INT8, RotateQuant, RoPE and ConvRot W4A4
// backends", "W4A4 correctness and performance scope"; PR #201 "Avoid activation
// pack/unpack in ConvRot W4A4", "Summary"; PR #155 "Add fused RotateQuant backend"):
//   y[m, j*g + c] = dtype( sum_i x[m, j*g + i] * R[i, c] )      (fp32 accumulation)
//   s[m] = max(fp32(max_k |y[m, k]|) / 7, FLT_MIN)   or the caller's tensor-wise scale
//   q[m, k] = clamp(round_half_even(y[m, k] / s[m]), -8, 7)
//
// The kernels, tried in this order:
//   rq_tc_kernel       bf16/fp16, g in {16, 64, 256}, unit K stride, 16-byte aligned x and
//                      R; rows of at most 128 groups (g = 256) or 128 64-channel group-rows
//                      (g = 16 and 64; up to 256 in two parts).  Whole rows fill the 128 lanes
//                      of a tcgen05.mma.kind::f16 chain against R^T resident in shared memory
//                      (block-diagonal for g = 16: one MMA per 16-channel group); the fp32
//                      result in tensor memory is rounded, reduced and quantized by sixteen
//                      epilogue warps, several tiles in flight.
//   rq_row_kernel      bf16/fp16, g in {16, 64}, rows that fit two buffers per warp.  Each warp
//                      owns whole rows, filled by its own TMA copies, and rotates them with
//                      mma.sync (y^T = R^T x^T) in place.
//   rq_mma_kernel      bf16/fp16, g in {16, 64}, longer rows.  A TMA producer fills a ring of
//                      row blocks; two groups of compute warps rotate them with mma.sync and
//                      quantize from shared memory.
//   rq_f32_g16_kernel  (ck_rq_f32.cu) fp32, g = 16, row-major or column-major: K split over
//                      a cluster, FP64 tensor-core rotation, absmax over distributed shared memory.
//   fp32, g in {64, 256}, row-major: launch_rq_f32_wide (ck_rq_tf32.cu) picks the split-TF32
//                      tensor-core kernel (g = 64) or the FFMA kernel (g = 256).
//   rq_generic_kernel  every dtype, g and stride: one row per CTA step, fp32 FFMA with R
//                      in shared memory (or read through L1 when it does not fit).
// The TMA-fed kernels store 16 codes at a time where the code rows are 16-byte aligned; the
// generic kernel stores 4.
#include <algorithm>
#include <type_traits>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <float.h>
#include <stdint.h>

#include "ck_device.cuh"
#include "ck_internal.h"

namespace ck {

// ===================================================================== generic kernel

constexpr int kGenThreads = 256;
constexpr int kGenMaxChunks = 16;  // 4-wide chunks kept in registers per thread: K <= 16384

template <typename T>
__device__ __forceinline__ float4 load4(const T* p);
template <>
__device__ __forceinline__ float4 load4<float>(const float* p) {
    return *reinterpret_cast<const float4*>(p);
}
template <>
__device__ __forceinline__ float4 load4<__half>(const __half* p) {
    uint2 u = *reinterpret_cast<const uint2*>(p);
    float2 a = __half22float2(*reinterpret_cast<__half2*>(&u.x));
    float2 b = __half22float2(*reinterpret_cast<__half2*>(&u.y));
    return make_float4(a.x, a.y, b.x, b.y);
}
template <>
__device__ __forceinline__ float4 load4<__nv_bfloat16>(const __nv_bfloat16* p) {
    uint2 u = *reinterpret_cast<const uint2*>(p);
    float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u.x));
    float2 b = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u.y));
    return make_float4(a.x, a.y, b.x, b.y);
}

// One rotated 4-wide chunk: columns c0..c0+3 of group j, rounded to T.
template <typename T>
__device__ __forceinline__ float4 rotate_chunk(const float* xs, const T* Rp, int g, int64_t k0) {
    const int64_t j0 = (k0 / g) * g;
    const int c0 = (int)(k0 - j0);
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    for (int i = 0; i < g; ++i) {
        const float xv = xs[j0 + i];
        const float4 r = load4<T>(Rp + (int64_t)i * g + c0);
        a0 = fmaf(xv, r.x, a0);
        a1 = fmaf(xv, r.y, a1);
        a2 = fmaf(xv, r.z, a2);
        a3 = fmaf(xv, r.w, a3);
    }
    return make_float4(round_through<T>(a0), round_through<T>(a1), round_through<T>(a2),
                       round_through<T>(a3));
}

__device__ __forceinline__ float amax4(float m, float4 v) {
    m = fmax_nan(m, fabsf(v.x));
    m = fmax_nan(m, fabsf(v.y));
    m = fmax_nan(m, fabsf(v.z));
    return fmax_nan(m, fabsf(v.w));
}

__device__ __forceinline__ void store_codes4(int8_t* dst, float4 v, const RowDivisor& d, bool vec) {
    const int q0 = quant_code_fast(v.x, d), q1 = quant_code_fast(v.y, d),
              q2 = quant_code_fast(v.z, d), q3 = quant_code_fast(v.w, d);
    if (vec) {
        *reinterpret_cast<uint32_t*>(dst) = pack4_codes(q0, q1, q2, q3);
    } else {
        dst[0] = (int8_t)q0;
        dst[1] = (int8_t)q1;
        dst[2] = (int8_t)q2;
        dst[3] = (int8_t)q3;
    }
}

__device__ __forceinline__ float row_scale(float amax, const float* scale_in, int qmax) {
    float s = scale_in ? *scale_in : __fdiv_rn(amax, (float)qmax);
    return (s < FLT_MIN) ? FLT_MIN : s;   // lower clamp; NaN stays NaN
}

template <typename T, bool kKeep>
__global__ void __launch_bounds__(kGenThreads)
    rq_generic_kernel(const T* __restrict__ x, int64_t M, int64_t K, int64_t sm, int64_t sk,
                      const T* __restrict__ R, int g, int r_in_smem,
                      const float* __restrict__ scale_in, int8_t* __restrict__ codes, int64_t ldq,
                      float* __restrict__ scales, int vec_codes, int qmax) {
    // the linear's GEMM, launched as this kernel's dependent, may start its prologue now
    grid_dependents_launch();
    extern __shared__ __align__(16) unsigned char gen_smem[];
    float* xs = reinterpret_cast<float*>(gen_smem);
    T* Rs = reinterpret_cast<T*>(xs + K);
    __shared__ float warp_max[kGenThreads / 32];

    const int tid = threadIdx.x;
    if (r_in_smem)
        for (int i = tid; i < g * g; i += kGenThreads) Rs[i] = R[i];
    const T* Rp = r_in_smem ? Rs : R;
    const int64_t nchunk = K / 4;

    for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
        __syncthreads();
        const T* xr = x + m * sm;
        for (int64_t k = tid; k < K; k += kGenThreads) xs[k] = Elem<T>::to_f(xr[k * sk]);
        __syncthreads();

        float4 keep[kKeep ? kGenMaxChunks : 1];
        float mx = 0.f;
        if (kKeep) {
#pragma unroll
            for (int it = 0; it < kGenMaxChunks; ++it) {
                const int64_t ci = tid + (int64_t)it * kGenThreads;
                if (ci < nchunk) {
                    keep[it] = rotate_chunk<T>(xs, Rp, g, ci * 4);
                    mx = amax4(mx, keep[it]);
                }
            }
        } else {
            for (int64_t ci = tid; ci < nchunk; ci += kGenThreads)
                mx = amax4(mx, rotate_chunk<T>(xs, Rp, g, ci * 4));
        }
        for (int o = 16; o > 0; o >>= 1) mx = fmax_nan(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if ((tid & 31) == 0) warp_max[tid >> 5] = mx;
        __syncthreads();
        float amax = 0.f;
        for (int w = 0; w < kGenThreads / 32; ++w) amax = fmax_nan(amax, warp_max[w]);
        const float s = row_scale(amax, scale_in, qmax);
        if (tid == 0) scales[m] = s;
        const RowDivisor dv(s, qmax);

        int8_t* qr = codes + m * ldq;
        if (kKeep) {
#pragma unroll
            for (int it = 0; it < kGenMaxChunks; ++it) {
                const int64_t ci = tid + (int64_t)it * kGenThreads;
                if (ci < nchunk) store_codes4(qr + ci * 4, keep[it], dv, vec_codes != 0);
            }
        } else {
            for (int64_t ci = tid; ci < nchunk; ci += kGenThreads)
                store_codes4(qr + ci * 4, rotate_chunk<T>(xs, Rp, g, ci * 4), dv, vec_codes != 0);
        }
    }
}

// ===================================================================== MMA kernel


template <typename T> struct MmaOp;
template <> struct MmaOp<__nv_bfloat16> {
    __device__ static __forceinline__ void run(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, "
            "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
    __device__ static __forceinline__ uint32_t pack(float lo, float hi) {
        __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&v);
    }
    __device__ static __forceinline__ float2 unpack(uint32_t u) {
        return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u));
    }
    // the pair as an f32x2 register: a bf16 is the high half of its fp32
    __device__ static __forceinline__ unsigned long long unpack2(uint32_t u) {
        return f2_pack(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
    }
    // running max of |.| over packed pairs, NaN-propagating
    __device__ static __forceinline__ uint32_t absmax2(uint32_t m, uint32_t v) {
        uint32_t a = v & 0x7FFF7FFFu;
        __nv_bfloat162 r = __hmax2_nan(*reinterpret_cast<__nv_bfloat162*>(&m),
                                       *reinterpret_cast<__nv_bfloat162*>(&a));
        return *reinterpret_cast<uint32_t*>(&r);
    }
};
template <> struct MmaOp<__half> {
    __device__ static __forceinline__ void run(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, "
            "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
    __device__ static __forceinline__ uint32_t pack(float lo, float hi) {
        __half2 v = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&v);
    }
    __device__ static __forceinline__ float2 unpack(uint32_t u) {
        return __half22float2(*reinterpret_cast<__half2*>(&u));
    }
    __device__ static __forceinline__ unsigned long long unpack2(uint32_t u) {
        const float2 f = unpack(u);
        return f2_pack(f.x, f.y);
    }
    __device__ static __forceinline__ uint32_t absmax2(uint32_t m, uint32_t v) {
        uint32_t a = v & 0x7FFF7FFFu;
        __half2 r = __hmax2_nan(*reinterpret_cast<__half2*>(&m), *reinterpret_cast<__half2*>(&a));
        return *reinterpret_cast<uint32_t*>(&r);
    }
};

__device__ __forceinline__ void stmatrix_x4(uint32_t saddr, uint32_t r0, uint32_t r1, uint32_t r2,
                                            uint32_t r3) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(saddr),
                 "r"(r0), "r"(r1), "r"(r2), "r"(r3)
                 : "memory");
}

// Four 8x8 b16 matrices stored transposed: lane i of matrix j gives the address of shared-
// memory row i, which receives column i of the fragment matrix.
__device__ __forceinline__ void stmatrix_x4_trans(uint32_t saddr, uint32_t r0, uint32_t r1,
                                                  uint32_t r2, uint32_t r3) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(saddr),
                 "r"(r0), "r"(r1), "r"(r2), "r"(r3)
                 : "memory");
}

// group-rows of x per step of the row kernel's rotation
template <int G> constexpr int kRowStep = G == 64 ? 8 : 16;

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t saddr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(saddr));
}

// Byte offset of 16-byte chunk `c` of group-row `rho` in the TMA-swizzled box buffer.
// G = 64: 128-byte rows, 128-byte swizzle (chunk ^= rho % 8).
// G = 16: 32-byte rows, 32-byte swizzle (chunk ^= (rho / 4) % 2).
template <int G>
__device__ __forceinline__ uint32_t swz_off(int rho, int c) {
    if (G == 64) return (uint32_t)rho * 128u + (uint32_t)((c ^ (rho & 7)) << 4);
    return (uint32_t)rho * 32u + (uint32_t)((c ^ ((rho >> 2) & 1)) << 4);
}

struct RqMmaParams {
    int64_t M, K, ldq;
    int Gn;          // groups per row (K / G)
    int GB;          // groups per TMA box
    int NB;          // boxes per row block
    int RB;          // rows per block
    int S;           // ring stages (row blocks in flight)
    uint32_t box_stride;  // bytes between box buffers in shared memory
    uint32_t box_bytes;   // bytes one box copy delivers
    uint32_t stage_bytes; // bytes of one ring stage (NB boxes)
    int vec_codes;
    int qmax;             // code grid [-qmax - 1, qmax]
};

constexpr int kRqMaxStages = 8;
constexpr int kRqGroupWarps = 8;                            // warps of one compute group
constexpr int kRqGroups = 2;                                // groups take alternate blocks
constexpr int kRqComputeWarps = kRqGroupWarps * kRqGroups;
constexpr int kRqThreads = (kRqComputeWarps + 1) * 32;      // + one TMA producer warp

// R transposed (RT[n][k] = R[k][n]) in shared memory: rows of G bf16/fp16 values with the
// 16-byte chunks of row n XOR-swizzled by n % 8 (rows of 32 bytes for G = 16 use n / 4 % 2),
// so that ldmatrix of 8 consecutive rows is bank-conflict free.
template <int G>
__device__ __forceinline__ uint32_t rt_off(int n, int chunk) {
    if (G == 16) return (uint32_t)n * 32u + (uint32_t)((chunk ^ ((n >> 2) & 1)) << 4);
    return (uint32_t)n * (uint32_t)(G * 2) + (uint32_t)(((chunk & ~7) | ((chunk & 7) ^ (n & 7))) << 4);
}

// One persistent CTA per SM.  Warp 16 streams row blocks into a ring of shared-memory stages
// with TMA (several blocks in flight per SM); two groups of eight compute warps take
// alternate blocks: rotate in place (B fragments of R from shared memory), reduce the row
// absmax, compute the row scales, quantize, store the codes, and release the stage.  The
// phases of one block are separated by mbarriers (bounded waits), so one group's scale
// step overlaps the other group's work.
template <typename T, int G>
__global__ void __launch_bounds__(kRqThreads, 1)
    rq_mma_kernel(const __grid_constant__ CUtensorMap xmap, const T* __restrict__ R,
                  const float* __restrict__ scale_in, int8_t* __restrict__ codes,
                  float* __restrict__ scales, RqMmaParams p, int* dev_status) {
    // the linear's GEMM, launched as this kernel's dependent, may start its prologue now
    grid_dependents_launch();
    constexpr int KT = G / 16;   // k-tiles of the m16n8k16 MMA
    constexpr int NT = G / 8;    // n-tiles
    extern __shared__ __align__(1024) unsigned char mma_smem[];
    unsigned char* ring = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(mma_smem) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t full_bar[kRqMaxStages], empty_bar[kRqMaxStages];
    __shared__ __align__(8) uint64_t rot_done[kRqMaxStages], scale_ready[kRqMaxStages];
    __shared__ unsigned int amax_bits[kRqMaxStages][16];
    __shared__ float row_s[kRqMaxStages][16], row_r[kRqMaxStages][16];
    __shared__ int abort_flag;
    __shared__ __align__(128) unsigned char rt_sh[G * G * 2];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t n_blocks = (p.M + p.RB - 1) / p.RB;
    const int my_blocks =
        blockIdx.x < n_blocks ? (int)((n_blocks - 1 - blockIdx.x) / gridDim.x) + 1 : 0;

    if (tid == 0) {
        for (int s = 0; s < p.S; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], kRqGroupWarps);
            mbar_init(&rot_done[s], kRqGroupWarps);
            mbar_init(&scale_ready[s], 1);
        }
        abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&xmap);
    }
    if (tid < kRqMaxStages * 16) amax_bits[tid >> 4][tid & 15] = 0u;
    // R transposed into shared memory (the B operand: n = output channel, k = input channel)
    for (int i = tid; i < G * G; i += kRqThreads) {
        const int n = i / G, k = i % G;
        const T v = R[k * G + n];
        *reinterpret_cast<T*>(rt_sh + rt_off<G>(n, k / 8) + (k % 8) * 2) = v;
    }
    __syncthreads();

    if (warp == kRqComputeWarps) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            int issued = 0;
            for (int i = 0; i < my_blocks; ++i) {
                const int s = i % p.S;
                if (i >= p.S &&
                    !mbar_wait(&empty_bar[s], (uint32_t)((i / p.S) - 1) & 1u, &abort_flag, dev_status))
                    break;
                const int64_t blk = blockIdx.x + (int64_t)i * gridDim.x;
                unsigned char* stage = ring + (size_t)s * p.stage_bytes;
                mbar_arrive_expect_tx(&full_bar[s], p.box_bytes * (uint32_t)p.NB);
                for (int bx = 0; bx < p.NB; ++bx)
                    tma_load_3d(stage + (size_t)bx * p.box_stride, &xmap, &full_bar[s], 0, bx * p.GB,
                                (int32_t)(blk * p.RB));
                ++issued;
            }
            if (abort_flag)   // copies still in flight land before the CTA leaves
                for (int j = issued > p.S ? issued - p.S : 0; j < issued; ++j)
                    mbar_wait(&full_bar[j % p.S], (uint32_t)(j / p.S) & 1u, nullptr, nullptr);
        }
    } else {
        // ---------------------------------------------------------------- compute warps
        const int group = warp / kRqGroupWarps, gw = warp % kRqGroupWarps;
        const int gtid = tid % (kRqGroupWarps * 32);
        const uint32_t rt_base = smem_u32(rt_sh);
        const int rows_per_box = p.RB * p.GB;            // valid group-rows in one box
        const int tiles_per_box = (rows_per_box + 15) / 16;
        const int n_tiles = tiles_per_box * p.NB;
        const int chunks_per_row = (int)(p.K / 16);

        for (int i = group; i < my_blocks; i += kRqGroups) {
            const int s = i % p.S;
            const uint32_t par = (uint32_t)(i / p.S) & 1u;
            const int64_t m0 = (blockIdx.x + (int64_t)i * gridDim.x) * p.RB;
            unsigned char* buf = ring + (size_t)s * p.stage_bytes;
            if (!mbar_wait(&full_bar[s], par, &abort_flag, dev_status)) break;

            // ---- rotation: 16 consecutive group-rows per MMA tile, y written back in place
            for (int t = gw; t < n_tiles; t += kRqGroupWarps) {
                const int bx = t / tiles_per_box;
                const int rho0 = (t - bx * tiles_per_box) * 16;
                const uint32_t base = smem_u32(buf + (size_t)bx * p.box_stride);
                uint32_t afr[KT][4];
                {
                    const int rho = rho0 + (lane & 7) + ((lane >> 3) & 1) * 8;
                    const int cadd = lane >> 4;   // 0: k 0-7, 1: k 8-15 of the k-tile
#pragma unroll
                    for (int kt = 0; kt < KT; ++kt)
                        ldmatrix_x4(afr[kt], base + swz_off<G>(rho, kt * 2 + cadd));
                }
                float acc[NT][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
                for (int kt = 0; kt < KT; ++kt) {
                    // B fragments of two n-tiles per ldmatrix.x4: matrices (nt, k 0-7),
                    // (nt, k 8-15), (nt + 1, k 0-7), (nt + 1, k 8-15) of this k-tile
#pragma unroll
                    for (int nt = 0; nt < NT; nt += 2) {
                        uint32_t b4[4];
                        const int n = nt * 8 + ((lane >> 4) << 3) + (lane & 7);
                        ldmatrix_x4(b4, rt_base + rt_off<G>(n, kt * 2 + ((lane >> 3) & 1)));
                        MmaOp<T>::run(acc[nt], afr[kt], b4[0], b4[1]);
                        MmaOp<T>::run(acc[nt + 1], afr[kt], b4[2], b4[3]);
                    }
                }
                // round to T, store in place with stmatrix (8x8 blocks: rows rho0..+7 and
                // rho0+8..+15 of n-tiles nt and nt + 1; rows past the box land in its padding),
                // row absmax
                const int rA = rho0 + (lane >> 2), rB = rA + 8;
                uint32_t mA2 = 0u, mB2 = 0u;
                {
                    const int srow = rho0 + (lane & 7) + ((lane >> 3) & 1) * 8;
                    const int sn = (lane >> 4) & 1;
#pragma unroll
                    for (int nt = 0; nt < NT; nt += 2) {
                        const uint32_t pA0 = MmaOp<T>::pack(acc[nt][0], acc[nt][1]);
                        const uint32_t pB0 = MmaOp<T>::pack(acc[nt][2], acc[nt][3]);
                        const uint32_t pA1 = MmaOp<T>::pack(acc[nt + 1][0], acc[nt + 1][1]);
                        const uint32_t pB1 = MmaOp<T>::pack(acc[nt + 1][2], acc[nt + 1][3]);
                        mA2 = MmaOp<T>::absmax2(MmaOp<T>::absmax2(mA2, pA0), pA1);
                        mB2 = MmaOp<T>::absmax2(MmaOp<T>::absmax2(mB2, pB0), pB1);
                        stmatrix_x4(base + swz_off<G>(srow, nt + sn), pA0, pB0, pA1, pB1);
                    }
                }
                const float2 fA = MmaOp<T>::unpack(mA2), fB = MmaOp<T>::unpack(mB2);
                float mA = fmax_nan(fA.x, fA.y), mB = fmax_nan(fB.x, fB.y);
                mA = fmax_nan(mA, __shfl_xor_sync(0xffffffffu, mA, 1));
                mA = fmax_nan(mA, __shfl_xor_sync(0xffffffffu, mA, 2));
                mB = fmax_nan(mB, __shfl_xor_sync(0xffffffffu, mB, 1));
                mB = fmax_nan(mB, __shfl_xor_sync(0xffffffffu, mB, 2));
                if ((lane & 3) == 0) {
                    if (rA < rows_per_box) atomicMax(&amax_bits[s][rA / p.GB], __float_as_uint(mA));
                    if (rB < rows_per_box) atomicMax(&amax_bits[s][rB / p.GB], __float_as_uint(mB));
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&rot_done[s]);
            if (!mbar_wait(&rot_done[s], par, &abort_flag, dev_status)) break;

            // ---- row scales (the group's first warp), published through scale_ready
            if (gw == 0) {
                if (lane < p.RB) {
                    const float sc = row_scale(__uint_as_float(amax_bits[s][lane]), scale_in, p.qmax);
                    const RowDivisor dv(sc, p.qmax);
                    row_s[s][lane] = sc;
                    row_r[s][lane] = dv.r;
                    amax_bits[s][lane] = 0u;     // ready for the stage's next block
                    if (m0 + lane < p.M) scales[m0 + lane] = sc;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&scale_ready[s]);
            }
            if (!mbar_wait(&scale_ready[s], par, &abort_flag, dev_status)) break;

            // ---- quantize: 16 consecutive channels per thread step, 16-byte code stores
            for (int r = 0; r < p.RB; ++r) {
                if (m0 + r >= p.M) break;
                RowDivisor dv(row_s[s][r], p.qmax);
                dv.r = row_r[s][r];
                int8_t* dst_row = codes + (m0 + r) * p.ldq;
                for (int c = gtid; c < chunks_per_row; c += kRqGroupWarps * 32) {
                    const int k = c * 16;
                    const int j = k / G, e = k - j * G;
                    int bx = 0, jj = j;
                    if (p.NB > 1) {
                        bx = j / p.GB;
                        jj = j - bx * p.GB;
                    }
                    const int rho = r * p.GB + jj;
                    const unsigned char* bb = buf + (size_t)bx * p.box_stride;
                    const uint4 u0 = *reinterpret_cast<const uint4*>(bb + swz_off<G>(rho, e / 8));
                    const uint4 u1 = *reinterpret_cast<const uint4*>(bb + swz_off<G>(rho, e / 8 + 1));
                    const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
                    float y[16];
#pragma unroll
                    for (int h = 0; h < 8; ++h) {
                        const float2 a = MmaOp<T>::unpack(w[h]);
                        y[2 * h] = a.x;
                        y[2 * h + 1] = a.y;
                    }
                    uint32_t out[4];
                    quant16(y, dv, out);
                    int8_t* dst = dst_row + k;
                    if (p.vec_codes) {
                        *reinterpret_cast<uint4*>(dst) = make_uint4(out[0], out[1], out[2], out[3]);
                    } else {
#pragma unroll
                        for (int q = 0; q < 16; ++q)
                            dst[q] = (int8_t)((out[q / 4] >> (8 * (q % 4))) & 0xFF);
                    }
                }
            }
            // the stage's shared memory is no longer read by this warp
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty_bar[s]);
        }
    }
    __syncthreads();
}

// ===================================================================== row kernel

// One persistent CTA per SM whose warps own whole rows.  Each warp keeps two row buffers
// filled by its own TMA copies (3-D boxes of group-rows, swizzled like the ring kernel's):
// as soon as it has quantized a row it refills that buffer with its row after next.  It
// rotates each row in place (mma.sync m16n8k16 with R^T in shared memory, results rounded to
// T and written back with stmatrix), reduces the row absmax with warp shuffles, writes the row
// scale, quantizes from shared memory and stores the codes 16 bytes per lane.  No barrier is
// shared between warps.
constexpr int kRowMaxWarps = 12;   // warps
constexpr int kRowBufs = 2;        // row buffers per compute warp

struct RqRowParams {
    int64_t M, K, ldq;
    int GR;               // group-rows per row (K / G)
    int GB;               // group-rows per TMA box (a multiple of 8 when a row takes >1 box)
    int NB;               // boxes per row
    int W;                // compute warps
    uint32_t buf_bytes;   // one row buffer (a multiple of 1024 bytes)
    uint32_t box_bytes;   // bytes one box delivers
    int vec_codes;
    int qmax;             // code grid [-qmax - 1, qmax]
};

template <typename T, int G, bool DYN>
__global__ void __launch_bounds__(kRowMaxWarps * 32, 1)
    rq_row_kernel(const __grid_constant__ CUtensorMap xmap, const T* __restrict__ R,
                  const float* __restrict__ scale_in, int8_t* __restrict__ codes,
                  float* __restrict__ scales, RqRowParams p, int* dev_status) {
    // the linear's GEMM, launched as this kernel's dependent, may start its prologue now
    grid_dependents_launch();
    constexpr int KT = G / 16;   // k-tiles of the m16n8k16 MMA (input channels)
    constexpr int MT = G / 16;   // m-tiles (output channels)
    extern __shared__ __align__(1024) unsigned char row_smem[];
    unsigned char* bufs = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(row_smem) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t full_bar[kRowMaxWarps * kRowBufs];
    __shared__ int abort_flag;
    __shared__ __align__(128) unsigned char rt_sh[G * G * 2];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int W = p.W;
    // this CTA's rows: blockIdx.x + gridDim.x * j; row j goes to warp j % W, buffer (j / W) % 2
    const int64_t my_rows =
        (int64_t)blockIdx.x < p.M ? (p.M - 1 - blockIdx.x) / gridDim.x + 1 : 0;

    if (tid == 0) {
        for (int b = 0; b < W * kRowBufs; ++b) mbar_init(&full_bar[b], 1);
        abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&xmap);
    }
    for (int i = tid; i < G * G; i += blockDim.x) {
        const int n = i / G, k = i % G;
        *reinterpret_cast<T*>(rt_sh + rt_off<G>(n, k / 8) + (k % 8) * 2) = R[k * G + n];
    }
    __syncthreads();

    if (warp < W) {
        // ---------------------------------------------------------------- row warps
        // row i of this warp is this CTA's row warp + i W, in buffer i % 2
        auto issue = [&](int64_t i) {   // lane 0: start the copy of the warp's row i
            const int64_t j = warp + i * W;
            if (j >= my_rows) return;
            const int bi = warp * kRowBufs + (int)(i % kRowBufs);
            unsigned char* dst = bufs + (size_t)bi * p.buf_bytes;
            mbar_arrive_expect_tx(&full_bar[bi], p.box_bytes * (uint32_t)p.NB);
            const int32_t row = (int32_t)(blockIdx.x + j * gridDim.x);
            for (int bx = 0; bx < p.NB; ++bx)
                tma_load_3d(dst + (size_t)bx * p.GB * G * 2, &xmap, &full_bar[bi], 0, bx * p.GB, row);
        };
        if (lane == 0) {
            issue(0);
            issue(1);
        }
        const uint32_t rt_base = smem_u32(rt_sh);
        const int units = (int)(p.K / 16);             // 16-element quantize units per row
        int64_t i = 0;
        for (;; ++i) {
            const int64_t j = warp + i * W;
            if (j >= my_rows) break;
            const int bi = warp * kRowBufs + (int)(i % kRowBufs);
            if (!__all_sync(0xffffffffu, mbar_wait(&full_bar[bi], (uint32_t)(i / kRowBufs) & 1u,
                                                   &abort_flag, dev_status)))
                break;
            const int64_t row = blockIdx.x + j * gridDim.x;
            unsigned char* buf = bufs + (size_t)bi * p.buf_bytes;
            const uint32_t base = smem_u32(buf);

            // ---- rotation y^T = R^T x^T: R^T is the A operand (fragments in registers), eight
            // (G = 64) or sixteen (G = 16) group-rows of x the B operand; the fp32 results are
            // rounded to T and stored transposed (stmatrix.trans) over x in place
            // A fragments of R^T (rows c = output channel, columns i = input channel), reloaded
            // per row so that they are not live across the quantize pass
            uint32_t ra[MT][KT][4];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int kt = 0; kt < KT; ++kt)
                    ldmatrix_x4(ra[mt][kt], rt_base + rt_off<G>(16 * mt + (lane & 7) + ((lane >> 3) & 1) * 8,
                                                                2 * kt + (lane >> 4)));
            uint32_t m2 = 0u;
            for (int rho0 = 0; rho0 < p.GR; rho0 += kRowStep<G>) {
                if constexpr (G == 64) {
                    uint32_t bq[KT][2];
#pragma unroll
                    for (int kp = 0; kp < KT; kp += 2) {
                        uint32_t r4[4];
                        ldmatrix_x4(r4, base + swz_off<G>(rho0 + (lane & 7), 2 * kp + (lane >> 3)));
                        bq[kp][0] = r4[0];
                        bq[kp][1] = r4[1];
                        bq[kp + 1][0] = r4[2];
                        bq[kp + 1][1] = r4[3];
                    }
                    float acc[MT][4];
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
#pragma unroll
                    for (int kt = 0; kt < KT; ++kt)
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt) MmaOp<T>::run(acc[mt], ra[mt][kt], bq[kt][0], bq[kt][1]);
                    // this lane's group-rows rho0 + 2 (lane % 4) + {0, 1}: absmax mask per half
                    const int rr = rho0 + 2 * (lane & 3);
                    const uint32_t keep = (rr < p.GR ? 0x0000FFFFu : 0u) | (rr + 1 < p.GR ? 0xFFFF0000u : 0u);
#pragma unroll
                    for (int mt = 0; mt < MT; mt += 2) {
                        const uint32_t q0 = MmaOp<T>::pack(acc[mt][0], acc[mt][1]);
                        const uint32_t q1 = MmaOp<T>::pack(acc[mt][2], acc[mt][3]);
                        const uint32_t q2 = MmaOp<T>::pack(acc[mt + 1][0], acc[mt + 1][1]);
                        const uint32_t q3 = MmaOp<T>::pack(acc[mt + 1][2], acc[mt + 1][3]);
                        m2 = MmaOp<T>::absmax2(m2, q0 & keep);
                        m2 = MmaOp<T>::absmax2(m2, q1 & keep);
                        m2 = MmaOp<T>::absmax2(m2, q2 & keep);
                        m2 = MmaOp<T>::absmax2(m2, q3 & keep);
                        stmatrix_x4_trans(base + swz_off<G>(rho0 + (lane & 7), 2 * mt + (lane >> 3)),
                                          q0, q1, q2, q3);
                    }
                } else {
                    // G = 16: one ldmatrix.x4 gives the B fragments of two n-tiles (rows
                    // rho0..+7 and rho0+8..+15); the same lane addresses serve the store
                    const uint32_t addr =
                        base + swz_off<G>(rho0 + ((lane >> 4) << 3) + (lane & 7), (lane >> 3) & 1);
                    uint32_t r4[4];
                    ldmatrix_x4(r4, addr);
                    float acc[2][4];
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
                        MmaOp<T>::run(acc[nt], ra[0][0], r4[2 * nt], r4[2 * nt + 1]);
                    }
                    uint32_t q[2][2];
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        const int rr = rho0 + 8 * nt + 2 * (lane & 3);
                        const uint32_t keep =
                            (rr < p.GR ? 0x0000FFFFu : 0u) | (rr + 1 < p.GR ? 0xFFFF0000u : 0u);
                        q[nt][0] = MmaOp<T>::pack(acc[nt][0], acc[nt][1]);
                        q[nt][1] = MmaOp<T>::pack(acc[nt][2], acc[nt][3]);
                        m2 = MmaOp<T>::absmax2(m2, q[nt][0] & keep);
                        m2 = MmaOp<T>::absmax2(m2, q[nt][1] & keep);
                    }
                    stmatrix_x4_trans(addr, q[0][0], q[0][1], q[1][0], q[1][1]);
                }
            }
            // ---- row scale (every lane of the warp holds the row's absmax)
            const float2 mf = MmaOp<T>::unpack(m2);
            float mx = fmax_nan(mf.x, mf.y);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmax_nan(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const float sc = row_scale(mx, DYN ? nullptr : scale_in, p.qmax);
            if (lane == 0) scales[row] = sc;
            const RowDivisor dv(sc, p.qmax);
            __syncwarp();   // the warp's stmatrix results are visible to all its lanes

            // ---- quantize: 16 consecutive channels per lane step, 16-byte code stores
            int8_t* dst_row = codes + row * p.ldq;
            for (int u = lane; u < units; u += 32) {
                const int k = u * 16;
                const int rho = k / G, e = k - rho * G;
                const uint4 u0 = *reinterpret_cast<const uint4*>(buf + swz_off<G>(rho, e / 8));
                const uint4 u1 = *reinterpret_cast<const uint4*>(buf + swz_off<G>(rho, e / 8 + 1));
                const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
                uint32_t out[4];
                if (DYN) {
                    unsigned long long y2[8];
#pragma unroll
                    for (int h = 0; h < 8; ++h) y2[h] = MmaOp<T>::unpack2(w[h]);
                    quant16_dyn2(y2, dv, out);
                } else {
                    float y[16];
#pragma unroll
                    for (int h = 0; h < 8; ++h) {
                        const float2 a = MmaOp<T>::unpack(w[h]);
                        y[2 * h] = a.x;
                        y[2 * h + 1] = a.y;
                    }
                    quant16(y, dv, out);
                }
                int8_t* dst = dst_row + k;
                if (p.vec_codes) {
                    *reinterpret_cast<uint4*>(dst) = make_uint4(out[0], out[1], out[2], out[3]);
                } else {
#pragma unroll
                    for (int q = 0; q < 16; ++q) dst[q] = (int8_t)((out[q / 4] >> (8 * (q % 4))) & 0xFF);
                }
            }
            // the buffer is no longer read by this warp: refill it with row i + 2 (the proxy
            // fence orders this warp's shared-memory accesses before the async copy's writes)
            __syncwarp();
            if (lane == 0) {
                fence_proxy_async_smem();
                issue(i + kRowBufs);
            }
        }
        // after an expired wait, copies still in flight land before the CTA leaves
        if (lane == 0)
            for (int64_t k = i; k < i + kRowBufs; ++k)
                if (warp + k * W < my_rows)
                    mbar_wait(&full_bar[warp * kRowBufs + (int)(k % kRowBufs)],
                              (uint32_t)(k / kRowBufs) & 1u, nullptr, nullptr);
    }
    __syncthreads();
}

// Row kernel for bf16/fp16, g in {16, 64}: every row fits one buffer and at least four compute
// warps with two buffers each fit in shared memory.  Returns CK_ERR_UNSUPPORTED otherwise.
template <typename T, int G>
static ck_status launch_row(const void* x, int64_t M, int64_t K, int64_t sm, const void* R,
                            const float* scale_in, int8_t* codes, int64_t ldq, float* scales,
                            int qmax, int* dev_status, cudaStream_t stream,
                            CUtensorMapDataType tdt) {
    RqRowParams p;
    p.M = M;
    p.K = K;
    p.ldq = ldq;
    p.GR = (int)(K / G);
    if (p.GR <= 256) {
        p.GB = p.GR;
        p.NB = 1;
    } else {
        p.GB = 256;
        p.NB = (p.GR + 255) / 256;
    }
    const int64_t rows_alloc = std::max<int64_t>(((int64_t)p.GR + 15) / 16 * 16, (int64_t)p.GB * p.NB);
    const int64_t buf = (rows_alloc * G * 2 + 1023) / 1024 * 1024;
    const int64_t budget = 200 * 1024;
    const int64_t warps = budget / (buf * kRowBufs);
    if (warps < 4) return CK_ERR_UNSUPPORTED;
    p.W = (int)std::min<int64_t>(warps, kRowMaxWarps);
    p.buf_bytes = (uint32_t)buf;
    p.box_bytes = (uint32_t)(G * 2 * p.GB);
    p.vec_codes = (aligned(codes, 16) && ldq % 16 == 0) ? 1 : 0;
    p.qmax = qmax;

    CUtensorMap map;
    const uint64_t dims[3] = {(uint64_t)G, (uint64_t)p.GR, (uint64_t)M};
    const uint64_t strides[2] = {(uint64_t)G * 2, (uint64_t)sm * 2};
    const uint32_t box[3] = {(uint32_t)G, (uint32_t)p.GB, 1u};
    ck_status st = encode_tma(&map, tdt, 3, x, dims, strides, box,
                              G == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_32B);
    if (st != CK_OK) return st;

    const size_t smem = (size_t)p.W * kRowBufs * p.buf_bytes + 1024;
    const int grid = (int)(M < num_sms() ? M : num_sms());
    const int threads = p.W * 32;
    auto run = [&](auto kern) -> ck_status {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return CK_ERR_CUDA;
        kern<<<grid, threads, smem, stream>>>(map, static_cast<const T*>(R), scale_in, codes,
                                              scales, p, dev_status);
        return cudaGetLastError() == cudaSuccess ? CK_OK : CK_ERR_CUDA;
    };
    return scale_in ? run(rq_row_kernel<T, G, false>) : run(rq_row_kernel<T, G, true>);
}

// ===================================================================== tensor-core kernel (g = 64, 256)

// One persistent CTA per SM for g in {64, 256} with a row of at most 128 groups.  A tile is
// the RB rows (RB = floor(128 / (K / g))) whose group-rows fill the 128 lanes of a
// tcgen05.mma.kind::f16 chain: D[group-row, c] = sum_i x[group-row, i] R[i, c], M = 128,
// N = g, K = g (g / 16 instructions), fp32 in TMEM.
//   warp 0       TMA producer: per tile g / 64 boxes (64 channels x K/g groups x RB rows),
//                each into a 16 KB stage of a ring (128-byte swizzle)
//   warp 1       TMEM allocation and the MMA-issuing thread; R^T is the B operand, resident
//                in shared memory; kTcAcc<G> accumulators of g columns in flight
//   warps 2-17   kTcAcc<G> groups of warps; group k finishes the tiles i = k (mod kTcAcc<G>),
//                whose accumulator is k.  Each warp owns one TMEM lane quarter (its warp
//                index mod 4) and a column range of the accumulator: tcgen05.ld of the
//                lane's group-row, round to the dtype, row absmax through shared atomics and
//                a barrier of the group's warps, then the row scale and the codes in 16-byte
//                stores.  For g = 64 the rounded values stay in registers between the two
//                steps; for g = 256 (128 columns a warp) the accumulator is read twice.
template <int G> constexpr int kTcAcc = G == 64 ? 4 : 2;         // kTcAcc * G <= 512 columns
template <int G> constexpr int kTcXStages = G == 64 ? 6 : 5;     // 16 KB stages
constexpr int kTcEpiWarp0 = 2, kTcEpiWarps = 16;
constexpr int kTcThreads = (kTcEpiWarp0 + kTcEpiWarps) * 32;
constexpr int kTcSlots = 3;                // row-absmax slots per group: its j-th tile uses j % 3
constexpr uint32_t kTcStageBytes = 128 * 128;

template <int G>
constexpr size_t tc_smem_bytes() {
    return (size_t)kTcXStages<G> * kTcStageBytes + (size_t)G * G * 2 + 1024;
}

// R^T (B operand, K-major, 128-byte swizzle) in shared memory: K in atoms of 64 values, atom a
// holds the G rows n (output channel) of 128 bytes with K = 64a .. 64a + 63; the 16-byte chunk
// of row n is XOR-swizzled by n % 8.
template <int G>
__device__ __forceinline__ uint32_t tc_rt_off(int n, int k) {
    return (uint32_t)(k >> 6) * (uint32_t)(G * 128) + (uint32_t)n * 128u +
           (uint32_t)((((k & 63) >> 3) ^ (n & 7)) << 4) + (uint32_t)(k & 7) * 2u;
}

struct RqTcParams {
    int64_t M, K, ldq;
    int GR;            // group-rows per row (K / g), at most 128
    int RB;            // rows per tile, RB * GR <= 128 (1 for split rows)
    int L;             // split rows: group-rows per part
    int tiles;
    uint32_t box_bytes;
    uint32_t idesc;
    int vec_codes;
    int qmax;          // code grid [-qmax - 1, qmax]
    uint64_t seed, offset;   // packed stochastic output: the Philox key and counter offset
    int dependent;           // launched as the programmatic dependent of the kernel before it
};

template <typename T, bool DYN>
__device__ __forceinline__ void tc_quant_store(const uint32_t (&yp)[8], const RowDivisor& dv,
                                               const float* scale_in, int8_t* dst, bool vec) {
    uint32_t out[4];
    if (DYN) {
        unsigned long long y2[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) y2[k] = MmaOp<T>::unpack2(yp[k]);
        quant16_dyn2(y2, dv, out);
    } else {
        float y[16];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const float2 a = MmaOp<T>::unpack(yp[k]);
            y[2 * k] = a.x;
            y[2 * k + 1] = a.y;
        }
        quant16(y, dv, out);
    }
    if (vec) {
        *reinterpret_cast<uint4*>(dst) = make_uint4(out[0], out[1], out[2], out[3]);
    } else {
#pragma unroll
        for (int k = 0; k < 16; ++k) dst[k] = (int8_t)((out[k / 4] >> (8 * (k % 4))) & 0xFF);
    }
}

// Sixteen codes of one row packed two to a byte (even channel in the low nibble), 8 bytes at
// dst.  PK = 1: rounded half to even, the codes tc_quant_store writes.  PK = 2: stochastic,
// q = clamp(floor(fl(t + u)), -8, 7) with t = fl(y / s) and u = (r >> 8) 2^-24, r word 0 of
// Philox4x32-10 at counter (e, offset) under key seed, e = row K + channel (e0 the first
// channel's); a NaN t gives 0.
template <typename T, bool DYN, int PK>
__device__ __forceinline__ void tc_packed_store(const uint32_t (&yp)[8], const RowDivisor& dv,
                                                uint8_t* dst, bool vec, uint64_t e0,
                                                uint64_t seed, uint64_t offset) {
    uint32_t out[4];   // sixteen codes, four a word, first code lowest
    if constexpr (PK == 1) {
        if (DYN) {
            unsigned long long y2[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) y2[k] = MmaOp<T>::unpack2(yp[k]);
            quant16_dyn2(y2, dv, out);
        } else {
            float y[16];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const float2 a = MmaOp<T>::unpack(yp[k]);
                y[2 * k] = a.x;
                y[2 * k + 1] = a.y;
            }
            quant16(y, dv, out);
        }
    } else {
        const PhiloxRun ph(seed, offset);
        int q[16];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const float2 a = MmaOp<T>::unpack(yp[k]);
            const float y[2] = {a.x, a.y};
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float t = dv.fast ? quotient_fast(y[e], dv.s, dv.r) : __fdiv_rn(y[e], dv.s);
                const uint64_t el = e0 + (uint64_t)(2 * k + e);
                const uint32_t rnd = ph.word0(el);
                const float u = __uint2float_rn(rnd >> 8) * 0x1p-24f;   // exact
                float v = floorf(__fadd_rn(t, u));
                v = fminf(fmaxf(v, -8.0f), 7.0f);
                q[2 * k + e] = t != t ? 0 : (int)v;
            }
        }
#pragma unroll
        for (int w = 0; w < 4; ++w) out[w] = pack4_codes(q[4 * w], q[4 * w + 1], q[4 * w + 2], q[4 * w + 3]);
    }
    // four byte codes c0 .. c3 of a word -> the two bytes (c0 & 15) | c1 << 4, (c2 & 15) | c3 << 4
    uint32_t h[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const uint32_t n = out[w] & 0x0F0F0F0Fu;
        h[w] = __byte_perm(n | (n >> 4), 0u, 0x4420);   // bytes 0 and 2, upper half zero
    }
    const uint32_t lo = h[0] | (h[1] << 16), hi = h[2] | (h[3] << 16);
    if (vec) {
        *reinterpret_cast<uint2*>(dst) = make_uint2(lo, hi);
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            dst[k] = (uint8_t)(lo >> (8 * k));
            dst[4 + k] = (uint8_t)(hi >> (8 * k));
        }
    }
}

// RG = G: R is the g x g rotation.  RG = 16 < G = 64: rows of g = 16 groups viewed as 64-channel
// group-rows; each of the four 16-channel groups is its own MMA (M = 128, N = 16, K = 16) of
// the group's 16 channels against R^T, into its own 16 accumulator columns, so no group sees
// another group's values (an Inf stays within its group, as in the per-group rotation).
//
// P = 2 (G = 64 only): rows of 129 to 256 group-rows, one row per tile in two parts of L <= 128
// group-rows.  Part a is its own TMA box (64 channels x L groups of the row) and its own
// 64-column block a of the tile's accumulator (D[l, 64 a + c] for group-row a L + l), so a
// group's accumulator has 128 columns; the epilogue reads both blocks twice (row absmax, then
// the codes).
// PK = 0: INT8 codes; PK = 1, 2: codes packed two to a byte at `codes` (row pitch ldq bytes),
// rounded half to even (1) or stochastically (2) (tc_packed_store).
template <typename T, int G, bool DYN, int RG = G, int P = 1, int PK = 0>
__global__ void __launch_bounds__(kTcThreads, 1)
    rq_tc_kernel(const __grid_constant__ CUtensorMap xmap, const T* __restrict__ R,
                 const float* __restrict__ scale_in, int8_t* __restrict__ codes,
                 float* __restrict__ scales, RqTcParams p, int* dev_status) {
    static_assert(P == 1 || G == 64, "split rows only at G = 64");
    static_assert(PK == 0 || (P == 1 && (G == 64 || G == 256)), "packed codes: one-part tiles");
    constexpr int kAcc = kTcAcc<G>, kStages = kTcXStages<G>, kAtoms = P > 1 ? P : G / 64;
    constexpr int kAccCols = G * P;                 // TMEM columns of one accumulator
    constexpr int kGrpWarps = kTcEpiWarps / kAcc;   // 4 or 8
    constexpr int kCols = G / (kGrpWarps / 4);      // accumulator columns a warp finishes
    extern __shared__ __align__(1024) unsigned char tc_smem[];
    unsigned char* base = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(tc_smem) + 1023) & ~uintptr_t(1023));
    unsigned char* xring = base;
    unsigned char* rt = base + (size_t)kStages * kTcStageBytes;   // R^T, 1024-aligned
    __shared__ __align__(8) uint64_t x_full[kStages], x_empty[kStages];
    __shared__ __align__(8) uint64_t d_full[kAcc], d_empty[kAcc], amax_bar[kAcc], drain_bar;
    __shared__ unsigned int amax_sh[kAcc][kTcSlots][128];
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_flag;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int my_tiles = (int)blockIdx.x < p.tiles ? (p.tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    const int my_boxes = my_tiles * kAtoms;
    // box n of this CTA: atom n % kAtoms of its tile n / kAtoms, into stage n % kStages
    auto issue = [&](int n) {
        const int s = n % kStages, a = n % kAtoms;
        const int t = (int)blockIdx.x + (n / kAtoms) * (int)gridDim.x;
        if constexpr (P > 1) {   // part a of row t: groups a L .. a L + L - 1
            mbar_arrive_expect_tx(&x_full[s], p.box_bytes);
            tma_load_3d(xring + (size_t)s * kTcStageBytes, &xmap, &x_full[s], 0, a * p.L, t);
            return;
        }
        mbar_arrive_expect_tx(&x_full[s], p.box_bytes);
        tma_load_3d(xring + (size_t)s * kTcStageBytes, &xmap, &x_full[s], 64 * a, 0, t * p.RB);
    };

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&x_full[s], 1);
            mbar_init(&x_empty[s], 1);
        }
        for (int b = 0; b < kAcc; ++b) {
            mbar_init(&d_full[b], 1);
            mbar_init(&d_empty[b], kGrpWarps);   // the warps of group b
            mbar_init(&amax_bar[b], kGrpWarps);
        }
        mbar_init(&drain_bar, 1);
        abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&xmap);
        // the first ring's worth of boxes goes out at once (while the CTA stages R^T) unless
        // the kernel must first wait for the one before it
        if (!p.dependent)
            for (int n = 0; n < kStages && n < my_boxes; ++n) issue(n);
    }
    for (int i = tid; i < kAcc * kTcSlots * 128; i += kTcThreads) (&amax_sh[0][0][0])[i] = 0u;
    if (p.dependent) {
        // launched as the programmatic dependent of the kernel before it on the stream: what
        // is above is on-chip set-up; x and R may be that kernel's output, and the codes and
        // scales its input, so no global memory is touched before it has completed
        grid_dependency_wait();
        if (tid == 0)
            for (int n = 0; n < kStages && n < my_boxes; ++n) issue(n);
    }
    // R^T[n][k] = R[k][n] is the MMA's B operand (N = c), staged in 8 x 8 blocks: a thread
    // loads rows k0 .. k0 + 7 of R at columns n0 .. n0 + 7 (16 bytes each), transposes them in
    // registers and stores the 16-byte chunks of rows n0 .. n0 + 7 of R^T.  Consecutive
    // threads take consecutive k0, so a warp's stores cover distinct swizzled chunks.
    if constexpr (RG != G) {
        // R^T in the diagonal blocks (the only ones the MMAs read), zeros elsewhere
        for (int i = tid; i < G * G; i += kTcThreads) {
            const int n = i / G, k = i % G;
            const T v = (n / RG == k / RG) ? R[(k % RG) * RG + (n % RG)] : Elem<T>::from_f(0.f);
            *reinterpret_cast<T*>(rt + tc_rt_off<G>(n, k)) = v;
        }
    } else
    for (int blk = tid; blk < (G / 8) * (G / 8); blk += kTcThreads) {
        const int k0 = (blk % (G / 8)) * 8, n0 = (blk / (G / 8)) * 8;
        uint32_t a[8][4];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(R + (size_t)(k0 + r) * G + n0));
            a[r][0] = v.x;
            a[r][1] = v.y;
            a[r][2] = v.z;
            a[r][3] = v.w;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            // word w of row n0 + j: (R[k0 + 2w][n0 + j], R[k0 + 2w + 1][n0 + j])
            const uint32_t sel = (j & 1) ? 0x7632u : 0x5410u;
            const uint4 o = make_uint4(__byte_perm(a[0][j / 2], a[1][j / 2], sel),
                                       __byte_perm(a[2][j / 2], a[3][j / 2], sel),
                                       __byte_perm(a[4][j / 2], a[5][j / 2], sel),
                                       __byte_perm(a[6][j / 2], a[7][j / 2], sel));
            *reinterpret_cast<uint4*>(rt + tc_rt_off<G>(n0 + j, k0)) = o;
        }
    }
    fence_proxy_async_smem();   // R^T, written by threads, is read by the tensor core
    if (warp == 1) {
        tmem_alloc(&tmem_base_sh, kAcc * kAccCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_sh;
    // the linear's GEMM, launched as this kernel's dependent, may start its prologue now:
    // after every CTA holds its tensor memory, so a GEMM CTA that lands on the same SM
    // and waits for its columns never stands in the way of a CTA of this kernel
    grid_dependents_launch();

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        // The warp walks the ring together (a vote makes each wait's outcome uniform) and one
        // elected lane issues, so the copy operands are computed uniformly across the warp.
        const bool leader = elect_one();
        int issued = my_boxes < kStages ? my_boxes : kStages;
        for (; issued < my_boxes; ++issued) {
            const int s = issued % kStages, f = issued / kStages;
            if (!__all_sync(0xffffffffu, mbar_wait(&x_empty[s], (uint32_t)(f - 1) & 1u, &abort_flag,
                                                   dev_status)))
                break;
            if (leader) issue(issued);
            __syncwarp();
        }
        if (leader && abort_flag)
            for (int j = issued > kStages ? issued - kStages : 0; j < issued; ++j)
                mbar_wait(&x_full[j % kStages], (uint32_t)(j / kStages) & 1u, nullptr, nullptr);
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        // the same warp-wide walk; the elected lane issues every MMA and commit (a commit
        // tracks the MMAs of its own thread)
        const bool leader = elect_one();
        const uint64_t adesc0 = smem_desc_k_sw128(smem_u32(xring));
        const uint64_t bdesc0 = smem_desc_k_sw128(smem_u32(rt));
        bool ok = true;
        for (int i = 0; i < my_tiles && ok; ++i) {
            const int b = i % kAcc;
            if (i >= kAcc &&
                !__all_sync(0xffffffffu, mbar_wait(&d_empty[b], (uint32_t)((i / kAcc) - 1) & 1u,
                                                   &abort_flag, dev_status)))
                break;
            for (int a = 0; a < kAtoms; ++a) {
                const int n = i * kAtoms + a, s = n % kStages;
                if (!__all_sync(0xffffffffu, mbar_wait(&x_full[s], (uint32_t)(n / kStages) & 1u,
                                                       &abort_flag, dev_status))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t adesc = adesc0 + (uint64_t)(s * (kTcStageBytes >> 4));
                const uint64_t bdesc = bdesc0 + (uint64_t)((P > 1 ? 0 : a) * ((G * 128) >> 4));
                if (leader) {
                    if constexpr (RG != G) {
                        // group gi: A channels 16 gi .. (32 bytes in), B = R^T rows 16 gi ..
                        // (16 rows of 128 bytes = 128 units in) at the same channels, N = 16
                        constexpr uint32_t idesc16 = idesc_f16(128, RG, std::is_same<T, __nv_bfloat16>::value);
#pragma unroll
                        for (int gi = 0; gi < G / RG; ++gi)
                            tc_mma_f16(tmem_base + (uint32_t)(b * kAccCols + (P > 1 ? 64 * a : 0) + RG * gi),
                                       adesc + (uint64_t)(gi * 2),
                                       bdesc + (uint64_t)(gi * ((RG * 128) >> 4) + gi * 2), idesc16, 0u);
                    } else {
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)   // K = 16 (32 bytes) per instruction
                            tc_mma_f16(tmem_base + (uint32_t)(b * kAccCols + (P > 1 ? 64 * a : 0)),
                                       adesc + (uint64_t)(kk * 2), bdesc + (uint64_t)(kk * 2), p.idesc,
                                       ((P == 1 && a > 0) || kk > 0) ? 1u : 0u);
                    }
                    tc_commit(&x_empty[s]);
                }
                __syncwarp();
            }
            if (ok && leader) tc_commit(&d_full[b]);
            __syncwarp();
        }
        if (leader) {
            tc_commit(&drain_bar);
            mbar_wait(&drain_bar, 0, nullptr, dev_status);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- epilogue warps
      if constexpr (P > 1) {
        // one row per tile; lane l of the group holds group-rows l (block 0) and L + l (block 1)
        const int q = warp & 3;
        const int e = warp - kTcEpiWarp0;
        const int grp = e / kGrpWarps;
        const int l = q * 32 + lane;
        const uint32_t tacc = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(grp * kAccCols);
        const bool zeroer = q == 0;
        int slot = 0;
        for (int i = grp, j = 0; i < my_tiles; i += kAcc, ++j) {
            const int64_t row = (int64_t)blockIdx.x + (int64_t)i * gridDim.x;
            const bool row_ok = row < p.M;
            if (!__all_sync(0xffffffffu, mbar_wait(&d_full[grp], (uint32_t)j & 1u, &abort_flag,
                                                   dev_status)))
                break;
            tc_fence_after();
            // pass 1: round to T, fold |y| of the lane's valid group-rows into the row absmax
            uint32_t m2 = 0u;
#pragma unroll 1
            for (int a = 0; a < P; ++a) {
                const bool gr_ok = l < p.L && a * p.L + l < p.GR;
#pragma unroll 1
                for (int c = 0; c < 64; c += 32) {
                    uint32_t v[32];
                    tc_ld_32x32b_x32(tacc + (uint32_t)(64 * a + c), v);
                    tc_wait_ld();
                    if (gr_ok) {
#pragma unroll
                        for (int k = 0; k < 16; ++k)
                            m2 = MmaOp<T>::absmax2(
                                m2, MmaOp<T>::pack(__uint_as_float(v[2 * k]), __uint_as_float(v[2 * k + 1])));
                    }
                }
            }
            if (zeroer && lane == 0) amax_sh[grp][slot == 2 ? 0 : slot + 1][0] = 0u;
            const float2 mf = MmaOp<T>::unpack(m2);
            if (row_ok && l < p.L) atomicMax(&amax_sh[grp][slot][0], __float_as_uint(fmax_nan(mf.x, mf.y)));
            __syncwarp();
            if (lane == 0) mbar_arrive(&amax_bar[grp]);
            if (!__all_sync(0xffffffffu, mbar_wait(&amax_bar[grp], (uint32_t)j & 1u, &abort_flag,
                                                   dev_status)))
                break;
            const unsigned int amax_bits = amax_sh[grp][slot][0];
            slot = slot == 2 ? 0 : slot + 1;
            const float sc = row_scale(__uint_as_float(amax_bits), DYN ? nullptr : scale_in, p.qmax);
            const RowDivisor dv(sc, p.qmax);
            if (row_ok && l == 0) scales[row] = sc;
            // pass 2: the codes, 64 per valid group-row
#pragma unroll 1
            for (int a = 0; a < P; ++a) {
                const int gr = a * p.L + l;
                const bool gr_ok = row_ok && l < p.L && gr < p.GR;
                int8_t* dst = codes + row * p.ldq + (int64_t)gr * G;
#pragma unroll 1
                for (int c = 0; c < 64; c += 32) {
                    uint32_t v[32];
                    tc_ld_32x32b_x32(tacc + (uint32_t)(64 * a + c), v);
                    tc_wait_ld();
                    if (gr_ok) {
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            uint32_t y8[8];
#pragma unroll
                            for (int k = 0; k < 8; ++k)
                                y8[k] = MmaOp<T>::pack(__uint_as_float(v[16 * u + 2 * k]),
                                                       __uint_as_float(v[16 * u + 2 * k + 1]));
                            tc_quant_store<T, DYN>(y8, dv, scale_in, dst + c + 16 * u,
                                                   p.vec_codes != 0);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&d_empty[grp]);   // done reading the accumulator
        }
      } else {
        const int q = warp & 3;                          // TMEM lanes 32q .. 32q + 31
        const int e = warp - kTcEpiWarp0;
        const int grp = e / kGrpWarps;                   // tiles i = grp (mod kAcc), accumulator grp
        const int h = (e % kGrpWarps) >> 2;              // column range h * kCols .. + kCols
        const int L = q * 32 + lane;                     // the lane's group-row of the tile
        const bool valid = L < p.RB * p.GR;
        const int r = valid ? L / p.GR : 0, rho = valid ? L - r * p.GR : 0;
        const uint32_t tacc =
            tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(grp * kAccCols + h * kCols);
        const bool zeroer = q == 0 && h == 0;
        int slot = 0;
        for (int i = grp, j = 0; i < my_tiles; i += kAcc, ++j) {
            const int t = (int)blockIdx.x + i * (int)gridDim.x;
            const int64_t row = (int64_t)t * p.RB + r;
            const bool row_ok = valid && row < p.M;
            if (!__all_sync(0xffffffffu, mbar_wait(&d_full[grp], (uint32_t)j & 1u, &abort_flag,
                                                   dev_status)))
                break;
            tc_fence_after();
            // round to T (the rotation's result dtype) and fold |y| into the row absmax
            uint32_t yp[kCols == 64 ? 32 : 1];
            uint32_t m2 = 0u;
            if constexpr (kCols == 64) {
                uint32_t v[64];
                tc_ld_32x32b_x32(tacc, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
                tc_ld_32x32b_x32(tacc + 32u, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
                tc_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&d_empty[grp]);   // the accumulator is in registers
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    yp[k] = MmaOp<T>::pack(__uint_as_float(v[2 * k]), __uint_as_float(v[2 * k + 1]));
                    m2 = MmaOp<T>::absmax2(m2, yp[k]);
                }
            } else {
#pragma unroll 1
                for (int c = 0; c < kCols; c += 32) {
                    uint32_t v[32];
                    tc_ld_32x32b_x32(tacc + (uint32_t)c, v);
                    tc_wait_ld();
#pragma unroll
                    for (int k = 0; k < 16; ++k)
                        m2 = MmaOp<T>::absmax2(
                            m2, MmaOp<T>::pack(__uint_as_float(v[2 * k]), __uint_as_float(v[2 * k + 1])));
                }
            }
            // slot (j + 1) % 3 was read during tile j - 2, before any warp of the group arrived
            // for tile j - 1; it is next written by tile j + 1, after this warp arrives for j
            if (zeroer)
                for (int k = lane; k < p.RB; k += 32) amax_sh[grp][slot == 2 ? 0 : slot + 1][k] = 0u;
            const float2 mf = MmaOp<T>::unpack(m2);
            if (row_ok) atomicMax(&amax_sh[grp][slot][r], __float_as_uint(fmax_nan(mf.x, mf.y)));
            __syncwarp();
            if (lane == 0) mbar_arrive(&amax_bar[grp]);
            if (!__all_sync(0xffffffffu, mbar_wait(&amax_bar[grp], (uint32_t)j & 1u, &abort_flag,
                                                   dev_status)))
                break;
            const unsigned int amax_bits = amax_sh[grp][slot][r];
            slot = slot == 2 ? 0 : slot + 1;
            const float sc = row_scale(__uint_as_float(amax_bits), DYN ? nullptr : scale_in, p.qmax);
            const RowDivisor dv(sc, p.qmax);
            if (row_ok && rho == 0 && h == 0) scales[row] = sc;
            int8_t* dst = codes + row * p.ldq + rho * G + h * kCols;
            if constexpr (kCols == 64 && PK != 0) {
                if (row_ok) {
                    // channels rho G .. rho G + 63 of the row: 32 bytes of packed codes
                    uint8_t* pdst = reinterpret_cast<uint8_t*>(codes) + row * p.ldq + rho * (G / 2);
                    const uint64_t e0 = (uint64_t)row * (uint64_t)p.K + (uint64_t)(rho * G);
                    if constexpr (PK == 1) {
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            tc_packed_store<T, DYN, PK>(*reinterpret_cast<const uint32_t(*)[8]>(&yp[8 * u]),
                                                        dv, pdst + 8 * u, p.vec_codes != 0,
                                                        e0 + (uint64_t)(16 * u), p.seed, p.offset);
                    } else {
                        // one run of 16 draws at a time: unrolled, the four runs' Philox chains
                        // spill (216 us against 147 at the headline shape)
#pragma unroll 1
                        for (int u = 0; u < 4; ++u)
                            tc_packed_store<T, DYN, PK>(*reinterpret_cast<const uint32_t(*)[8]>(&yp[8 * u]),
                                                        dv, pdst + 8 * u, p.vec_codes != 0,
                                                        e0 + (uint64_t)(16 * u), p.seed, p.offset);
                    }
                }
            } else if constexpr (kCols == 64) {
                if (row_ok) {
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        tc_quant_store<T, DYN>(*reinterpret_cast<const uint32_t(*)[8]>(&yp[8 * u]),
                                               dv, scale_in, dst + 16 * u, p.vec_codes != 0);
                }
            } else {
#pragma unroll 1
                for (int c = 0; c < kCols; c += 32) {
                    uint32_t v[32];
                    tc_ld_32x32b_x32(tacc + (uint32_t)c, v);
                    tc_wait_ld();
                    if (row_ok) {
                        // packed codes: channel k0 of this chunk is byte k0 / 2 of the row
                        const int k0 = rho * G + h * kCols + c;
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            uint32_t y8[8];
#pragma unroll
                            for (int k = 0; k < 8; ++k)
                                y8[k] = MmaOp<T>::pack(__uint_as_float(v[16 * u + 2 * k]),
                                                       __uint_as_float(v[16 * u + 2 * k + 1]));
                            if constexpr (PK != 0)
                                tc_packed_store<T, DYN, PK>(
                                    y8, dv, reinterpret_cast<uint8_t*>(codes) + row * p.ldq + k0 / 2 + 8 * u,
                                    p.vec_codes != 0, (uint64_t)row * (uint64_t)p.K + (uint64_t)(k0 + 16 * u),
                                    p.seed, p.offset);
                            else
                                tc_quant_store<T, DYN>(y8, dv, scale_in, dst + c + 16 * u,
                                                       p.vec_codes != 0);
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&d_empty[grp]);   // done reading the accumulator
            }
        }
      }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kAcc * kAccCols);
    }
}

// Tensor-core kernel for bf16/fp16, g in {64, 256}, K / g <= 128 (P = 1), or g = 64 rows of
// 129 .. 128 P groups split in P parts.  Returns CK_ERR_UNSUPPORTED otherwise.
template <typename T, int G, int RG = G, int P = 1, int PK = 0>
static ck_status launch_tc(const void* x, int64_t M, int64_t K, int64_t sm, const void* R,
                           const float* scale_in, int8_t* codes, int64_t ldq, float* scales,
                           int qmax, int* dev_status, cudaStream_t stream,
                           CUtensorMapDataType tdt, uint64_t seed = 0, uint64_t offset = 0) {
    RqTcParams p;
    p.seed = seed;
    p.offset = offset;
    p.dependent = M <= 64 ? 1 : 0;   // see the launch below
    p.M = M;
    p.K = K;
    p.ldq = ldq;
    if (K % G != 0 || K / G < 1 || K / G > 128 * P || (P > 1 && K / G <= 128))
        return CK_ERR_UNSUPPORTED;
    p.GR = (int)(K / G);
    p.RB = P > 1 ? 1 : 128 / p.GR;
    p.L = P > 1 ? (p.GR + P - 1) / P : p.GR;
    const int64_t tiles = (M + p.RB - 1) / p.RB;
    if (tiles >= (1LL << 31) / p.RB) return CK_ERR_UNSUPPORTED;
    p.tiles = (int)tiles;
    p.box_bytes = (uint32_t)(p.RB * p.L * 128);
    p.idesc = idesc_f16(128, G, std::is_same<T, __nv_bfloat16>::value);
    // 16-byte code stores, or 8-byte packed stores
    p.vec_codes = PK == 0 ? ((aligned(codes, 16) && ldq % 16 == 0) ? 1 : 0)
                          : ((aligned(codes, 8) && ldq % 8 == 0) ? 1 : 0);
    p.qmax = qmax;

    // x as (channel within group, group, row); each box is 64 channels (128 bytes) of every
    // group of RB rows, fetched at channel offsets 0, 64, .. G - 64
    CUtensorMap map;
    const uint64_t dims[3] = {(uint64_t)G, (uint64_t)p.GR, (uint64_t)M};
    const uint64_t strides[2] = {(uint64_t)G * 2, (uint64_t)sm * 2};
    const uint32_t box[3] = {64u, (uint32_t)p.L, (uint32_t)p.RB};
    ck_status st = encode_tma(&map, tdt, 3, x, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != CK_OK) return st;

    const size_t smem = tc_smem_bytes<G>();
    const int grid = (int)(p.tiles < num_sms() ? p.tiles : num_sms());
    auto run = [&](auto kern) -> ck_status {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return CK_ERR_CUDA;
        // few rows (M <= 64): the programmatic dependent of the kernel before it (the kernel
        // waits for it before touching global memory), so that its CTAs set up on the SMs that
        // kernel has already left; with many rows that launch measured slower (126.5 -> 129.5
        // us a headline step) and the launch is an ordinary one
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.gridDim = dim3((unsigned)grid, 1, 1);
        cfg.blockDim = dim3(kTcThreads, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = stream;
        cfg.attrs = attr;
        cfg.numAttrs = p.dependent ? 1 : 0;
        if (cudaLaunchKernelEx(&cfg, kern, map, static_cast<const T*>(R), scale_in, codes, scales,
                               p, dev_status) != cudaSuccess)
            return CK_ERR_CUDA;
        return cudaGetLastError() == cudaSuccess ? CK_OK : CK_ERR_CUDA;
    };
    return scale_in ? run(rq_tc_kernel<T, G, false, RG, P, PK>)
                    : run(rq_tc_kernel<T, G, true, RG, P, PK>);
}

// The packed quantizer on the tensor-core kernel: bf16/fp16 rows of unit stride with g = 16 or
// 64 and at most 128 64-channel group-rows, or g = 256 and at most 128 groups;
// CK_ERR_UNSUPPORTED otherwise.
ck_status launch_rotate_quant_packed_tc(const void* x, ck_dtype dt, int64_t M, int64_t K,
                                        int64_t sm, int64_t sk, const void* R, int g,
                                        const float* scale_in, bool stochastic, uint64_t seed,
                                        uint64_t offset, uint8_t* packed, int64_t ldp,
                                        float* scales, cudaStream_t stream) {
    const bool half16 = dt == CK_BF16 || dt == CK_F16;
    if (!half16 || (g != 16 && g != 64 && g != 256) || sk != 1 || !aligned(x, 16) ||
        !aligned(R, 16) || sm % 8 != 0 || sm <= 0 || K % 64 != 0 || K / 64 > 128 ||
        (g == 256 && (K % 256 != 0 || K / 256 > 128)) || M >= (1LL << 31))
        return CK_ERR_UNSUPPORTED;
    const bool bf = dt == CK_BF16;
    const CUtensorMapDataType tdt = bf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    int8_t* out = reinterpret_cast<int8_t*>(packed);
#define CK_RQP_ARGS x, M, K, sm, R, scale_in, out, ldp, scales, 7, nullptr, stream, tdt, seed, offset
    if (g == 256) {
        if (bf)
            return stochastic ? launch_tc<__nv_bfloat16, 256, 256, 1, 2>(CK_RQP_ARGS)
                              : launch_tc<__nv_bfloat16, 256, 256, 1, 1>(CK_RQP_ARGS);
        return stochastic ? launch_tc<__half, 256, 256, 1, 2>(CK_RQP_ARGS)
                          : launch_tc<__half, 256, 256, 1, 1>(CK_RQP_ARGS);
    }
    if (g == 64) {
        if (bf)
            return stochastic ? launch_tc<__nv_bfloat16, 64, 64, 1, 2>(CK_RQP_ARGS)
                              : launch_tc<__nv_bfloat16, 64, 64, 1, 1>(CK_RQP_ARGS);
        return stochastic ? launch_tc<__half, 64, 64, 1, 2>(CK_RQP_ARGS)
                          : launch_tc<__half, 64, 64, 1, 1>(CK_RQP_ARGS);
    }
    if (bf)
        return stochastic ? launch_tc<__nv_bfloat16, 64, 16, 1, 2>(CK_RQP_ARGS)
                          : launch_tc<__nv_bfloat16, 64, 16, 1, 1>(CK_RQP_ARGS);
    return stochastic ? launch_tc<__half, 64, 16, 1, 2>(CK_RQP_ARGS)
                      : launch_tc<__half, 64, 16, 1, 1>(CK_RQP_ARGS);
#undef CK_RQP_ARGS
}

// ===================================================================== host launch

template <typename T, int G>
static ck_status launch_mma(const void* x, int64_t M, int64_t K, int64_t sm, const void* R,
                            const float* scale_in, int8_t* codes, int64_t ldq, float* scales,
                            int qmax, int* dev_status, cudaStream_t stream,
                            CUtensorMapDataType tdt) {
    RqMmaParams p;
    p.M = M;
    p.K = K;
    p.ldq = ldq;
    p.Gn = (int)(K / G);
    p.NB = (p.Gn + 255) / 256;
    p.GB = (p.Gn + p.NB - 1) / p.NB;
    const int sms = num_sms();
    auto stride_for = [&](int rb) {
        const uint32_t tile_rows = (uint32_t)(((rb * p.GB) + 15) / 16 * 16);
        return (tile_rows * G * 2 + 1023u) & ~1023u;
    };
    // rows per block: a stage of about 32 KB, and at least 4 blocks per CTA
    int RB = 16;
    while (RB > 1 && (size_t)stride_for(RB) * p.NB > 36 * 1024) RB >>= 1;
    while (RB > 1 && (M + RB - 1) / RB < 4LL * sms) RB >>= 1;
    p.RB = RB;
    p.box_bytes = (uint32_t)(RB * p.GB * G * 2);
    p.box_stride = stride_for(RB);
    p.stage_bytes = p.box_stride * (uint32_t)p.NB;
    // ring depth: as many stages as fit in about 190 KB
    p.S = (int)((190u * 1024u) / p.stage_bytes);
    if (p.S > kRqMaxStages) p.S = kRqMaxStages;
    if (p.S < 2) return CK_ERR_UNSUPPORTED;
    p.vec_codes = (aligned(codes, 16) && ldq % 16 == 0) ? 1 : 0;
    p.qmax = qmax;

    CUtensorMap map;
    const uint64_t dims[3] = {(uint64_t)G, (uint64_t)p.Gn, (uint64_t)M};
    const uint64_t strides[2] = {(uint64_t)G * 2, (uint64_t)sm * 2};
    const uint32_t box[3] = {(uint32_t)G, (uint32_t)p.GB, (uint32_t)RB};
    ck_status st = encode_tma(&map, tdt, 3, x, dims, strides, box,
                              G == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_32B);
    if (st != CK_OK) return st;

    const size_t smem = (size_t)p.S * p.stage_bytes + 1024;
    auto kern = rq_mma_kernel<T, G>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return CK_ERR_CUDA;
    const int64_t n_blocks = (M + RB - 1) / RB;
    const int grid = (int)(n_blocks < sms ? n_blocks : sms);
    kern<<<grid, kRqThreads, smem, stream>>>(map, static_cast<const T*>(R), scale_in, codes,
                                             scales, p, dev_status);
    return cudaGetLastError() == cudaSuccess ? CK_OK : CK_ERR_CUDA;
}

template <typename T>
static ck_status launch_generic(const void* x, int64_t M, int64_t K, int64_t sm, int64_t sk,
                                const void* R, int g, const float* scale_in, int8_t* codes,
                                int64_t ldq, float* scales, int qmax, cudaStream_t stream) {
    const size_t r_bytes = (size_t)g * g * sizeof(T);
    const size_t xs_bytes = (size_t)K * sizeof(float);
    const int r_in_smem = (xs_bytes + r_bytes <= 200 * 1024) ? 1 : 0;
    const size_t smem = xs_bytes + (r_in_smem ? r_bytes : 0);
    if (smem > 220 * 1024) return CK_ERR_UNSUPPORTED;
    const int vec = (aligned(codes, 4) && ldq % 4 == 0) ? 1 : 0;
    const int grid = (int)(M < 4LL * num_sms() ? M : 4LL * num_sms());
    const bool keep = K <= (int64_t)kGenThreads * 4 * kGenMaxChunks;
    if (keep) {
        auto kern = rq_generic_kernel<T, true>;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return CK_ERR_CUDA;
        kern<<<grid, kGenThreads, smem, stream>>>(static_cast<const T*>(x), M, K, sm, sk,
                                                  static_cast<const T*>(R), g, r_in_smem,
                                                  scale_in, codes, ldq, scales, vec, qmax);
    } else {
        auto kern = rq_generic_kernel<T, false>;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return CK_ERR_CUDA;
        kern<<<grid, kGenThreads, smem, stream>>>(static_cast<const T*>(x), M, K, sm, sk,
                                                  static_cast<const T*>(R), g, r_in_smem,
                                                  scale_in, codes, ldq, scales, vec, qmax);
    }
    return cudaGetLastError() == cudaSuccess ? CK_OK : CK_ERR_CUDA;
}

ck_status launch_rotate_quant(const void* x, ck_dtype dt, int64_t M, int64_t K, int64_t sm,
                              int64_t sk, const void* R, int g, const float* scale_in,
                              int8_t* codes, int64_t ldq, float* scales, int qmax,
                              int* dev_status, cudaStream_t stream) {
    if (M == 0) return CK_OK;
    const bool half16 = dt == CK_BF16 || dt == CK_F16;
    const bool mma_ok = half16 && (g == 16 || g == 64) && sk == 1 && aligned(x, 16) && sm % 8 == 0 &&
                        sm > 0 && M < (1LL << 31) && K / g <= (1LL << 31);
    const bool tc_ok = half16 && (g == 64 || g == 256) && sk == 1 && aligned(x, 16) &&
                       aligned(R, 16) && sm % 8 == 0 && sm > 0 && M < (1LL << 31);
    const bool bf = dt == CK_BF16;
    const CUtensorMapDataType tdt = bf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
#define CK_RQ_ARGS x, M, K, sm, R, scale_in, codes, ldq, scales, qmax, dev_status, stream, tdt
    if (tc_ok) {
        ck_status st;
        if (bf)
            st = g == 64 ? launch_tc<__nv_bfloat16, 64>(CK_RQ_ARGS) : launch_tc<__nv_bfloat16, 256>(CK_RQ_ARGS);
        else
            st = g == 64 ? launch_tc<__half, 64>(CK_RQ_ARGS) : launch_tc<__half, 256>(CK_RQ_ARGS);
        if (st != CK_ERR_UNSUPPORTED) return st;
        if (g == 64) {   // rows of 129 to 256 groups, in two parts
            st = bf ? launch_tc<__nv_bfloat16, 64, 64, 2>(CK_RQ_ARGS) : launch_tc<__half, 64, 64, 2>(CK_RQ_ARGS);
            if (st != CK_ERR_UNSUPPORTED) return st;
        }
    }
    // g = 16 rows of whole 64-channel groups: the tensor-core kernel with a block-diagonal R
    const bool tc16_ok = half16 && g == 16 && K % 64 == 0 && sk == 1 && aligned(x, 16) &&
                         sm % 8 == 0 && sm > 0 && M < (1LL << 31);
    if (tc16_ok) {
        ck_status st = bf ? launch_tc<__nv_bfloat16, 64, 16>(CK_RQ_ARGS)
                          : launch_tc<__half, 64, 16>(CK_RQ_ARGS);
        if (st != CK_ERR_UNSUPPORTED) return st;
        st = bf ? launch_tc<__nv_bfloat16, 64, 16, 2>(CK_RQ_ARGS) : launch_tc<__half, 64, 16, 2>(CK_RQ_ARGS);
        if (st != CK_ERR_UNSUPPORTED) return st;
    }
    if (mma_ok) {
        ck_status st;
        if (bf)
            st = g == 64 ? launch_row<__nv_bfloat16, 64>(CK_RQ_ARGS) : launch_row<__nv_bfloat16, 16>(CK_RQ_ARGS);
        else
            st = g == 64 ? launch_row<__half, 64>(CK_RQ_ARGS) : launch_row<__half, 16>(CK_RQ_ARGS);
        if (st != CK_ERR_UNSUPPORTED) return st;
        if (bf)
            return g == 64 ? launch_mma<__nv_bfloat16, 64>(CK_RQ_ARGS) : launch_mma<__nv_bfloat16, 16>(CK_RQ_ARGS);
        return g == 64 ? launch_mma<__half, 64>(CK_RQ_ARGS) : launch_mma<__half, 16>(CK_RQ_ARGS);
    }
#undef CK_RQ_ARGS
    if (dt == CK_F32 && (g == 64 || g == 256)) {
        const ck_status st = launch_rq_f32_wide(x, M, K, sm, sk, R, g, scale_in, codes, ldq,
                                                scales, qmax, dev_status, stream);
        if (st != CK_ERR_UNSUPPORTED) return st;
    }
    if (dt == CK_F32 && g == 16) {
        const ck_status st = launch_rq_f32_g16(x, M, K, sm, sk, R, scale_in, codes, ldq, scales,
                                               qmax, dev_status, stream);
        if (st != CK_ERR_UNSUPPORTED) return st;
    }
    switch (dt) {
        case CK_F32:
            return launch_generic<float>(x, M, K, sm, sk, R, g, scale_in, codes, ldq, scales, qmax, stream);
        case CK_F16:
            return launch_generic<__half>(x, M, K, sm, sk, R, g, scale_in, codes, ldq, scales, qmax, stream);
        case CK_BF16:
            return launch_generic<__nv_bfloat16>(x, M, K, sm, sk, R, g, scale_in, codes, ldq, scales,
                                                 qmax, stream);
        default:
            return CK_ERR_INVALID_ARG;
    }
}

}  // namespace ck
