// ck_rq_tf32.cu -- stage 1 for fp32 activations with g = 64 on the tensor cores: the group-wise
// rotation formed from four TF32 products per term (split TF32), the row-wise scale and the
// INT8-stored codes.
//
// Operation (comfy-kitchen PR #198 "Consolidate INT8, RotateQuant, RoPE and ConvRot W4A4
// backends", "W4A4 correctness and performance scope": the rotation keeps the FP32 input dtype;
// PR #155 "Add fused RotateQuant backend": group sizes 16/64/256):
//   y[m, 64 j + c] = sum_i x[m, 64 j + i] R[i, c]                   (fp32 accuracy)
//   s[m] = max(fp32(max_k |y[m, k]|) / qmax, FLT_MIN)              (or the caller's scale)
//   q[m, k] = clamp(round_half_even(y[m, k] / s[m]), -qmax - 1, qmax)
//
// Split TF32.  A TF32 MMA reads the top 19 bits of each fp32 operand (sign, exponent, 10
// mantissa bits): t(v), v with its low 13 bits cleared.  x splits exactly into three values
// that a TF32 read keeps whole, hi = t(x) (x as stored), mid = t(x - hi) and lo = x - hi - mid
// (at most 2 significant bits left), and R into Rhi = t(R) (R as stored) and Rlo = R - t(R):
//   x R ~ hi Rhi + hi Rlo + mid Rhi + lo Rhi,
// every product exact in the fp32 accumulator's terms; what is dropped (mid Rlo, lo Rlo and the
// low bits of Rlo that a TF32 read clears) is below 2^-20 |x| |R|, and an R whose entries TF32
// holds exactly (an identity, a Hadamard matrix) gives hi + mid + lo = x itself.  A +-inf x is
// moved whole into mid (hi = 0), so that inf meets R only through mid Rhi: inf R[i][c], NaN
// where R is 0, as in the exact rotation.
//
// One CTA per SM, persistent over tiles of RB rows (RB K / 64 <= 128 group-rows, one 64-channel
// group per TMEM lane), or of one row in two parts of L <= 128 group-rows (P = 2, K / 64 up to
// 256), each part its own 64-column block of the accumulator:
//   warp 0      TMA of x: per tile and part, two boxes of 32 channels (128 bytes, 128-byte
//               swizzle) of every group, into a ring of 16 KB stages
//   warps 2-5   the split: mid and lo of each stage into two twin stages (and +-inf moved out
//               of hi); four warps, so that the split keeps pace with the copies and the MMAs
//   warp 1      TMEM and the MMAs: per 8 values of i, tcgen05.mma kind::tf32 of hi Rhi, hi Rlo,
//               mid Rhi and lo Rhi (M = 128 group-rows, N = 64 channels), R^T (hi and lo)
//               resident in shared memory; the whole warp walks the ring, one elected lane
//               issues
//   warps 6-21  four groups of four epilogue warps (four tiles in flight): read the fp32
//               accumulator twice from TMEM, the row absmax through shared atomics and a group
//               barrier, the scale, the codes in 16-byte stores
// Every wait is bounded; a timeout records CK_ERR_TIMEOUT and the kernel drains and returns.
#include <cuda.h>
#include <float.h>
#include <stdint.h>

#include "ck_device.cuh"
#include "ck_internal.h"

namespace ck {

namespace rqtf {
constexpr int kWarpTma = 0, kWarpMma = 1, kWarpSplit0 = 2, kSplitWarps = 4;
constexpr int kEpiWarp0 = 6, kEpiWarps = 16, kGrpWarps = 4;
constexpr int kThreads = (kEpiWarp0 + kEpiWarps) * 32;
constexpr int kAcc = kEpiWarps / kGrpWarps;       // tiles in flight
constexpr int kStages = 3;                        // 16 KB x stages (and as many mid and lo)
constexpr uint32_t kStageBytes = 128 * 128;
constexpr uint32_t kRtBytes = 64 * 64 * 4;        // R^T, two K-atoms of 32 values
constexpr int kSlots = 3;                         // row-absmax slots per group
constexpr size_t kSmem = 3 * (size_t)kStages * kStageBytes + 2 * (size_t)kRtBytes + 1024;
}  // namespace rqtf

struct RqTf32Params {
    int64_t M, K, ldq;
    int GR;            // group-rows per row (K / 64)
    int RB;            // rows per tile (1 for split rows)
    int L;             // group-rows per part (GR, or ceil(GR / 2) for split rows)
    int tiles;
    uint32_t box_bytes;
    uint32_t idesc;
    int vec_codes;
    int qmax;
};

// Instruction descriptor for tcgen05.mma kind::tf32, fp32 accumulator, A and B K-major:
// [4,6) D format (1 = f32), [7,10) A format (2 = tf32), [10,13) B format, [17,23) N >> 3,
// [24,29) M >> 4.
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N) {
    return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]^T, tf32 inputs, fp32 accumulator, one CTA; K = 8 a step.
__device__ __forceinline__ void tc_mma_tf32(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// x with the 13 low mantissa bits cleared: the value a TF32 read sees.
__device__ __forceinline__ float tf32_trunc(float v) {
    return __uint_as_float(__float_as_uint(v) & 0xFFFFE000u);
}

// Byte offset of R^T[n][k] (n: output channel, k: input channel) in a K-major, 128-byte
// swizzled B operand of two K-atoms of 32 values: atom k / 32 holds 64 rows n of 128 bytes,
// whose 16-byte chunks are XOR-swizzled by n % 8.
__device__ __forceinline__ uint32_t tf_rt_off(int n, int k) {
    return (uint32_t)(k >> 5) * 8192u + (uint32_t)n * 128u +
           (uint32_t)((((k & 31) >> 2) ^ (n & 7)) << 4) + (uint32_t)(k & 3) * 4u;
}

template <bool DYN, int P>
__global__ void __launch_bounds__(rqtf::kThreads, 1)
    rq_tf32_kernel(const __grid_constant__ CUtensorMap xmap, const float* __restrict__ R,
                   const float* __restrict__ scale_in, int8_t* __restrict__ codes,
                   float* __restrict__ scales, RqTf32Params p, int* dev_status) {
    using namespace rqtf;
    constexpr int kAtoms = 2 * P;                   // (part, channel half) boxes per tile
    constexpr int kAccCols = 64 * P;
    extern __shared__ __align__(1024) unsigned char tf_smem[];
    unsigned char* base = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(tf_smem) + 1023) & ~uintptr_t(1023));
    unsigned char* xring = base;                                          // hi (x) stages
    unsigned char* mring = base + (size_t)kStages * kStageBytes;          // mid stages
    unsigned char* lring = base + 2 * (size_t)kStages * kStageBytes;      // lo stages
    unsigned char* rt_hi = base + 3 * (size_t)kStages * kStageBytes;      // R^T, 1024-aligned
    unsigned char* rt_lo = rt_hi + kRtBytes;
    __shared__ __align__(8) uint64_t x_full[kStages], l_full[kStages], x_empty[kStages];
    __shared__ __align__(8) uint64_t d_full[kAcc], d_empty[kAcc], amax_bar[kAcc], drain_bar;
    __shared__ unsigned int amax_sh[kAcc][kSlots][128];
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_flag;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int my_tiles = (int)blockIdx.x < p.tiles ? (p.tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    const int my_boxes = my_tiles * kAtoms;
    // box n of this CTA: atom n % kAtoms (part a / 2, channels 32 (a % 2) ..) of its tile n / kAtoms
    auto issue = [&](int n) {
        const int s = n % kStages, a = n % kAtoms;
        const int t = (int)blockIdx.x + (n / kAtoms) * (int)gridDim.x;
        mbar_arrive_expect_tx(&x_full[s], p.box_bytes);
        tma_load_3d(xring + (size_t)s * kStageBytes, &xmap, &x_full[s], 32 * (a & 1),
                    (a >> 1) * p.L, t * p.RB);
    };

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&x_full[s], 1);
            mbar_init(&l_full[s], kSplitWarps);
            mbar_init(&x_empty[s], 1);
        }
        for (int b = 0; b < kAcc; ++b) {
            mbar_init(&d_full[b], 1);
            mbar_init(&d_empty[b], kGrpWarps);
            mbar_init(&amax_bar[b], kGrpWarps);
        }
        mbar_init(&drain_bar, 1);
        abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&xmap);
        for (int n = 0; n < kStages && n < my_boxes; ++n) issue(n);
    }
    for (int i = tid; i < kAcc * kSlots * 128; i += kThreads) (&amax_sh[0][0][0])[i] = 0u;
    // R^T hi and lo: element (n, k) is R[k][n]
    for (int i = tid; i < 64 * 64; i += kThreads) {
        const int k = i >> 6, n = i & 63;
        const float r = R[i];
        const float rh = tf32_trunc(r);
        const float rl = __fsub_rn(r, rh);
        *reinterpret_cast<float*>(rt_hi + tf_rt_off(n, k)) = r;
        *reinterpret_cast<float*>(rt_lo + tf_rt_off(n, k)) = rl;
    }
    fence_proxy_async_smem();
    if (warp == kWarpMma) {
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

    if (warp == kWarpTma) {
        // ---------------------------------------------------------------- TMA producer
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
    } else if (warp >= kWarpSplit0 && warp < kWarpSplit0 + kSplitWarps) {
        // ---------------------------------------------------------------- split
        // mid and lo stages s from x element by element (the stages share one layout); a +-inf
        // x goes whole into mid and leaves 0 in hi
        const int st = (warp - kWarpSplit0) * 32 + lane;   // 0 .. 32 kSplitWarps - 1
        for (int n = 0; n < my_boxes; ++n) {
            const int s = n % kStages;
            if (!__all_sync(0xffffffffu, mbar_wait(&x_full[s], (uint32_t)(n / kStages) & 1u,
                                                   &abort_flag, dev_status)))
                break;
            float4* xs = reinterpret_cast<float4*>(xring + (size_t)s * kStageBytes);
            float4* ms = reinterpret_cast<float4*>(mring + (size_t)s * kStageBytes);
            float4* ls = reinterpret_cast<float4*>(lring + (size_t)s * kStageBytes);
            // v = hi + mid + lo exactly: r = v - t(v), mid = t(r), lo = r - mid
            auto split3 = [](float v, float& m, float& l) {
                const float r = __fsub_rn(v, tf32_trunc(v));
                m = tf32_trunc(r);
                l = __fsub_rn(r, m);
            };
#pragma unroll 4
            for (int i = st; i < (int)(kStageBytes / 16); i += 32 * kSplitWarps) {
                float4 v = xs[i];
                float4 m, l;
                split3(v.x, m.x, l.x);
                split3(v.y, m.y, l.y);
                split3(v.z, m.z, l.z);
                split3(v.w, m.w, l.w);
                const bool ix = isinf(v.x), iy = isinf(v.y), iz = isinf(v.z), iw = isinf(v.w);
                if (ix | iy | iz | iw) {
                    if (ix) { m.x = v.x; l.x = 0.f; v.x = 0.f; }
                    if (iy) { m.y = v.y; l.y = 0.f; v.y = 0.f; }
                    if (iz) { m.z = v.z; l.z = 0.f; v.z = 0.f; }
                    if (iw) { m.w = v.w; l.w = 0.f; v.w = 0.f; }
                    xs[i] = v;
                }
                ms[i] = m;
                ls[i] = l;
            }
            fence_proxy_async_smem();   // the mid and lo stages (and hi edits) feed the tensor core
            __syncwarp();
            if (lane == 0) mbar_arrive(&l_full[s]);
        }
    } else if (warp == kWarpMma) {
        // ---------------------------------------------------------------- MMA issuer
        const bool leader = elect_one();
        const uint64_t xdesc0 = smem_desc_k_sw128(smem_u32(xring));
        const uint64_t mdesc0 = smem_desc_k_sw128(smem_u32(mring));
        const uint64_t ldesc0 = smem_desc_k_sw128(smem_u32(lring));
        const uint64_t bh0 = smem_desc_k_sw128(smem_u32(rt_hi));
        const uint64_t bl0 = smem_desc_k_sw128(smem_u32(rt_lo));
        bool ok = true;
        for (int i = 0; i < my_tiles && ok; ++i) {
            const int b = i % kAcc;
            if (i >= kAcc &&
                !__all_sync(0xffffffffu, mbar_wait(&d_empty[b], (uint32_t)((i / kAcc) - 1) & 1u,
                                                   &abort_flag, dev_status)))
                break;
            for (int a = 0; a < kAtoms; ++a) {
                const int n = i * kAtoms + a, s = n % kStages;
                const uint32_t par = (uint32_t)(n / kStages) & 1u;
                if (!__all_sync(0xffffffffu, mbar_wait(&x_full[s], par, &abort_flag, dev_status)) ||
                    !__all_sync(0xffffffffu, mbar_wait(&l_full[s], par, &abort_flag, dev_status))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t ah = xdesc0 + (uint64_t)(s * (kStageBytes >> 4));
                const uint64_t am = mdesc0 + (uint64_t)(s * (kStageBytes >> 4));
                const uint64_t al = ldesc0 + (uint64_t)(s * (kStageBytes >> 4));
                const uint64_t bh = bh0 + (uint64_t)((a & 1) * (8192 >> 4));
                const uint64_t bl = bl0 + (uint64_t)((a & 1) * (8192 >> 4));
                const uint32_t d = tmem_base + (uint32_t)(b * kAccCols + 64 * (a >> 1));
                if (leader) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {   // K = 8 (32 bytes) per instruction
                        const uint32_t acc = ((a & 1) | kk) != 0 ? 1u : 0u;
                        tc_mma_tf32(d, ah + (uint64_t)(kk * 2), bh + (uint64_t)(kk * 2), p.idesc, acc);
                        tc_mma_tf32(d, ah + (uint64_t)(kk * 2), bl + (uint64_t)(kk * 2), p.idesc, 1u);
                        tc_mma_tf32(d, am + (uint64_t)(kk * 2), bh + (uint64_t)(kk * 2), p.idesc, 1u);
                        tc_mma_tf32(d, al + (uint64_t)(kk * 2), bh + (uint64_t)(kk * 2), p.idesc, 1u);
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
        const int q = warp & 3;                          // TMEM lanes 32 q .. 32 q + 31
        const int grp = (warp - kEpiWarp0) / kGrpWarps;  // tiles i = grp (mod kAcc)
        const int l = q * 32 + lane;                     // the lane's group-row of the part
        // P = 1: lane l is group-row rho of row r of the tile; P = 2: group-rows l and L + l of
        // the tile's one row
        const bool lane_ok = P > 1 ? l < p.L : l < p.RB * p.GR;
        const int r = (P == 1 && lane_ok) ? l / p.GR : 0;
        const int rho = (P == 1 && lane_ok) ? l - r * p.GR : l;
        const uint32_t tacc = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(grp * kAccCols);
        int slot = 0;
        for (int i = grp, j = 0; i < my_tiles; i += kAcc, ++j) {
            const int t = (int)blockIdx.x + i * (int)gridDim.x;
            const int64_t row = (int64_t)t * p.RB + r;
            const bool row_ok = lane_ok && row < p.M;
            if (!__all_sync(0xffffffffu, mbar_wait(&d_full[grp], (uint32_t)j & 1u, &abort_flag,
                                                   dev_status)))
                break;
            tc_fence_after();
            // pass 1: |y| of the lane's valid group-rows into the row absmax
            float mx = 0.f;
#pragma unroll 1
            for (int a = 0; a < P; ++a) {
                const bool gr_ok = row_ok && (P == 1 || a * p.L + l < p.GR);
#pragma unroll 1
                for (int c = 0; c < 64; c += 32) {
                    uint32_t v[32];
                    tc_ld_32x32b_x32(tacc + (uint32_t)(64 * a + c), v);
                    tc_wait_ld();
                    if (gr_ok) {
#pragma unroll
                        for (int k = 0; k < 32; ++k) mx = fmax_nan(mx, fabsf(__uint_as_float(v[k])));
                    }
                }
            }
            // slot (j + 1) % 3 was read during tile j - 2, before any warp of the group arrived
            // for tile j - 1; it is next written by tile j + 1, after this warp arrives for j
            if (q == 0)
                for (int k = lane; k < p.RB; k += 32) amax_sh[grp][slot == 2 ? 0 : slot + 1][k] = 0u;
            if (row_ok) atomicMax(&amax_sh[grp][slot][r], __float_as_uint(mx));
            __syncwarp();
            if (lane == 0) mbar_arrive(&amax_bar[grp]);
            if (!__all_sync(0xffffffffu, mbar_wait(&amax_bar[grp], (uint32_t)j & 1u, &abort_flag,
                                                   dev_status)))
                break;
            const unsigned int amax_bits = amax_sh[grp][slot][r];
            slot = slot == 2 ? 0 : slot + 1;
            const float sc0 = DYN ? __fdiv_rn(__uint_as_float(amax_bits), (float)p.qmax) : *scale_in;
            const float sc = sc0 < FLT_MIN ? FLT_MIN : sc0;   // lower clamp; NaN stays NaN
            const RowDivisor dv(sc, p.qmax);
            if (row_ok && rho == 0) scales[row] = sc;
            // pass 2: the codes, 64 per valid group-row
#pragma unroll 1
            for (int a = 0; a < P; ++a) {
                const int gr = P > 1 ? a * p.L + l : rho;
                const bool gr_ok = row_ok && (P == 1 || gr < p.GR);
                int8_t* dst = codes + row * p.ldq + (int64_t)gr * 64;
#pragma unroll 1
                for (int c = 0; c < 64; c += 32) {
                    uint32_t v[32];
                    tc_ld_32x32b_x32(tacc + (uint32_t)(64 * a + c), v);
                    tc_wait_ld();
                    if (gr_ok) {
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            uint32_t out[4];
                            if (DYN) {
                                unsigned long long y2[8];
#pragma unroll
                                for (int k = 0; k < 8; ++k)
                                    y2[k] = f2_pack(__uint_as_float(v[16 * u + 2 * k]),
                                                    __uint_as_float(v[16 * u + 2 * k + 1]));
                                quant16_dyn2(y2, dv, out);
                            } else {
                                float y[16];
#pragma unroll
                                for (int k = 0; k < 16; ++k) y[k] = __uint_as_float(v[16 * u + k]);
                                quant16(y, dv, out);
                            }
                            int8_t* o = dst + c + 16 * u;
                            if (p.vec_codes) {
                                *reinterpret_cast<uint4*>(o) = make_uint4(out[0], out[1], out[2], out[3]);
                            } else {
#pragma unroll
                                for (int k = 0; k < 16; ++k) o[k] = (int8_t)((out[k / 4] >> (8 * (k % 4))) & 0xFF);
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&d_empty[grp]);   // done reading the accumulator
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kAcc * kAccCols);
    }
}

// fp32, g = 64, unit K stride, 16-byte-aligned x and R, row pitch a multiple of 4 floats,
// K / 64 <= 256.  Returns CK_ERR_UNSUPPORTED otherwise.
ck_status launch_rq_tf32(const void* x, int64_t M, int64_t K, int64_t sm, int64_t sk,
                         const void* R, const float* scale_in, int8_t* codes, int64_t ldq,
                         float* scales, int qmax, int* dev_status, cudaStream_t stream) {
    using namespace rqtf;
    if (sk != 1 || !aligned(x, 16) || !aligned(R, 16) || K % 64 != 0 || K / 64 > 256 ||
        (M > 1 && (sm % 4 != 0 || sm < K)) || M >= (1LL << 31))
        return CK_ERR_UNSUPPORTED;
    RqTf32Params p;
    p.M = M;
    p.K = K;
    p.ldq = ldq;
    p.GR = (int)(K / 64);
    const bool split = p.GR > 128;
    p.RB = split ? 1 : 128 / p.GR;
    p.L = split ? (p.GR + 1) / 2 : p.GR;
    const int64_t tiles = (M + p.RB - 1) / p.RB;
    if (tiles >= (1LL << 31) / p.RB) return CK_ERR_UNSUPPORTED;
    p.tiles = (int)tiles;
    p.box_bytes = (uint32_t)(p.RB * p.L * 128);
    p.idesc = idesc_tf32(128, 64);
    p.vec_codes = (aligned(codes, 16) && ldq % 16 == 0) ? 1 : 0;
    p.qmax = qmax;

    // x as (channel within group, group, row); each box is 32 channels (128 bytes) of L groups
    // of RB rows
    CUtensorMap map;
    const uint64_t dims[3] = {64, (uint64_t)p.GR, (uint64_t)M};
    const uint64_t strides[2] = {256, (uint64_t)(M > 1 ? sm : K) * 4};
    const uint32_t box[3] = {32u, (uint32_t)p.L, (uint32_t)p.RB};
    const ck_status st = encode_tma(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, x, dims, strides, box,
                                    CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != CK_OK) return st;
    const int grid = (int)(p.tiles < num_sms() ? p.tiles : num_sms());
    auto run = [&](auto kern) -> ck_status {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem) !=
            cudaSuccess)
            return CK_ERR_CUDA;
        kern<<<grid, kThreads, kSmem, stream>>>(map, static_cast<const float*>(R), scale_in, codes,
                                                scales, p, dev_status);
        return cudaGetLastError() == cudaSuccess ? CK_OK : CK_ERR_CUDA;
    };
    if (split)
        return scale_in ? run(rq_tf32_kernel<false, 2>) : run(rq_tf32_kernel<true, 2>);
    return scale_in ? run(rq_tf32_kernel<false, 1>) : run(rq_tf32_kernel<true, 1>);
}

ck_status launch_rq_f32_wide(const void* x, int64_t M, int64_t K, int64_t sm, int64_t sk,
                             const void* R, int g, const float* scale_in, int8_t* codes,
                             int64_t ldq, float* scales, int qmax, int* dev_status,
                             cudaStream_t stream) {
    if (g == 64)
        return launch_rq_tf32(x, M, K, sm, sk, R, scale_in, codes, ldq, scales, qmax, dev_status,
                              stream);
    if (g == 256)
        return launch_rq_f32_ffma256(x, M, K, sm, sk, R, scale_in, codes, ldq, scales, qmax,
                                     dev_status, stream);
    return CK_ERR_UNSUPPORTED;
}

}  // namespace ck
