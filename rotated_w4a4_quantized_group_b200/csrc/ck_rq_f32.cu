// ck_rq_f32.cu -- stage 1 for fp32 activations with g = 16: the group-wise rotation in fp32
// (the input dtype), the row-wise signed-INT4 scale and the INT8-stored codes.
//
// Operation (comfy-kitchen PR #198 "Consolidate INT8, RotateQuant, RoPE and ConvRot W4A4
// backends", "W4A4 correctness and performance scope": the rotation keeps the FP32 input
// dtype; PR #201 "Avoid activation pack/unpack in ConvRot W4A4", "Correctness and tests":
// contiguous, strided and transposed inputs):
//   y[m, 16 j + c] = fp32( sum_i x[m, 16 j + i] * R[i, c] )   the sum formed in fp64
//   s[m] = max(fp32(max_k |y[m, k]|) / qmax, FLT_MIN)          (or the caller's tensor-wise scale)
//   q[m, k] = clamp(round_half_even(y[m, k] / s[m]), -qmax - 1, qmax)
// with qmax = 7 (signed INT4 codes) or 127 (the INT8 codes of the W8A8 variant).
//
// The sum: a product of two fp32 values is exact in fp64.  Four chained FP64 MMAs
// (mma.sync m8n8k4 .f64, k-steps i = 0-3, 4-7, 8-11, 12-15, from a zero accumulator) gave
// the same fp64 value as adding the sixteen products in i order with fp64 fused
// multiply-adds on 524,288 random fp32 sums on B200 (bit for bit), and y is that value
// rounded once to fp32; the parity tests compare these codes, scales and outputs with the
// oracle's in-order fp64 sum.
//
// Row-major input (unit K stride) and column-major input (unit M stride, the transposed view
// of a (K, M) buffer) are both read by TMA straight from HBM, each byte once:
//   - a block of RB rows is split along K over a thread-block cluster of C CTAs, each holding
//     its K slice of the block in shared memory (at most 64 KB; two or three CTAs per SM);
//   - column-major input: 16 rows per block, boxes of 16 rows x 256 channels (64-byte rows);
//     row-major input: boxes of up to 256 groups x RB rows, as (channel, group, row);
//   - eight warps rotate the slice in place: 8 group-rows x 16 channels per task, x converted
//     exactly to fp64 as the MMA's A fragments, R as its B fragments (eight fp64 registers a
//     lane), y rounded to fp32 over x in shared memory (64-byte swizzled boxes keep the
//     fragment loads and stores at most 2-way bank conflicted);
//   - the row absmax of the slice is reduced in shared memory, then over the cluster through
//     distributed shared memory (each CTA reads its peers' partial maxima; no multicast);
//   - each CTA quantizes its slice from shared memory and stores its codes.
// Every CTA of a cluster walks the same row blocks and takes every cluster barrier, also after
// a timeout (which skips the work but not the barriers), so no barrier waits for a CTA that
// left.  Rows past M arrive as zeros and are not stored.
#include <cuda.h>
#include <float.h>
#include <stdint.h>

#include "ck_device.cuh"
#include "ck_internal.h"

namespace ck {

namespace rqf32 {
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxBoxes = 16;
constexpr int kMaxRB = 16;
constexpr int kColRB = 16;              // column-major blocks: 16 rows = 64-byte box rows
constexpr int kColBoxK = 256;           // channels per column-major box
constexpr size_t kTileBudget = 64 * 1024;
constexpr int kMaxCluster = 16;
}  // namespace rqf32

struct RqF32Params {
    int64_t M, K, ldq;
    int64_t nblocks;      // row blocks of RB rows
    int KS;               // channels per CTA (its K slice), a multiple of 16
    int RB;               // rows per block
    int nboxes;           // TMA boxes per CTA and block
    int GBb;              // row-major: groups per box (all of the slice's groups, or 256)
    uint32_t box_bytes;   // bytes one box delivers (what its mbarrier expects)
    uint32_t box_stride;  // bytes between box buffers (box_bytes rounded up to 1024)
    int vec_codes;        // 16-byte code stores are aligned
    int qmax;             // code grid [-qmax - 1, qmax]: 7 (INT4) or 127 (INT8)
};

// Float offset of word w (0..15) of 64-byte row `row` of a box stored with TMA's 64-byte
// swizzle (box bases 1024-byte aligned): the 16-byte chunk index is XORed with (row / 2) % 4.
__device__ __forceinline__ uint32_t sw64(uint32_t row, uint32_t w) {
    return row * 16u + ((((w >> 2) ^ (row >> 1)) & 3u) << 2) + (w & 3u);
}

// D (8 x 8, fp64) += A (8 x 4) * B (4 x 8): lane l holds A[l / 4][l % 4], B[l % 4][l / 4] and
// D[l / 4][2 (l % 4) + {0, 1}].
__device__ __forceinline__ void dmma_8x8x4(double& d0, double& d1, double a, double b) {
    asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
                 : "+d"(d0), "+d"(d1)
                 : "d"(a), "d"(b));
}

// Sixteen codes of a row: the dynamic-scale path (no clamp needed) or the general one.
__device__ __forceinline__ void quant16_any(const float (&y)[16], const RowDivisor& dv, bool dyn,
                                            uint32_t (&out)[4]) {
    if (dyn) {
        unsigned long long y2[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) y2[i] = f2_pack(y[2 * i], y[2 * i + 1]);
        quant16_dyn2(y2, dv, out);
    } else {
        quant16(y, dv, out);
    }
}

__device__ __forceinline__ float f32_row_scale(float amax, const float* scale_in, int qmax) {
    const float s = scale_in ? *scale_in : __fdiv_rn(amax, (float)qmax);
    return (s < FLT_MIN) ? FLT_MIN : s;   // lower clamp; NaN stays NaN
}

// MINB: CTAs per SM the registers are budgeted for (2: up to 128 a thread; 3: up to 85)
template <bool COL, int MINB>
__global__ void __launch_bounds__(rqf32::kThreads, MINB)
    rq_f32_g16_kernel(const __grid_constant__ CUtensorMap xmap, const float* __restrict__ R,
                      const float* __restrict__ scale_in, int8_t* __restrict__ codes,
                      float* __restrict__ scales, RqF32Params p, int* dev_status) {
    // the linear's GEMM, launched as this kernel's dependent, may start its prologue now
    grid_dependents_launch();
    using namespace rqf32;
    extern __shared__ __align__(1024) unsigned char f32_smem[];
    float* tile = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(f32_smem) + 1023) &
                                           ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t full[kMaxBoxes];
    __shared__ unsigned int amax_sh[2][kMaxRB];   // this CTA's partial row maxima (|y| bits)
    __shared__ float row_s[kMaxRB], row_r[kMaxRB];
    __shared__ unsigned int peer_sh[kMaxCluster][kMaxRB];   // every CTA's partial maxima
    __shared__ int abort_flag;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t rank = cluster_ctarank(), ncta = cluster_nctarank();
    const int64_t k0 = (int64_t)rank * p.KS;      // the slice's first channel
    const int ngroups = p.KS / 16;
    const uint32_t box_floats = p.box_stride / 4u;

    // R as the MMA's B fragments: k-step ks, channel half nh -> R[4 ks + l % 4][8 nh + l / 4]
    const int fr = lane >> 2, fc = lane & 3;   // fragment row (group-row) and column of the lane
    double rb[4][2];
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
#pragma unroll
        for (int nh = 0; nh < 2; ++nh) rb[ks][nh] = (double)__ldg(R + (4 * ks + fc) * 16 + 8 * nh + fr);

    if (tid == 0) {
        for (int b = 0; b < p.nboxes; ++b) mbar_init(&full[b], 1);
        abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&xmap);
    }
    if (tid < 2 * kMaxRB) (&amax_sh[0][0])[tid] = 0u;
    __syncthreads();

    uint32_t it = 0;   // row blocks this CTA has taken: the parity of full[] and amax_sh
    for (int64_t blk = blockIdx.y; blk < p.nblocks; blk += gridDim.y, ++it) {
        const int64_t m0 = blk * p.RB;
        const uint32_t par = it & 1u;
        const bool skip = abort_flag != 0;     // read after the previous block's barriers
        // ---------------------------------------------------------------- loads
        if (tid == 0 && !skip) {
            for (int b = 0; b < p.nboxes; ++b) {
                float* dst = tile + (size_t)b * box_floats;
                mbar_arrive_expect_tx(&full[b], p.box_bytes);
                if (COL)
                    tma_load_2d(dst, &xmap, &full[b], (int32_t)m0, (int32_t)(k0 + (int64_t)b * kColBoxK));
                else
                    tma_load_3d(dst, &xmap, &full[b], 0, (int32_t)(k0 / 16 + (int64_t)b * p.GBb),
                                (int32_t)m0);
            }
        }
        // ---------------------------------------------------------------- rotate in place
        int waited = 0;   // boxes of this block the warp has seen complete
        auto wait_box = [&](int b) -> bool {
            while (waited <= b) {
                if (!__all_sync(0xffffffffu, mbar_wait(&full[waited], par, &abort_flag, dev_status)))
                    return false;
                ++waited;
            }
            return true;
        };
        bool ok = !skip;
        if (COL) {
            // task = (row half h, groups j and j + 4): rows 8 h .. 8 h + 7 of the block, channels
            // 16 j .. and 16 (j + 4) .. of the slice; x[m][k] sits in 64-byte tile row k, word m.
            // A warp keeps one row half, so its lanes' rows (8 h + l / 4) stay fixed.  The swizzle
            // phase of tile row 16 j + r is (r / 2) % 4 whatever j, so the lane's offsets within a
            // group are fixed too: loads at k-step ks, stores at channel pair (nh, e)
            const int h = warp & 1;
            const uint32_t m = 8u * h + fr;
            uint32_t lda[4], sta[4];
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) lda[ks] = sw64(4u * ks + fc, m);
#pragma unroll
            for (int nh = 0; nh < 2; ++nh)
#pragma unroll
                for (int e = 0; e < 2; ++e) sta[2 * nh + e] = sw64(8u * nh + 2u * fc + e, m);
            float mx = 0.f;
            // warp pair q takes groups 8 i + q and 8 i + q + 4 (one 256-channel box holds both)
            const int q = warp >> 1;   // 0 .. 3
            for (int j0 = q; ok && j0 < ngroups; j0 += 8) {
                const int j1 = j0 + 4;   // may lie past the slice
                const bool two = j1 < ngroups;
                if (!wait_box((16 * (two ? j1 : j0)) / kColBoxK)) {
                    ok = false;
                    break;
                }
                float* xs0 = tile + (size_t)j0 * 256;
                float* xs1 = tile + (size_t)(two ? j1 : j0) * 256;
                double a0[4], a1[4];
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    a0[ks] = (double)xs0[lda[ks]];
                    a1[ks] = (double)xs1[lda[ks]];
                }
                __syncwarp();   // every lane has read the groups before any lane overwrites them
                double d[2][2][2];
#pragma unroll
                for (int nh = 0; nh < 2; ++nh)
#pragma unroll
                    for (int t = 0; t < 2; ++t) d[t][nh][0] = d[t][nh][1] = 0.0;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
#pragma unroll
                    for (int nh = 0; nh < 2; ++nh) {
                        dmma_8x8x4(d[0][nh][0], d[0][nh][1], a0[ks], rb[ks][nh]);
                        dmma_8x8x4(d[1][nh][0], d[1][nh][1], a1[ks], rb[ks][nh]);
                    }
#pragma unroll
                for (int nh = 0; nh < 2; ++nh)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const float y0 = __double2float_rn(d[0][nh][e]);
                        mx = fmax_nan(mx, fabsf(y0));
                        xs0[sta[2 * nh + e]] = y0;
                        if (two) {
                            const float y1 = __double2float_rn(d[1][nh][e]);
                            mx = fmax_nan(mx, fabsf(y1));
                            xs1[sta[2 * nh + e]] = y1;
                        }
                    }
            }
            // row 8 h + l / 4: its four fragment columns are lanes 4 (l / 4) .. + 3
            mx = fmax_nan(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmax_nan(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            if (fc == 0) atomicMax(&amax_sh[par][m], __float_as_uint(mx));
        } else {
            // task = (row m, groups 16 o .. 16 o + 15 of the slice) as two fragment sets of 8
            // group-rows.  Warps own rows: wpr warps share a row (taking every wpr-th 16 groups),
            // a warp takes every (8 / wpr)-th row.  Group j of box b = j / GBb is 64-byte row
            // (m GBb + j - b GBb) of the box
            const int o16 = (ngroups + 15) / 16;
            const int wpr = p.RB >= kWarps ? 1 : kWarps / p.RB;
            // the box of group j: 0 when one box holds the slice's groups, else j / 256 (boxes
            // of 256 groups)
            const int bshift = p.nboxes == 1 ? 30 : 8;
            for (int mrow = warp / wpr; ok && mrow < p.RB; mrow += kWarps / wpr) {
                float mx = 0.f;
                for (int o = warp % wpr; ok && o < o16; o += wpr) {
                    const int jlast = (16 * o + 15) < ngroups ? (16 * o + 15) : (ngroups - 1);
                    if (!wait_box(jlast >> bshift)) {
                        ok = false;
                        break;
                    }
                    double a[2][4];
                    float* bxs[2];
                    uint32_t rows_[2];
                    bool jv[2];
#pragma unroll
                    for (int t2 = 0; t2 < 2; ++t2) {
                        const int j = 16 * o + 8 * t2 + fr;
                        jv[t2] = j < ngroups;
                        const int b = jv[t2] ? j >> bshift : 0;
                        bxs[t2] = tile + (size_t)b * box_floats;
                        rows_[t2] = jv[t2] ? (uint32_t)(mrow * p.GBb + (j - b * p.GBb)) : 0u;
                        const uint32_t ph = (rows_[t2] >> 1) & 3u;
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            a[t2][ks] = jv[t2] ? (double)bxs[t2][rows_[t2] * 16u + (((uint32_t)ks ^ ph) << 2) + fc] : 0.0;
                    }
                    __syncwarp();
                    double d[2][2][2];
#pragma unroll
                    for (int nh = 0; nh < 2; ++nh)
#pragma unroll
                        for (int t2 = 0; t2 < 2; ++t2) d[t2][nh][0] = d[t2][nh][1] = 0.0;
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
#pragma unroll
                        for (int nh = 0; nh < 2; ++nh) {
                            dmma_8x8x4(d[0][nh][0], d[0][nh][1], a[0][ks], rb[ks][nh]);
                            dmma_8x8x4(d[1][nh][0], d[1][nh][1], a[1][ks], rb[ks][nh]);
                        }
#pragma unroll
                    for (int t2 = 0; t2 < 2; ++t2) {
                        if (!jv[t2]) continue;
                        const uint32_t ph = (rows_[t2] >> 1) & 3u;
#pragma unroll
                        for (int nh = 0; nh < 2; ++nh) {
                            const float y0 = __double2float_rn(d[t2][nh][0]);
                            const float y1 = __double2float_rn(d[t2][nh][1]);
                            mx = fmax_nan(mx, fmax_nan(fabsf(y0), fabsf(y1)));
                            // words 8 nh + 2 fc, + 1: chunk 2 nh + fc / 2
                            const uint32_t off = rows_[t2] * 16u +
                                                 ((((uint32_t)(2 * nh) + (fc >> 1)) ^ ph) << 2) +
                                                 2u * (fc & 1);
                            *reinterpret_cast<float2*>(bxs[t2] + off) = make_float2(y0, y1);
                        }
                    }
                }
#pragma unroll
                for (int dd = 16; dd > 0; dd >>= 1) mx = fmax_nan(mx, __shfl_xor_sync(0xffffffffu, mx, dd));
                if (lane == 0) atomicMax(&amax_sh[par][mrow], __float_as_uint(mx));
            }
        }
        __syncthreads();
        // ---------------------------------------------------------------- row scales
        // every CTA of the cluster takes this barrier once per block, whatever happened above
        if (ncta > 1) cluster_sync_all();
        // peer maxima: thread (row m, CTA q) reads one word, then each row's thread takes the
        // maximum of the CTA's slots (one distributed read per thread, all in parallel)
        for (int i = tid; i < p.RB * (int)ncta; i += kThreads) {
            const int m = i % p.RB;
            const uint32_t q = (uint32_t)(i / p.RB);
            peer_sh[q][m] = q == rank ? amax_sh[par][m] : dsmem_load_u32(&amax_sh[par][m], q);
        }
        __syncthreads();
        if (tid < p.RB) {
            unsigned int bits = 0u;
            for (uint32_t q = 0; q < ncta; ++q) bits = peer_sh[q][tid] > bits ? peer_sh[q][tid] : bits;
            const float s = f32_row_scale(__uint_as_float(bits), scale_in, p.qmax);
            const RowDivisor dv(s, p.qmax);
            row_s[tid] = s;
            row_r[tid] = dv.r;
            if (rank == 0 && m0 + tid < p.M && !skip) scales[m0 + tid] = s;
        }
        __syncthreads();
        // ---------------------------------------------------------------- quantize + store
        if (ok) {
            const int rows = (int)((p.M - m0) < p.RB ? (p.M - m0) : p.RB);
            if (COL) {
                // thread -> (row m = u % 16, group j = u / 16): 16 values down tile column m
                for (int u = tid; u < 16 * ngroups; u += kThreads) {
                    const int m = u & 15, j = u >> 4;
                    if (m >= rows) continue;
                    RowDivisor dv(row_s[m], p.qmax);
                    dv.r = row_r[m];
                    float y[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) y[i] = tile[sw64(16u * j + i, (uint32_t)m)];
                    uint32_t out[4];
                    quant16_any(y, dv, scale_in == nullptr, out);
                    int8_t* dst = codes + (m0 + m) * p.ldq + k0 + 16 * j;
                    if (p.vec_codes) {
                        *reinterpret_cast<uint4*>(dst) = make_uint4(out[0], out[1], out[2], out[3]);
                    } else {
#pragma unroll
                        for (int q = 0; q < 16; ++q) dst[q] = (int8_t)((out[q / 4] >> (8 * (q % 4))) & 0xFF);
                    }
                }
            } else {
                // thread -> (row m, group j) of the slice: 16 consecutive values; (m, j) advance
                // by kThreads groups at a time without a division
                int m = tid / ngroups, j = tid - m * ngroups;
                const int dm = kThreads / ngroups, dj = kThreads - dm * ngroups;
                for (; m < rows; m += dm, j += dj) {
                    if (j >= ngroups) {
                        j -= ngroups;
                        ++m;
                        if (m >= rows) break;
                    }
                    RowDivisor dv(row_s[m], p.qmax);
                    dv.r = row_r[m];
                    const int b = p.nboxes == 1 ? 0 : j >> 8;   // boxes of 256 groups
                    const float* bx = tile + (size_t)b * box_floats;
                    const uint32_t row = (uint32_t)(m * p.GBb + (j - b * p.GBb));
                    float y[16];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float4 v = *reinterpret_cast<const float4*>(bx + sw64(row, 4u * q));
                        y[4 * q] = v.x;
                        y[4 * q + 1] = v.y;
                        y[4 * q + 2] = v.z;
                        y[4 * q + 3] = v.w;
                    }
                    uint32_t out[4];
                    quant16_any(y, dv, scale_in == nullptr, out);
                    int8_t* dst = codes + (m0 + m) * p.ldq + k0 + 16 * j;
                    if (p.vec_codes) {
                        *reinterpret_cast<uint4*>(dst) = make_uint4(out[0], out[1], out[2], out[3]);
                    } else {
#pragma unroll
                        for (int q = 0; q < 16; ++q) dst[q] = (int8_t)((out[q / 4] >> (8 * (q % 4))) & 0xFF);
                    }
                }
            }
        }
        // the tile is free for the next block's copies; the other maximum slot is free too (its
        // last readers, the peers, read it before this block's cluster barrier)
        if (tid < kMaxRB) amax_sh[par ^ 1u][tid] = 0u;
        __syncthreads();
        if (abort_flag != 0 && !skip) {   // block-uniform: read after the barrier
            // copies of this block still in flight land before the tile is reused or left
            if (tid == 0)
                for (int b = 0; b < p.nboxes; ++b) mbar_wait(&full[b], par, nullptr, nullptr);
            __syncthreads();
        }
    }
    // no CTA leaves while a peer may still read its partial maxima
    if (ncta > 1) cluster_sync_all();
}

ck_status launch_rq_f32_g16(const void* x, int64_t M, int64_t K, int64_t sm, int64_t sk,
                            const void* R, const float* scale_in, int8_t* codes, int64_t ldq,
                            float* scales, int qmax, int* dev_status, cudaStream_t stream) {
    using namespace rqf32;
    const bool col = sm == 1 && sk != 1;
    const bool row = sk == 1;
    if (!(col || row) || !aligned(x, 16) || K % 16 != 0 || M >= (1LL << 31)) return CK_ERR_UNSUPPORTED;
    if (col && (sk % 4 != 0 || sk < M)) return CK_ERR_UNSUPPORTED;
    if (row && (sm % 4 != 0 || (M > 1 && sm < K))) return CK_ERR_UNSUPPORTED;

    RqF32Params p;
    p.M = M;
    p.K = K;
    p.ldq = ldq;
    int C = 0;
    if (col) {
        p.RB = kColRB;
        // the smallest cluster whose slices (multiples of 16 channels) fit the tile budget
        for (int c = 1; c <= kMaxCluster && !C; ++c) {
            if (K % (16 * c) != 0) continue;
            const int64_t ks = K / c;
            const int64_t nb = (ks + kColBoxK - 1) / kColBoxK;
            if (nb <= kMaxBoxes && (size_t)nb * kColBoxK * kColRB * 4 <= kTileBudget) C = c;
        }
        if (!C) return CK_ERR_UNSUPPORTED;
        p.KS = (int)(K / C);
        p.nboxes = (p.KS + kColBoxK - 1) / kColBoxK;
        p.GBb = 0;
        p.box_bytes = (uint32_t)(kColBoxK * kColRB * 4);
        p.box_stride = p.box_bytes;
    } else {
        for (int c = 1; c <= kMaxCluster && !C; ++c) {
            if (K % (16 * c) != 0) continue;
            const int64_t groups = K / c / 16;
            const int64_t gbb = groups < 256 ? groups : 256;
            const int64_t nb = (groups + gbb - 1) / gbb;
            if (nb <= kMaxBoxes && (size_t)nb * ((gbb * 64 + 1023) / 1024 * 1024) <= kTileBudget) C = c;
        }
        if (!C) return CK_ERR_UNSUPPORTED;
        p.KS = (int)(K / C);
        const int groups = p.KS / 16;
        p.GBb = groups < 256 ? groups : 256;
        p.nboxes = (groups + p.GBb - 1) / p.GBb;
        // rows per block: as many as fit the budget, at most 16 and at most M
        int rb = kMaxRB;
        while (rb > 1 && (size_t)p.nboxes * (((size_t)p.GBb * 64 * rb + 1023) / 1024 * 1024) > kTileBudget)
            --rb;
        if (rb > kMaxRB) rb = kMaxRB;
        if (rb > M) rb = (int)M;
        if (rb < 1) return CK_ERR_UNSUPPORTED;
        p.RB = rb;
        p.box_bytes = (uint32_t)(p.GBb * 64 * p.RB);
        p.box_stride = (p.box_bytes + 1023u) & ~1023u;
    }
    p.nblocks = (M + p.RB - 1) / p.RB;
    p.vec_codes = (aligned(codes, 16) && ldq % 16 == 0) ? 1 : 0;
    p.qmax = qmax;

    CUtensorMap map;
    ck_status st;
    if (col) {
        // x^T as (M, K): element (m, k) at x + (m + k sk) floats
        const uint64_t dims[2] = {(uint64_t)M, (uint64_t)K};
        const uint64_t strides[1] = {(uint64_t)sk * 4};
        const uint32_t box[2] = {(uint32_t)kColRB, (uint32_t)kColBoxK};
        st = encode_tma(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, x, dims, strides, box,
                        CU_TENSOR_MAP_SWIZZLE_64B);
    } else {
        // x as (channel within group, group, row)
        const uint64_t dims[3] = {16, (uint64_t)(K / 16), (uint64_t)M};
        const uint64_t strides[2] = {64, (uint64_t)sm * 4};
        const uint32_t box[3] = {16, (uint32_t)p.GBb, (uint32_t)p.RB};
        st = encode_tma(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, x, dims, strides, box,
                        CU_TENSOR_MAP_SWIZZLE_64B);
    }
    if (st != CK_OK) return st;

    const size_t smem = (size_t)p.nboxes * p.box_stride + 1024;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3((unsigned)C, 1, 1);
    // persistent clusters: as many as can be resident, at most one per block.  Three CTAs per
    // SM (registers capped at 85) when the blocks outnumber what two CTAs per SM hold: more
    // CTAs overlap one another's load, rotation, cluster exchange and quantize phases; with
    // fewer blocks the wider register budget makes each CTA faster.
    auto prepare = [&](auto kern, int& max_clusters) -> ck_status {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return CK_ERR_CUDA;
        if (C > 8 && cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed,
                                          1) != cudaSuccess)
            return CK_ERR_UNSUPPORTED;
        max_clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg) != cudaSuccess ||
            max_clusters < 1)
            return CK_ERR_UNSUPPORTED;
        return CK_OK;
    };
    auto run = [&](auto kern, int max_clusters) -> ck_status {
        const int64_t gy = p.nblocks < max_clusters ? p.nblocks : max_clusters;
        cfg.gridDim = dim3((unsigned)C, (unsigned)gy, 1);
        if (cudaLaunchKernelEx(&cfg, kern, map, static_cast<const float*>(R), scale_in, codes,
                               scales, p, dev_status) != cudaSuccess)
            return CK_ERR_CUDA;
        return CK_OK;
    };
    auto k2 = col ? rq_f32_g16_kernel<true, 2> : rq_f32_g16_kernel<false, 2>;
    auto k3 = col ? rq_f32_g16_kernel<true, 3> : rq_f32_g16_kernel<false, 3>;
    int mc2 = 0, mc3 = 0;
    st = prepare(k2, mc2);
    if (st != CK_OK) return st;
    if (p.nblocks > mc2) {
        st = prepare(k3, mc3);
        if (st != CK_OK) return st;
        st = mc3 > mc2 ? run(k3, mc3) : run(k2, mc2);
    } else {
        st = run(k2, mc2);
    }
    if (st != CK_OK) return st;
    return cudaGetLastError() == cudaSuccess ? CK_OK : CK_ERR_CUDA;
}

}  // namespace ck
