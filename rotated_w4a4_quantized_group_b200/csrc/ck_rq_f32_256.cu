// ck_rq_f32_256.cu -- stage 1 for fp32 activations with g = 256: the group-wise rotation as
// fp32 fused multiply-adds, the row-wise scale and the INT8-stored codes.
//
// Operation (comfy-kitchen PR #198 "Consolidate INT8, RotateQuant, RoPE and ConvRot W4A4
// backends", "W4A4 correctness and performance scope": the rotation keeps the FP32 input
// dtype; PR #155 "Add fused RotateQuant backend": group sizes 16/64/256):
//   y[m, 256 j + c] = fp32 FMA chain over i = 0 .. 255 in order of x[m, 256 j + i] R[i, c]
//   s[m] = max(fp32(max_k |y[m, k]|) / qmax, FLT_MIN)          (or the caller's scale)
//   q[m, k] = clamp(round_half_even(y[m, k] / s[m]), -qmax - 1, qmax)
//
// 256 fused multiply-adds per element make this ALU-bound (8192 x 3840: 8.05 G FMA, 224 us of
// the B200's FFMA rate, against 24 us of HBM).  R (256 KB) does not fit in shared memory beside
// the rows, so it streams through it in slices of 32 rows (32 KB, TMA, two slots), once per
// block of rows; the partial sums stay in registers across the slices:
//   - a block is RB whole rows (RB K / 256 <= 64 group-rows; a 3-D TMA box of 256 channels x
//     K / 256 groups x RB rows) in one of two buffers, the next block's copy in flight;
//   - warp w computes group-rows w, w + 8, .. of the block, NJ = ceil(group-rows / 8) <= 8 of
//     them (a template parameter: the FMA step has no per-row branch; the buffers hold 8 NJ
//     group-rows and the padding ones are never folded into a maximum or stored), lane l the
//     channels 4 l .. 4 l + 3 and 128 + 4 l .. 128 + 4 l + 3 of each: 8 NJ fp32 accumulators.
//     Per value of i a lane reads two 16-byte pieces of R's row (the warp's 32 lanes read two
//     contiguous 512-byte runs: no bank conflict) and each x value once, broadcast to the
//     warp, so shared memory serves about one 128-byte wavefront per six FMA instructions and
//     the FMA pipe, not the load pipe, sets the pace;
//   - after the last slice: the row absmax over each group-row by a warp reduction and shared
//     atomics, the row scales, and the codes from the registers in 4-byte stores (a warp
//     writes two contiguous 128-byte runs of a group-row).
// Every wait is bounded; a timeout records CK_ERR_TIMEOUT, the kernel stops issuing copies,
// waits for those in flight and returns.
#include <cuda.h>
#include <float.h>
#include <stdint.h>

#include "ck_device.cuh"
#include "ck_internal.h"

namespace ck {

namespace rqf256 {
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRows = 8;                    // group-rows a warp owns (at most)
constexpr int kMaxGR = kWarps * kRows;      // group-rows a block (64)
constexpr int kSlice = 32;                  // rows of R per slice
constexpr int kSlices = 256 / kSlice;
constexpr uint32_t kSliceBytes = kSlice * 256 * 4;
constexpr int kMaxRB = 64;
}  // namespace rqf256

struct RqF256Params {
    int64_t M, K, ldq, nblocks;
    int RB;               // rows per block
    int gpr;              // group-rows per row, K / 256
    uint32_t box_bytes;   // RB K 4
    int vec_codes, qmax;
};

// NJ: group-rows a warp computes, ceil(RB K / 256 / 8).  Every warp computes NJ of them (the
// x buffers hold 8 NJ group-rows), so the FMA step has no per-row branch; group-rows past the
// block's (never written by the copy) are neither folded into a maximum nor stored.
template <int NJ>
__global__ void __launch_bounds__(rqf256::kThreads, 1)
    rq_f32_ffma256_kernel(const __grid_constant__ CUtensorMap xmap,
                          const __grid_constant__ CUtensorMap rmap,
                          const float* __restrict__ scale_in, int8_t* __restrict__ codes,
                          float* __restrict__ scales, RqF256Params p, int* dev_status) {
    // the linear's GEMM, launched as this kernel's dependent, may start its prologue now
    grid_dependents_launch();
    using namespace rqf256;
    extern __shared__ __align__(1024) unsigned char f256_smem[];
    float* const base = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(f256_smem) + 127) &
                                                 ~uintptr_t(127));
    float* const rslot0 = base;                                 // R rows 32 s .. 32 s + 31
    float* const rslot1 = base + kSlice * 256;
    float* const xbuf0 = base + 2 * kSlice * 256;               // the two row-block buffers
    float* const xbuf1 = xbuf0 + (size_t)NJ * kWarps * 256;
    __shared__ __align__(8) uint64_t xfull[2], rfull[2];
    __shared__ unsigned int amax_sh[kMaxRB];
    __shared__ float row_s[kMaxRB], row_r[kMaxRB];
    __shared__ int abort_flag;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int ngr = p.RB * p.gpr;                                 // group-rows a block
    const int nmine = (int)((p.nblocks - 1 - blockIdx.x) / gridDim.x + 1);
    const int nslices = nmine * kSlices;                          // R slices this CTA reads
    int xissued = 0, rissued = 0;                                 // thread 0's copies
    auto issue_x = [&](int b) {
        float* dst = (b & 1) ? xbuf1 : xbuf0;
        mbar_arrive_expect_tx(&xfull[b & 1], p.box_bytes);
        tma_load_3d(dst, &xmap, &xfull[b & 1], 0, 0,
                    (int32_t)(((int64_t)blockIdx.x + (int64_t)b * gridDim.x) * p.RB));
    };
    auto issue_r = [&](int n) {   // slice n % kSlices into slot n % 2
        mbar_arrive_expect_tx(&rfull[n & 1], kSliceBytes);
        tma_load_2d((n & 1) ? rslot1 : rslot0, &rmap, &rfull[n & 1], 0, (n % kSlices) * kSlice);
    };
    if (tid < kMaxRB) amax_sh[tid] = 0u;
    if (tid == 0) {
        mbar_init(&xfull[0], 1);
        mbar_init(&xfull[1], 1);
        mbar_init(&rfull[0], 1);
        mbar_init(&rfull[1], 1);
        abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&xmap);
        tma_prefetch_desc(&rmap);
        for (; xissued < 2 && xissued < nmine; ++xissued) issue_x(xissued);
        for (; rissued < 2 && rissued < nslices; ++rissued) issue_r(rissued);
    }
    __syncthreads();

    const int c0 = 4 * lane;          // channels c0 .. c0 + 3 and 128 + c0 .. 128 + c0 + 3
    for (int it = 0; it < nmine; ++it) {
        const int64_t m0 = ((int64_t)blockIdx.x + (int64_t)it * gridDim.x) * p.RB;
        const float* xt = (it & 1) ? xbuf1 : xbuf0;
        bool ok = abort_flag == 0 &&
                  mbar_wait(&xfull[it & 1], (uint32_t)(it >> 1) & 1u, &abort_flag, dev_status);
        float acc[NJ][8];
#pragma unroll
        for (int j = 0; j < NJ; ++j)
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[j][c] = 0.f;
        for (int s = 0; s < kSlices; ++s) {
            const int n = it * kSlices + s;
            ok = ok && mbar_wait(&rfull[n & 1], (uint32_t)(n >> 1) & 1u, &abort_flag, dev_status);
            if (__all_sync(0xffffffffu, ok)) {
                const float* rs = (n & 1) ? rslot1 : rslot0;
                const float* xs = xt + (size_t)warp * 256 + kSlice * s;   // group-row warp, i = 32 s
#pragma unroll 1
                for (int i = 0; i < kSlice; i += 4) {
                    // every operand of the step is loaded before the first FMA, so that the
                    // loads' latency is paid once per step, not once per group-row
                    float4 ra[4], rb[4], xv[NJ];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        ra[u] = *reinterpret_cast<const float4*>(rs + (i + u) * 256 + c0);
                        rb[u] = *reinterpret_cast<const float4*>(rs + (i + u) * 256 + 128 + c0);
                    }
#pragma unroll
                    for (int j = 0; j < NJ; ++j)
                        xv[j] = *reinterpret_cast<const float4*>(xs + (size_t)j * kWarps * 256 + i);
#pragma unroll
                    for (int j = 0; j < NJ; ++j) {
                        {
                            const float xq[4] = {xv[j].x, xv[j].y, xv[j].z, xv[j].w};
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                acc[j][0] = __fmaf_rn(xq[u], ra[u].x, acc[j][0]);
                                acc[j][1] = __fmaf_rn(xq[u], ra[u].y, acc[j][1]);
                                acc[j][2] = __fmaf_rn(xq[u], ra[u].z, acc[j][2]);
                                acc[j][3] = __fmaf_rn(xq[u], ra[u].w, acc[j][3]);
                                acc[j][4] = __fmaf_rn(xq[u], rb[u].x, acc[j][4]);
                                acc[j][5] = __fmaf_rn(xq[u], rb[u].y, acc[j][5]);
                                acc[j][6] = __fmaf_rn(xq[u], rb[u].z, acc[j][6]);
                                acc[j][7] = __fmaf_rn(xq[u], rb[u].w, acc[j][7]);
                            }
                        }
                    }
                }
            }
            __syncthreads();   // every warp is done with this R slot (and, at s = 7, the rows)
            if (tid == 0 && abort_flag == 0) {
                if (rissued < nslices) issue_r(rissued++);
                if (s == kSlices - 1 && xissued < nmine) issue_x(xissued++);
            }
        }
        ok = __syncthreads_and(ok) != 0;
        // ---------------------------------------------------------------- row maxima
        if (ok) {
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
                if (warp + kWarps * j < ngr) {
                    float mx = 0.f;
#pragma unroll
                    for (int c = 0; c < 8; ++c) mx = fmax_nan(mx, fabsf(acc[j][c]));
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) mx = fmax_nan(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                    const int gr = warp + kWarps * j;
                    if (lane == 0) atomicMax(&amax_sh[gr / p.gpr], __float_as_uint(mx));
                }
            }
        }
        __syncthreads();
        if (tid < p.RB) {
            const float sc0 = scale_in ? *scale_in : __fdiv_rn(__uint_as_float(amax_sh[tid]), (float)p.qmax);
            const float sc = sc0 < FLT_MIN ? FLT_MIN : sc0;   // lower clamp; NaN stays NaN
            const RowDivisor dv(sc, p.qmax);
            row_s[tid] = sc;
            row_r[tid] = dv.r;
            if (ok && m0 + tid < p.M) scales[m0 + tid] = sc;
            amax_sh[tid] = 0u;
        }
        __syncthreads();
        // ---------------------------------------------------------------- codes
        if (ok) {
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
                if (warp + kWarps * j < ngr) {
                    const int gr = warp + kWarps * j;
                    const int m = gr / p.gpr, gi = gr - m * p.gpr;
                    if (m0 + m < p.M) {
                        RowDivisor dv(row_s[m], p.qmax);
                        dv.r = row_r[m];
                        int q[8];
#pragma unroll
                        for (int c = 0; c < 8; ++c) q[c] = quant_code_fast(acc[j][c], dv);
                        int8_t* dst = codes + (m0 + m) * p.ldq + (int64_t)gi * 256 + c0;
                        if (p.vec_codes) {
                            *reinterpret_cast<uint32_t*>(dst) = pack4_codes(q[0], q[1], q[2], q[3]);
                            *reinterpret_cast<uint32_t*>(dst + 128) = pack4_codes(q[4], q[5], q[6], q[7]);
                        } else {
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                dst[c] = (int8_t)q[c];
                                dst[128 + c] = (int8_t)q[4 + c];
                            }
                        }
                    }
                }
            }
        }
    }
    // after a timeout, copies still in flight land before the CTA leaves
    if (tid == 0 && abort_flag != 0) {
        for (int b = xissued > 2 ? xissued - 2 : 0; b < xissued; ++b)
            mbar_wait(&xfull[b & 1], (uint32_t)(b >> 1) & 1u, nullptr, nullptr);
        for (int n = rissued > 2 ? rissued - 2 : 0; n < rissued; ++n)
            mbar_wait(&rfull[n & 1], (uint32_t)(n >> 1) & 1u, nullptr, nullptr);
    }
    __syncthreads();
}

// fp32, g = 256, unit K stride, 16-byte-aligned x, R and row pitch, K / 256 <= 64.  Returns
// CK_ERR_UNSUPPORTED when the shape does not fit.
ck_status launch_rq_f32_ffma256(const void* x, int64_t M, int64_t K, int64_t sm, int64_t sk,
                                const void* R, const float* scale_in, int8_t* codes, int64_t ldq,
                                float* scales, int qmax, int* dev_status, cudaStream_t stream) {
    using namespace rqf256;
    if (sk != 1 || !aligned(x, 16) || !aligned(R, 16) || K % 256 != 0 || K / 256 > kMaxGR ||
        (M > 1 && (sm % 4 != 0 || sm < K)) || M >= (1LL << 31))
        return CK_ERR_UNSUPPORTED;
    const int gpr = (int)(K / 256);
    int64_t rb = kMaxGR / gpr;
    if (rb > kMaxRB) rb = kMaxRB;
    const int64_t spread = (M + num_sms() - 1) / num_sms();   // small M: a block per SM
    if (rb > spread) rb = spread < 1 ? 1 : spread;
    if (rb > M) rb = M;
    RqF256Params p;
    p.M = M;
    p.K = K;
    p.ldq = ldq;
    p.RB = (int)rb;
    p.gpr = gpr;
    p.nblocks = (M + rb - 1) / rb;
    p.box_bytes = (uint32_t)(rb * K * 4);
    p.vec_codes = (aligned(codes, 4) && ldq % 4 == 0) ? 1 : 0;
    p.qmax = qmax;

    CUtensorMap xm, rm;
    {
        const uint64_t dims[3] = {256, (uint64_t)gpr, (uint64_t)M};
        const uint64_t strides[2] = {1024, (uint64_t)(M > 1 ? sm : K) * 4};
        const uint32_t box[3] = {256, (uint32_t)gpr, (uint32_t)rb};
        const ck_status st = encode_tma(&xm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, x, dims, strides,
                                        box, CU_TENSOR_MAP_SWIZZLE_NONE);
        if (st != CK_OK) return st;
    }
    {
        // R as (c, i): a box is kSlice rows i of all 256 channels
        const uint64_t dims[2] = {256, 256};
        const uint64_t strides[1] = {1024};
        const uint32_t box[2] = {256, (uint32_t)kSlice};
        const ck_status st = encode_tma(&rm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, R, dims, strides,
                                        box, CU_TENSOR_MAP_SWIZZLE_NONE);
        if (st != CK_OK) return st;
    }
    const int nj = (int)((rb * gpr + kWarps - 1) / kWarps);   // group-rows a warp, 1 .. 8
    const size_t smem = 128 + 2 * (size_t)kSliceBytes + 2 * (size_t)nj * kWarps * 1024;
    const int grid = (int)(p.nblocks < num_sms() ? p.nblocks : num_sms());
    auto run = [&](auto kern) -> ck_status {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return CK_ERR_CUDA;
        kern<<<grid, kThreads, smem, stream>>>(xm, rm, scale_in, codes, scales, p, dev_status);
        return cudaGetLastError() == cudaSuccess ? CK_OK : CK_ERR_CUDA;
    };
    switch (nj) {
        case 1: return run(rq_f32_ffma256_kernel<1>);
        case 2: return run(rq_f32_ffma256_kernel<2>);
        case 3: return run(rq_f32_ffma256_kernel<3>);
        case 4: return run(rq_f32_ffma256_kernel<4>);
        case 5: return run(rq_f32_ffma256_kernel<5>);
        case 6: return run(rq_f32_ffma256_kernel<6>);
        case 7: return run(rq_f32_ffma256_kernel<7>);
        default: return run(rq_f32_ffma256_kernel<8>);
    }
}

}  // namespace ck
