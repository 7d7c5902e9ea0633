// ck_w4a4_splitk.cu -- stage 2 for few activation rows (M <= 64): the same INT4 x INT4 GEMM
// and epilogue as ck_w4a4_gemm.cu, with K split over a thread-block cluster so that the
// packed weights stream from HBM on many SMs at once.
//
// Operation (comfy-kitchen PR #198 "Consolidate INT8, RotateQuant, RoPE and ConvRot W4A4
// backends", "W4A4 correctness and performance scope"; decode-sized batches as in PR #193
// "HIP port of #191: W6A8 decode in the W4A8 kernels"):
//   acc[m, n] = sum_k q[m, k] * w[n, k]                  (exact INT32)
//   out[m, n] = cvt(((fp32(acc) * a_scale[m]) * w_scale[n]) + bias[n])
//
// With few rows the work is a weight read: 128-channel tiles give only N / 128 CTAs (30 for
// N = 3840).  Here each tile's K is split over a cluster of S CTAs (S * N / 128 ~ one CTA per
// SM), and each CTA:
//   warps 0, 2  issue TMA copies of the CTA's whole K range at once, one box per lane: packed
//               weights (warp 0; 128 rows x 64 bytes per k-block, 64-byte swizzle) and codes
//               (warp 2; BNA rows x 128 bytes, 128-byte swizzle), two k-blocks per box, one
//               mbarrier per box; the codes only once the kernel before this one (stage 1,
//               of which this kernel is the programmatic dependent) has completed, so the
//               weights stream in and are expanded while stage 1 still runs;
//   warps 4-7   expand the weight nibbles (one weight row per thread) into tensor memory in
//               chunks of up to six k-blocks, the MMA's A operand, then read the accumulator;
//   warp 1      allocates tensor memory and issues tcgen05.mma kind::i8 (128 x BNA x 32, A from
//               tensor memory) into one INT32 accumulator;
// then every CTA writes its partial accumulator to shared memory, and after a cluster barrier
// each CTA sums its share of the tile over all S partials through distributed shared memory
// (integer addition: exact and order-free), applies the epilogue and stores the outputs.
// Every CTA takes both cluster barriers whatever happened before them, so none waits for a
// CTA that left; every mbarrier wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "ck_device.cuh"
#include "ck_gemm_common.cuh"
#include "ck_internal.h"

namespace ck {

namespace splitk {
constexpr int BW = 128;                      // weight rows (channels) per tile: MMA M
constexpr int BK = 128;                      // K elements per k-block
constexpr int THREADS = 256;
constexpr int WARP_TMA = 0, WARP_MMA = 1, WARP_TMA2 = 2, UNP_WARP0 = 4;
constexpr int KB_MAX = 32;                   // k-blocks of one CTA held in shared memory
constexpr int CHUNK_KB = 6;                  // k-blocks expanded into tensor memory at a time
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t ACC_COL = CHUNK_KB * 32;  // accumulator columns [192, 192 + BNA)
constexpr int MAX_CLUSTER = 8;
constexpr int MAX_M = 64;
constexpr uint32_t W_BYTES = BW * BK / 2;    // 8 KB per k-block
constexpr size_t SMEM_BUDGET = 220 * 1024;
static_assert(ACC_COL + MAX_M <= TMEM_COLS, "accumulator fits the allocation");
}  // namespace splitk

struct SplitKParams {
    int64_t M, N;
    int num_kb;          // k-blocks of K
    int kb_per;          // k-blocks per cluster rank (the last rank may have fewer)
    int BNA;             // activation rows, a multiple of 16: the MMA's N
    int box3d;           // 1: (byte, row, k-block) boxes of two k-blocks; 0: one box per k-block
    uint32_t x_bytes;    // BNA * 128: one k-block of codes
    uint32_t idesc;
    const float* a_scale;
    const void* w_scale;
    const void* bias;
    OutSegs segs;        // where each channel's outputs go
    int* dev_status;
};

template <typename OutT, typename ScaleT, bool X16>
__global__ void __launch_bounds__(splitk::THREADS, 1)
    w4a4_splitk_kernel(const __grid_constant__ CUtensorMap xmap,
                       const __grid_constant__ CUtensorMap wmap, SplitKParams p) {
    using namespace splitk;
    extern __shared__ __align__(1024) unsigned char sk_smem[];
    unsigned char* base = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(sk_smem) + 1023) & ~uintptr_t(1023));
    const int kb_slots = (p.kb_per + 1) & ~1;    // box pairs may fill one k-block past the range
    unsigned char* wbuf = base;
    unsigned char* xbuf = wbuf + (size_t)kb_slots * W_BYTES;
    int32_t* partial = reinterpret_cast<int32_t*>(xbuf + (size_t)kb_slots * p.x_bytes);  // [BNA][128]

    // w_full[i] / x_full[i]: the weights / codes of k-block pair i have landed
    __shared__ __align__(8) uint64_t w_full[KB_MAX / 2], x_full[KB_MAX / 2], a_full, chunk_done,
        acc_full, drain_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_ctarank(), ncta = cluster_nctarank();
    const int kb_lo = (int)rank * p.kb_per;
    const int n_kb = (p.num_kb - kb_lo) < p.kb_per ? (p.num_kb - kb_lo) : p.kb_per;
    const int npairs = (n_kb + 1) / 2;
    const int nchunks = (n_kb + CHUNK_KB - 1) / CHUNK_KB;
    const int n0 = (int)blockIdx.y * BW;

    if (tid == 0) {
        for (int i = 0; i < KB_MAX / 2; ++i) {
            mbar_init(&w_full[i], 1);
            mbar_init(&x_full[i], 1);
        }
        mbar_init(&a_full, 4);
        mbar_init(&chunk_done, 1);
        mbar_init(&acc_full, 1);
        mbar_init(&drain_bar, 1);
        abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&xmap);
        tma_prefetch_desc(&wmap);
    }
    if (warp == WARP_MMA) {
        tmem_alloc(&tmem_base_sh, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_sh;
    // a kernel launched as this one's programmatic dependent (the next linear's stage 1) may
    // set up on the SMs this kernel leaves: after every CTA holds its tensor memory
    grid_dependents_launch();

    if (warp == WARP_TMA || warp == WARP_TMA2) {
        // ---------------------------------------------------------------- TMA: the whole range
        // lane i of warp WARP_TMA brings pair i's weights, lane i of warp WARP_TMA2 its codes,
        // each on its own barrier: one box per issuing thread, so the copies do not queue
        // behind one another.  The codes may be the output of the kernel before this one (its
        // programmatic dependent launch lets the weights stream and expand meanwhile).
        uint64_t* bar = warp == WARP_TMA ? w_full : x_full;
        const uint32_t bytes = warp == WARP_TMA ? W_BYTES : p.x_bytes;
        if (warp == WARP_TMA2) grid_dependency_wait();
        for (int i = lane; i < npairs; i += 32) {
            const int kb = kb_lo + 2 * i;
            const uint32_t nk = p.box3d ? 2u : (uint32_t)((n_kb - 2 * i) < 2 ? (n_kb - 2 * i) : 2);
            mbar_arrive_expect_tx(&bar[i], nk * bytes);
            if (p.box3d) {
                if (warp == WARP_TMA)
                    tma_load_3d(wbuf + (size_t)(2 * i) * W_BYTES, &wmap, &bar[i], 0, n0, kb);
                else
                    tma_load_3d(xbuf + (size_t)(2 * i) * p.x_bytes, &xmap, &bar[i], 0, 0, kb);
            } else {
                for (uint32_t j = 0; j < nk; ++j) {
                    if (warp == WARP_TMA)
                        tma_load_2d(wbuf + (size_t)(2 * i + j) * W_BYTES, &wmap, &bar[i],
                                    (kb + (int)j) * (BK / 2), n0);
                    else
                        tma_load_2d(xbuf + (size_t)(2 * i + j) * p.x_bytes, &xmap, &bar[i],
                                    (kb + (int)j) * BK, 0);
                }
            }
        }
    } else if (warp == WARP_MMA) {
        // ---------------------------------------------------------------- MMA issuer
        // the warp walks the chunks together (votes make each wait's outcome uniform, so the
        // MMA operands are computed uniformly); one elected lane issues every MMA and commit.
        // Its waits start once the kernel before this one has completed.
        grid_dependency_wait();
        const bool leader = elect_one();
        const uint64_t bdesc0 = smem_desc_k_sw128(smem_u32(xbuf));
        const uint32_t kstep = p.x_bytes >> 4;
        bool ok = true;
        for (int c = 0; ok && c < nchunks; ++c) {
            if (!__all_sync(0xffffffffu, mbar_wait(&a_full, (uint32_t)c & 1u, &abort_flag, p.dev_status))) {
                ok = false;
                break;
            }
            const int kb0 = c * CHUNK_KB;
            const int nc = (n_kb - kb0) < CHUNK_KB ? (n_kb - kb0) : CHUNK_KB;
            // the codes of the chunk landed
            for (int i = kb0 / 2; i <= (kb0 + nc - 1) / 2; ++i)
                if (!__all_sync(0xffffffffu, mbar_wait(&x_full[i], 0, &abort_flag, p.dev_status))) ok = false;
            if (!ok) break;
            tc_fence_after();
            if (leader) {
                for (int j = 0; j < nc; ++j) {
                    const int kb = kb0 + j;
                    const uint64_t bdesc = bdesc0 + (uint64_t)((uint32_t)kb * kstep);
#pragma unroll
                    for (int kk = 0; kk < BK / 32; ++kk)
                        tc_mma_i8_ts(tmem_base + ACC_COL, tmem_base + (uint32_t)(32 * j + 8 * kk),
                                     bdesc + (uint64_t)(kk * 2), p.idesc,
                                     (kb | kk) != 0 ? 1u : 0u);
                }
                tc_commit(&chunk_done);
            }
            __syncwarp();
        }
        if (leader) {
            if (ok) tc_commit(&acc_full);
            // every MMA issued above has completed once drain_bar flips
            tc_commit(&drain_bar);
            mbar_wait(&drain_bar, 0, nullptr, p.dev_status);
        }
        __syncwarp();
    } else if (warp >= UNP_WARP0) {
        // ---------------------------------------------------------------- expand, accumulate
        const int q = warp & 3;                    // TMEM lanes 32 q .. 32 q + 31
        const int r = q * 32 + lane;               // the thread's weight row in the tile
        const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16);
        // 16-byte chunk c of the row under the 64-byte swizzle: c ^ ((r / 2) % 4)
        const uint32_t sw = (uint32_t)((r >> 1) & 3);
        bool ok = true;
        for (int c = 0; ok && c < nchunks; ++c) {
            if (c > 0) {   // the chunk's tensor memory is free once the previous chunk's MMAs ended
                grid_dependency_wait();   // MMAs that need the codes
                if (!__all_sync(0xffffffffu, mbar_wait(&chunk_done, (uint32_t)(c - 1) & 1u,
                                                       &abort_flag, p.dev_status))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
            }
            const int kb0 = c * CHUNK_KB;
            const int nc = (n_kb - kb0) < CHUNK_KB ? (n_kb - kb0) : CHUNK_KB;
            for (int j = 0; j < nc; ++j) {
                const int kb = kb0 + j;
                if (!__all_sync(0xffffffffu, mbar_wait(&w_full[kb >> 1], 0, &abort_flag,
                                                       p.dev_status))) {
                    ok = false;
                    break;
                }
                const unsigned char* wrow = wbuf + (size_t)kb * W_BYTES + (size_t)r * 64;
                uint32_t v[32];
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const uint4 u = *reinterpret_cast<const uint4*>(wrow + ((((uint32_t)h) ^ sw) << 4));
                    const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        if (X16) unpack_word_x16(w4[i], v[8 * h + 2 * i], v[8 * h + 2 * i + 1]);
                        else unpack_word_s(w4[i], v[8 * h + 2 * i], v[8 * h + 2 * i + 1]);
                    }
                }
                tc_st_32x32b_x16(t_row + (uint32_t)(32 * j), *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
                tc_st_32x32b_x16(t_row + (uint32_t)(32 * j + 16), *reinterpret_cast<uint32_t(*)[16]>(&v[16]));
            }
            tc_wait_st();
            if (!ok) break;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&a_full);
        }
        tc_wait_st();
        // the CTA's partial accumulator, transposed into shared memory as [row m][channel]
        if (ok && __all_sync(0xffffffffu, mbar_wait(&acc_full, 0, &abort_flag, p.dev_status))) {
            tc_fence_after();
            for (int m0 = 0; m0 < p.BNA; m0 += 16) {
                uint32_t a[16];
                tc_ld_32x32b_x16(t_row + ACC_COL + (uint32_t)m0, a);
                tc_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) partial[(m0 + i) * BW + r] = (int32_t)a[i];
            }
        }
        tc_fence_before();
    }

    // ---------------------------------------------------------------- cluster reduction
    __syncthreads();
    if (ncta > 1) cluster_sync_all();
    grid_dependency_wait();   // the row scales, as the codes
    if (!abort_flag) {
        // this CTA's share of the tile's 4-channel vectors: [lo, hi) of BNA * 32
        const int nvec = p.BNA * (BW / 4);
        const int lo = (int)(((int64_t)nvec * rank) / ncta), hi = (int)(((int64_t)nvec * (rank + 1)) / ncta);
        for (int vi = lo + tid; vi < hi; vi += THREADS) {
            const int m = vi / (BW / 4), c4 = (vi % (BW / 4)) * 4;
            if ((int64_t)m >= p.M) continue;
            int32_t s[4] = {0, 0, 0, 0};
            for (uint32_t qr = 0; qr < ncta; ++qr) {
                const uint4 u = dsmem_load_v4(partial + m * BW + c4, qr);
                s[0] += (int32_t)u.x;
                s[1] += (int32_t)u.y;
                s[2] += (int32_t)u.z;
                s[3] += (int32_t)u.w;
            }
            const float a_s = __ldg(p.a_scale + m);
            int sg = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int64_t n = (int64_t)n0 + c4 + e;
                if (n >= p.N) break;
                while (sg + 1 < p.segs.n && n >= p.segs.start[sg + 1]) ++sg;
                const int acc = X16 ? (s[e] >> 4) : s[e];   // exact: 16 divides the sum
                float o = __int2float_rn(acc);
                o = __fmul_rn(o, a_s);
                o = __fmul_rn(o, load_scale<ScaleT>(p.w_scale, n));
                if (p.bias) o = __fadd_rn(o, load_scale<ScaleT>(p.bias, n));
                OutStore<OutT>::one(static_cast<OutT*>(p.segs.ptr[sg]) + m * p.segs.ldo[sg] +
                                        (n - p.segs.start[sg]), o);
            }
        }
    }
    // no CTA leaves while a peer may still read its partial accumulator, nor with a copy of its
    // own still landing (after a timeout the copies were never waited for)
    if (ncta > 1) cluster_sync_all();
    if (warp == WARP_TMA && lane == 0 && abort_flag)
        for (int i = 0; i < npairs; ++i) {
            mbar_wait(&w_full[i], 0, nullptr, nullptr);
            mbar_wait(&x_full[i], 0, nullptr, nullptr);
        }
    __syncthreads();
    if (warp == WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

template <typename OutT, typename ScaleT>
static ck_status splitk_launch_typed(const CUtensorMap& xmap, const CUtensorMap& wmap,
                                     const SplitKParams& p, int S, int tiles_n, size_t smem,
                                     bool x16, bool dep, cudaStream_t stream) {
    auto kern = x16 ? w4a4_splitk_kernel<OutT, ScaleT, true> : w4a4_splitk_kernel<OutT, ScaleT, false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return CK_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3((unsigned)S, (unsigned)tiles_n, 1);
    cfg.blockDim = dim3(splitk::THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int max_clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg) != cudaSuccess || max_clusters < 1)
        return CK_ERR_UNSUPPORTED;
    cfg.numAttrs = dep ? 2 : 1;
    if (cudaLaunchKernelEx(&cfg, kern, xmap, wmap, p) != cudaSuccess) return CK_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? CK_OK : CK_ERR_CUDA;
}

template <typename OutT>
static ck_status splitk_launch_out(const CUtensorMap& xmap, const CUtensorMap& wmap,
                                   const SplitKParams& p, int S, int tiles_n, size_t smem,
                                   bool x16, bool dep, ck_dtype scale_dt, cudaStream_t stream) {
    switch (scale_dt) {
        case CK_F32:
            return splitk_launch_typed<OutT, float>(xmap, wmap, p, S, tiles_n, smem, x16, dep,
                                                    stream);
        case CK_F16:
            return splitk_launch_typed<OutT, __half>(xmap, wmap, p, S, tiles_n, smem, x16, dep,
                                                     stream);
        case CK_BF16:
            return splitk_launch_typed<OutT, __nv_bfloat16>(xmap, wmap, p, S, tiles_n, smem, x16,
                                                            dep, stream);
        default: return CK_ERR_INVALID_ARG;
    }
}

ck_status launch_w4a4_splitk(const int8_t* codes, int64_t ldq, const float* a_scale, int64_t M,
                             int64_t K, const int8_t* w_packed, int64_t w_ld, int64_t N,
                             const void* w_scale, ck_dtype scale_dt, const void* bias,
                             const OutSegs& segs, ck_dtype out_dt, bool after_stage1,
                             int* dev_status, cudaStream_t stream) {
    using namespace splitk;
    if (M < 1 || M > MAX_M || N < 1) return CK_ERR_UNSUPPORTED;
    const int sms = num_sms();
    SplitKParams p;
    p.M = M;
    p.N = N;
    p.num_kb = (int)((K + BK - 1) / BK);
    p.BNA = (int)((M + 15) / 16 * 16);
    p.x_bytes = (uint32_t)p.BNA * BK;
    p.box3d = K % BK == 0 ? 1 : 0;
    const int64_t tiles_n = (N + BW - 1) / BW;
    if (tiles_n >= 65536) return CK_ERR_UNSUPPORTED;
    // about one CTA per SM: S splits per tile, each holding its whole K range in shared memory
    int S = (int)((sms + tiles_n - 1) / tiles_n);
    if (S > MAX_CLUSTER) S = MAX_CLUSTER;
    if (S > p.num_kb) S = p.num_kb;
    if (S < 1) S = 1;
    auto smem_for = [&](int kb_per) {
        const int slots = (kb_per + 1) & ~1;
        return (size_t)slots * (W_BYTES + p.x_bytes) + (size_t)p.BNA * BW * 4 + 1024;
    };
    int kb_per = (p.num_kb + S - 1) / S;
    while ((kb_per > KB_MAX || smem_for(kb_per) > SMEM_BUDGET) && S < MAX_CLUSTER) {
        ++S;
        kb_per = (p.num_kb + S - 1) / S;
    }
    if (kb_per > KB_MAX || smem_for(kb_per) > SMEM_BUDGET) return CK_ERR_UNSUPPORTED;
    S = (p.num_kb + kb_per - 1) / kb_per;   // every rank has at least one k-block
    p.kb_per = kb_per;
    p.idesc = idesc_i8(BW, p.BNA);
    p.a_scale = a_scale;
    p.w_scale = w_scale;
    p.bias = bias;
    p.segs = segs;
    p.dev_status = dev_status;

    CUtensorMap xmap, wmap;
    ck_status st;
    if (p.box3d) {
        const uint64_t dims[3] = {(uint64_t)BK, (uint64_t)M, (uint64_t)p.num_kb};
        const uint64_t strides[2] = {(uint64_t)ldq, (uint64_t)BK};
        const uint32_t box[3] = {BK, (uint32_t)p.BNA, 2};
        st = encode_tma(&xmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, codes, dims, strides, box,
                        CU_TENSOR_MAP_SWIZZLE_128B);
        if (st != CK_OK) return st;
        const uint64_t wdims[3] = {(uint64_t)(BK / 2), (uint64_t)N, (uint64_t)p.num_kb};
        const uint64_t wstrides[2] = {(uint64_t)w_ld, (uint64_t)(BK / 2)};
        const uint32_t wbox[3] = {BK / 2, BW, 2};
        st = encode_tma(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, w_packed, wdims, wstrides, wbox,
                        CU_TENSOR_MAP_SWIZZLE_64B);
    } else {
        const uint64_t dims[2] = {(uint64_t)K, (uint64_t)M};
        const uint64_t strides[1] = {(uint64_t)ldq};
        const uint32_t box[2] = {BK, (uint32_t)p.BNA};
        st = encode_tma(&xmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, codes, dims, strides, box,
                        CU_TENSOR_MAP_SWIZZLE_128B);
        if (st != CK_OK) return st;
        const uint64_t wdims[2] = {(uint64_t)(K / 2), (uint64_t)N};
        const uint64_t wstrides[1] = {(uint64_t)w_ld};
        const uint32_t wbox[2] = {BK / 2, BW};
        st = encode_tma(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, w_packed, wdims, wstrides, wbox,
                        CU_TENSOR_MAP_SWIZZLE_64B);
    }
    if (st != CK_OK) return st;
    const size_t smem = smem_for(kb_per);
    const bool x16 = K <= (1LL << 21) - 1;
    switch (out_dt) {
        case CK_F32:
            return splitk_launch_out<float>(xmap, wmap, p, S, (int)tiles_n, smem, x16,
                                            after_stage1, scale_dt, stream);
        case CK_F16:
            return splitk_launch_out<__half>(xmap, wmap, p, S, (int)tiles_n, smem, x16,
                                             after_stage1, scale_dt, stream);
        case CK_BF16:
            return splitk_launch_out<__nv_bfloat16>(xmap, wmap, p, S, (int)tiles_n, smem, x16,
                                                    after_stage1, scale_dt, stream);
        default: return CK_ERR_INVALID_ARG;
    }
}

}  // namespace ck
