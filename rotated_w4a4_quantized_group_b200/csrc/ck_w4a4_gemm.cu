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
// Persistent, warp-specialised, one CTA per SM.  The unpacked weights are the MMA's A
// operand and live in tensor memory; the activation codes are its B operand, staged in
// shared memory by TMA.  A tile is 128 output channels x BNA activation rows (BNA <= 192)
// and is accumulated transposed, D[n, m] (TMEM lane = channel n, column = row m):
//   warps 0, 3  TMA producers of the codes, BNA rows x 128 bytes per k-block, 128-byte swizzle:
//               warp 0 the even k-blocks of each super-stage, warp 3 the odd ones
//   warp 2      TMA producer of the packed weights: 128 rows x 64 bytes, 64-byte swizzle
//   warps 8-23  unpack, in two sets of eight that take alternate super-stages: each thread
//               owns one weight row (a TMEM lane) and one half of each k-block's K; it expands
//               64 four-bit codes per k-block to bytes and writes them into the set's TMEM
//               weight buffer with tcgen05.st
//   warp 1      TMEM allocation and the MMAs: tcgen05.mma kind::i8 with A from TMEM, 128 x BNA
//               x 32 per instruction.  The whole warp walks the ring and takes every wait (a
//               vote makes each outcome uniform) and one elected lane issues; waits, fences
//               and commits cost far more than an MMA issue, so the ring is organised in
//               super-stages of G = 2 k-blocks: one wait for the codes, one for the weights and
//               one commit per 8 MMAs (INT8 weights, W8: G = 1, for a deeper shared-memory ring)
//   warps 4-7, 24-27  epilogue, two warps per TMEM lane quarter taking alternate 16-row
//               chunks: tcgen05.ld of the finished accumulator, fp32 scale/bias, and 16-byte
//               stores of 16 rows x 32 channels staged in shared memory, overlapped with the
//               MMAs of the next tile (two accumulators); the tile's row scales are loaded
//               before its accumulator is ready
// TMEM columns: accumulators [0, BNA) and [BNA, 2 BNA), then nb (2-4) weight buffers of G
// k-blocks (32 columns each).  Every role walks its ring indices incrementally.
//
// Launched after stage 1 inside the linear, the kernel is stage 1's programmatic dependent:
// the weight producer and the unpack start at once, and the roles that read stage 1's output
// (the code producers, the epilogue's row scales) or whose bounded waits would otherwise run
// while stage 1 still does (the MMA warp, the unpack from its first wait on an MMA, the weight
// producer from the super-stage whose slot needs such an unpack) first wait for stage 1 to
// complete (griddepcontrol.wait; at once when the kernel was launched normally).
//
// Weight bytes.  For K < 2^21 each code w is written as the byte 16 w (its nibble moved to
// the byte's high half: two logic operations per four codes instead of a sign extension);
// the exact accumulator 16 acc then fits in int32 (|16 acc| <= 16 * 64 * K < 2^31) and the
// epilogue recovers acc with an arithmetic shift.  Larger K uses sign-extended bytes.
//
// Every wait is bounded (ck_device.cuh); out-of-range rows, channels and K arrive as zeros
// from TMA and are masked at the store.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "ck_device.cuh"
#include "ck_gemm_common.cuh"
#include "ck_internal.h"

namespace ck {

namespace gemm {
constexpr int BW = 128;                  // weight rows (output channels) per tile: MMA M
constexpr int BK = 128;                  // K elements per stage (bytes of codes)
constexpr int BNA_MAX = 192;             // activation rows per tile: MMA N
constexpr int XS_MAX = 8;                // code super-stages in shared memory
constexpr int G_MAX = 2;                 // k-blocks per super-stage (one 3-D box of each operand)
constexpr int NB_MAX = 4;                // TMEM weight buffers (one super-stage each)
constexpr int W_ST_MAX = 2 * G_MAX;      // packed-weight k-block buffers: G per unpack set
constexpr int ND = 16;                   // super-stage completion barriers (> XS_MAX + 1)
constexpr uint32_t W_BYTES = BW * BK / 2;    // 8 KB
constexpr uint32_t A_STAGE_COLS = BK / 4;    // 32 TMEM columns of 4 bytes per stage
constexpr uint32_t TMEM_COLS = 512;
constexpr int WARP_TMA_X = 0, WARP_MMA = 1, WARP_TMA_W = 2, WARP_TMA_X2 = 3;
// epilogue: warps 4..7 and 24..27, two per TMEM lane quarter, taking alternate 16-row chunks
constexpr int EPI_WARP0 = 4, EPI_WARP1 = 24, EPI_WARPS = 8;
constexpr int UNP_WARP0 = 8, UNP_SET_WARPS = 8, UNP_SETS = 2;   // warps 8..23
constexpr int UNP_WARPS = UNP_SET_WARPS * UNP_SETS;
constexpr int THREADS = (EPI_WARP1 + 4) * 32;
constexpr int64_t SCALED16_MAX_K = (1LL << 21) - 1;   // 16 * 64 * K < 2^31
constexpr size_t SMEM_BUDGET = 220 * 1024;
// per epilogue warp: one 16-row x 32-channel chunk of outputs (fp32 at most) staged for
// 16-byte stores
constexpr uint32_t EPI_STAGE_BYTES = 16 * 32 * 4;
static_assert(UNP_WARP0 % 4 == 0 && EPI_WARP0 % 4 == 0 && EPI_WARP1 % 4 == 0,
              "TMEM lane quarters follow warp % 4");
static_assert(UNP_WARP0 + UNP_WARPS == EPI_WARP1, "warp roles tile the CTA");
static_assert(BNA_MAX % 32 == 0, "the epilogue preloads row scales 32 rows at a time");
static_assert(UNP_SETS == 2, "the packed-weight stages are split between two unpack sets");
static_assert(ND == 16 && ND > XS_MAX + 1, "completion barrier index and parity use 4 bits");
}  // namespace gemm

struct GemmParams {
    int64_t M, N;
    int num_kb;        // K blocks of BK
    int nss;           // super-stages per tile: ceil(num_kb / G)
    int box3d;         // 1: one TMA box per super-stage (K % BK == 0), 0: one per k-block
    int BNA;           // activation rows per tile (multiple of 16, <= BNA_MAX)
    int tiles_n;       // tiles along N (channels)
    int tiles;         // total tiles
    int G;             // k-blocks per super-stage
    int nb;            // TMEM weight buffers, 2 <= nb <= NB_MAX
    int xs;            // code super-stages in shared memory
    uint32_t idesc;    // MMA instruction descriptor for 128 x BNA
    const float* a_scale;
    const void* w_scale;
    const void* bias;
    OutSegs segs;      // where each channel's outputs go
    int* dev_status;
};

// W8: the W8A8 variant.  The weights are INT8 codes (N, K): TMA brings 128 rows x 128 bytes per
// k-block (128-byte swizzle) into a ring slot next to the codes' slot of the same super-stage,
// and the MMA reads them from shared memory as its A operand; no expansion, no tensor-memory
// weight buffers, and both producers arrive on the slot's barrier.
template <typename OutT, typename ScaleT, bool X16, bool W8>
__global__ void __launch_bounds__(gemm::THREADS, 1)
    w4a4_gemm_kernel(const __grid_constant__ CUtensorMap xmap,
                     const __grid_constant__ CUtensorMap wmap, GemmParams p) {
    using namespace gemm;
    extern __shared__ __align__(1024) unsigned char gemm_smem[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(gemm_smem) + 1023) & ~uintptr_t(1023));
    // packed-weight stage of k-block it: it % 2G, so each unpack set has its own G stages and
    // waits for their fills in order
    const uint32_t G = (uint32_t)p.G, XS = (uint32_t)p.xs, NB = (uint32_t)p.nb;
    const uint32_t x_bytes = (uint32_t)p.BNA * BK;          // one k-block of codes
    const uint32_t xss_bytes = G * x_bytes;                  // one super-stage
    unsigned char* x_ring = smem;
    unsigned char* w_ring = x_ring + (size_t)XS * xss_bytes;   // W8: XS slots of G k-blocks
    constexpr uint32_t W8_BYTES = BW * BK;                      // one INT8 weight k-block, 16 KB
    unsigned char* epi_stage = w_ring + (W8 ? (size_t)XS * G * W8_BYTES : (size_t)2 * G * W_BYTES);

    __shared__ __align__(8) uint64_t x_full[XS_MAX], w_full[UNP_SETS], w_empty[UNP_SETS];
    __shared__ __align__(8) uint64_t a_full[NB_MAX], done[ND];
    __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2], drain_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // super-stages this CTA runs: nss per tile (its tiles blockIdx.x, + gridDim.x, ...),
    // numbered 0.. across tiles; super-stage ss is k-blocks [s G, s G + n_k) of local tile
    // ss / nss, s = ss % nss, n_k = min(G, num_kb - s G)
    const uint32_t my_tiles =
        (uint32_t)((p.tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x);
    const uint32_t nss = (uint32_t)p.nss;
    const uint32_t my_ss = my_tiles * nss;
    auto ss_nk = [&](uint32_t ss) -> uint32_t {
        const uint32_t kb0 = (ss % nss) * G;
        return ((uint32_t)p.num_kb - kb0) < G ? ((uint32_t)p.num_kb - kb0) : G;
    };

    if (tid == 0) {
        // the two codes producers, and the INT8 weights producer (W8)
        for (int s = 0; s < XS_MAX; ++s) mbar_init(&x_full[s], W8 ? 3 : 2);
        for (int s = 0; s < UNP_SETS; ++s) {
            mbar_init(&w_full[s], 1);
            mbar_init(&w_empty[s], UNP_SET_WARPS);
        }
        for (int s = 0; s < NB_MAX; ++s) mbar_init(&a_full[s], UNP_SET_WARPS);
        for (int s = 0; s < ND; ++s) mbar_init(&done[s], 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&acc_full[s], 1);
            mbar_init(&acc_empty[s], EPI_WARPS);
        }
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
    const uint32_t a_col0 = 2u * (uint32_t)p.BNA;

    // super-stage s completes (all its MMAs done) on done[s % 16] with parity (s / 16) & 1
    auto wait_done = [&](uint32_t s) -> bool {
        return mbar_wait(&done[s & (ND - 1)], (s >> 4) & 1u, &abort_flag, p.dev_status);
    };

    if (warp == WARP_TMA_X || warp == WARP_TMA_X2) {
        // ---------------------------------------------------------------- codes producers
        // warp WARP_TMA_X brings the even k-blocks of each super-stage, warp WARP_TMA_X2 the
        // odd ones: one box per issuing thread and k-block, so two boxes load at once
        if (lane == 0) {
            grid_dependency_wait();   // the codes may be the output of the kernel before this one
            const uint32_t par = warp == WARP_TMA_X2 ? 1u : 0u;
            uint32_t issued = 0, slot = 0;
            bool ok = true;
            for (uint32_t ss = 0; ok && ss < my_ss; ++ss) {
                if (ss >= XS && !wait_done(ss - XS)) {
                    ok = false;
                    break;
                }
                const int t = (int)blockIdx.x + (int)(ss / nss) * (int)gridDim.x;
                const int32_t m0 = (t / p.tiles_n) * p.BNA;
                const int32_t kb0 = (int32_t)((ss % nss) * G);
                const uint32_t n_k = ss_nk(ss);
                unsigned char* dst = x_ring + (size_t)slot * xss_bytes;
                const uint32_t mine = n_k > par ? (n_k - par + 1) / 2 : 0;   // k-blocks par, par + 2, ..
                if (mine) {
                    mbar_arrive_expect_tx(&x_full[slot], mine * x_bytes);
                    for (uint32_t j = par; j < n_k; j += 2)
                        tma_load_2d(dst + (size_t)j * x_bytes, &xmap, &x_full[slot],
                                    (kb0 + (int32_t)j) * BK, m0);
                } else {
                    mbar_arrive(&x_full[slot]);
                }
                ++issued;
                if (++slot == XS) slot = 0;
            }
            if (!ok)   // copies still in flight land before the CTA leaves
                for (uint32_t j = issued > XS ? issued - XS : 0; j < issued; ++j)
                    mbar_wait(&x_full[j % XS], (j / XS) & 1u, nullptr, nullptr);
        }
    } else if (warp == WARP_TMA_W && W8) {
        // ---------------------------------------------------------------- INT8 W producer
        // super-stage ss fills weight slot ss % XS, on the codes' barrier of that slot
        if (lane == 0) {
            uint32_t issued = 0, slot = 0;
            bool ok = true;
            for (uint32_t ss = 0; ok && ss < my_ss; ++ss) {
                if (ss >= XS && !wait_done(ss - XS)) {
                    ok = false;
                    break;
                }
                const int t = (int)blockIdx.x + (int)(ss / nss) * (int)gridDim.x;
                const int32_t n0 = (t % p.tiles_n) * BW;
                const int32_t kb0 = (int32_t)((ss % nss) * G);
                const uint32_t n_k = ss_nk(ss);
                unsigned char* dst = w_ring + (size_t)slot * G * W8_BYTES;
                if (p.box3d) {
                    mbar_arrive_expect_tx(&x_full[slot], G * W8_BYTES);
                    tma_load_3d(dst, &wmap, &x_full[slot], 0, n0, kb0);
                } else {
                    mbar_arrive_expect_tx(&x_full[slot], n_k * W8_BYTES);
                    for (uint32_t j = 0; j < n_k; ++j)
                        tma_load_2d(dst + (size_t)j * W8_BYTES, &wmap, &x_full[slot],
                                    (kb0 + (int32_t)j) * BK, n0);
                }
                ++issued;
                if (++slot == XS) slot = 0;
            }
            if (!ok)
                for (uint32_t j = issued > XS ? issued - XS : 0; j < issued; ++j)
                    mbar_wait(&x_full[j % XS], (j / XS) & 1u, nullptr, nullptr);
        }
    } else if (warp == WARP_TMA_W) {
        // ---------------------------------------------------------------- packed W producer
        // super-stage ss fills the G k-block buffers of unpack set ss % 2 (fill ss / 2)
        if (lane == 0) {
            uint32_t issued = 0;
            bool ok = true;
            for (uint32_t ss = 0; ok && ss < my_ss; ++ss) {
                const uint32_t set = ss & 1u;
                // this wait needs the unpack warps' pass over super-stage ss - 2, which follows
                // their pass over ss - 4, which waited for the MMAs of ss - 4 - NB: MMAs that
                // need the codes, from the kernel before this one
                if (ss == NB + 2 * UNP_SETS) grid_dependency_wait();
                if (ss >= UNP_SETS &&
                    !mbar_wait(&w_empty[set], ((ss >> 1) - 1) & 1u, &abort_flag, p.dev_status)) {
                    ok = false;
                    break;
                }
                const int t = (int)blockIdx.x + (int)(ss / nss) * (int)gridDim.x;
                const int32_t n0 = (t % p.tiles_n) * BW;
                const int32_t kb0 = (int32_t)((ss % nss) * G);
                const uint32_t n_k = ss_nk(ss);
                unsigned char* dst = w_ring + (size_t)set * G * W_BYTES;
                if (p.box3d) {
                    mbar_arrive_expect_tx(&w_full[set], G * W_BYTES);
                    tma_load_3d(dst, &wmap, &w_full[set], 0, n0, kb0);
                } else {
                    mbar_arrive_expect_tx(&w_full[set], n_k * W_BYTES);
                    for (uint32_t j = 0; j < n_k; ++j)
                        tma_load_2d(dst + (size_t)j * W_BYTES, &wmap, &w_full[set],
                                    (kb0 + (int32_t)j) * (BK / 2), n0);
                }
                ++issued;
            }
            if (!ok)
                for (uint32_t j = issued > UNP_SETS ? issued - UNP_SETS : 0; j < issued; ++j)
                    mbar_wait(&w_full[j & 1u], (j >> 1) & 1u, nullptr, nullptr);
        }
    } else if (warp == WARP_MMA) {
        // ---------------------------------------------------------------- MMA issuer
        // The whole warp walks the ring and takes every wait (a vote makes each decision
        // uniform), so every value an MMA takes is computed uniformly across the warp; one lane,
        // elected once, issues all MMAs and commits (a commit tracks its own thread's MMAs).
        // Its waits start once the kernel before this one (stage 1) has completed, so none of
        // their time limits covers the rest of that kernel.
        grid_dependency_wait();
        const bool leader = elect_one();
        // descriptor of code k-block 0 of slot 0; k-block j of slot s starts
        // (s G + j) x_bytes later (start-address field counts 16-byte units)
        const uint64_t bdesc0 = smem_desc_k_sw128(smem_u32(x_ring));
        const uint32_t kstep = x_bytes >> 4;
        const uint64_t adesc0 = smem_desc_k_sw128(smem_u32(w_ring));   // W8 weights
        uint32_t slot = 0, xphase = 0, lt = 0;
        RingPos rb;   // TMEM weight buffer of the super-stage
        uint32_t d_tmem = tmem_base;
        for (uint32_t ss = 0; ss < my_ss; ++ss, rb.step(NB)) {
            if (!__all_sync(0xffffffffu, mbar_wait(&x_full[slot], xphase, &abort_flag, p.dev_status)))
                break;
            if (!W8 && !__all_sync(0xffffffffu, mbar_wait(&a_full[rb.idx], rb.phase, &abort_flag,
                                                          p.dev_status)))
                break;
            tc_fence_after();
            const uint32_t kb0 = (ss % nss) * G;
            const uint32_t n_k = ss_nk(ss);
            const uint32_t a_ss = tmem_base + a_col0 + rb.idx * G * A_STAGE_COLS;
            if (kb0 == 0) {
                // a new tile: its accumulator must have been drained by the epilogue
                const uint32_t acc = lt & 1u;
                if (lt >= 2 && !__all_sync(0xffffffffu, mbar_wait(&acc_empty[acc], ((lt >> 1) - 1) & 1u,
                                                                  &abort_flag, p.dev_status)))
                    break;
                tc_fence_after();
                d_tmem = tmem_base + acc * (uint32_t)p.BNA;
            }
            const bool last = kb0 + n_k == (uint32_t)p.num_kb;
            if (leader) {
                for (uint32_t j = 0; j < n_k; ++j) {
                    const uint64_t bdesc = bdesc0 + (uint64_t)((slot * G + j) * kstep);
                    const uint32_t a_tmem = a_ss + j * A_STAGE_COLS;
                    const uint64_t adesc = adesc0 + (uint64_t)((slot * G + j) * (W8_BYTES >> 4));
#pragma unroll
                    for (int kk = 0; kk < BK / 32; ++kk) {
                        // one MMA K step: 32 bytes of K = 8 TMEM columns of A (or 32 bytes of
                        // the 128-byte swizzled A row for W8), 32 bytes of the swizzled B row
                        const uint32_t acc_flag = ((kb0 + j) | (uint32_t)kk) != 0 ? 1u : 0u;
                        if (W8)
                            tc_mma_i8(d_tmem, adesc + (uint64_t)(kk * 2), bdesc + (uint64_t)(kk * 2),
                                      p.idesc, acc_flag);
                        else
                            tc_mma_i8_ts(d_tmem, a_tmem + (uint32_t)(kk * 8),
                                         bdesc + (uint64_t)(kk * 2), p.idesc, acc_flag);
                    }
                }
                if (last) tc_commit(&acc_full[lt & 1u]);
                tc_commit(&done[ss & (ND - 1)]);
            }
            __syncwarp();
            if (last) ++lt;
            if (++slot == XS) {
                slot = 0;
                xphase ^= 1u;
            }
        }
        // every MMA issued above has completed once drain_bar flips
        if (leader) {
            tc_commit(&drain_bar);
            mbar_wait(&drain_bar, 0, nullptr, p.dev_status);
        }
        __syncwarp();
    } else if (!W8 && warp >= UNP_WARP0 && warp < UNP_WARP0 + UNP_WARPS) {
        // ---------------------------------------------------------------- unpack into TMEM
        const int u = warp - UNP_WARP0;
        const int q = warp & 3;                        // TMEM lanes 32q .. 32q + 31
        const int h = (u >> 2) & 1;                    // K half of each k-block
        const uint32_t set = (uint32_t)(u / UNP_SET_WARPS);   // super-stages ss == set (mod 2)
        const int r = q * 32 + lane;                   // weight row of the tile
        // 16-byte chunks 2h and 2h + 1 of the row under the 64-byte swizzle (chunk index
        // XOR address bits 7-8, i.e. (r >> 1) & 3 for 64-byte rows)
        const uint32_t phase = (uint32_t)((r >> 1) & 3);
        const uint32_t off0 = (uint32_t)r * 64u + (((uint32_t)(2 * h) ^ phase) << 4);
        const uint32_t off1 = (uint32_t)r * 64u + (((uint32_t)(2 * h + 1) ^ phase) << 4);
        const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + a_col0 + (uint32_t)(h * 16);
        bool ok = true;
        uint32_t buf = set;   // TMEM weight buffer of super-stage ss: ss % NB
        const unsigned char* wset = w_ring + (size_t)set * G * W_BYTES;
        for (uint32_t ss = set; ok && ss < my_ss; ss += UNP_SETS) {
            const uint32_t t_buf = t_row + buf * G * A_STAGE_COLS;
            const uint32_t n_k = ss_nk(ss);
            // every lane waits; the warp leaves together (tcgen05.st below is .aligned)
            if (!__all_sync(0xffffffffu, mbar_wait(&w_full[set], (ss >> 1) & 1u, &abort_flag,
                                                   p.dev_status))) {
                ok = false;
                break;
            }
            uint4 c0[G_MAX], c1[G_MAX];
#pragma unroll
            for (uint32_t j = 0; j < (uint32_t)G_MAX; ++j) {
                if (j < n_k) {
                    const unsigned char* wst = wset + (size_t)j * W_BYTES;
                    c0[j] = *reinterpret_cast<const uint4*>(wst + off0);
                    c1[j] = *reinterpret_cast<const uint4*>(wst + off1);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&w_empty[set]);
            // expand into registers before waiting for the tensor-memory buffer, so that only
            // the stores lie between the MMAs of super-stage ss - NB completing and those of ss
            uint32_t v[G_MAX][16];
#pragma unroll
            for (uint32_t j = 0; j < (uint32_t)G_MAX; ++j) {
                if (j < n_k) {
                    const uint32_t c[8] = {c0[j].x, c0[j].y, c0[j].z, c0[j].w,
                                           c1[j].x, c1[j].y, c1[j].z, c1[j].w};
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        if (X16) unpack_word_x16(c[i], v[j][2 * i], v[j][2 * i + 1]);
                        else unpack_word_s(c[i], v[j][2 * i], v[j][2 * i + 1]);
                    }
                }
            }
            // the buffer is free once the MMAs of its previous super-stage (ss - NB) completed
            // (MMAs that need the codes: the wait starts after the kernel before this one)
            if (ss >= NB && ss < NB + UNP_SETS) grid_dependency_wait();   // once
            if (ss >= NB && !__all_sync(0xffffffffu, wait_done(ss - NB))) break;
            tc_fence_after();
#pragma unroll
            for (uint32_t j = 0; j < (uint32_t)G_MAX; ++j)
                if (j < n_k) tc_st_32x32b_x16(t_buf + j * A_STAGE_COLS, v[j]);
            tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&a_full[buf]);
            buf += UNP_SETS;
            if (buf >= NB) buf -= NB;
        }
        tc_wait_st();   // no tensor-memory store is pending when the CTA frees its columns
    } else if ((warp >= EPI_WARP0 && warp < EPI_WARP0 + 4) || warp >= EPI_WARP1) {
        // ---------------------------------------------------------------- epilogue
        const int q = warp & 3;                        // TMEM lanes 32q .. 32q + 31
        const int eh = warp >= EPI_WARP1 ? 1 : 0;      // rows 32k + 16 eh .. + 15 of each 32
        grid_dependency_wait();   // so may the row scales
        uint32_t lt = 0;
        for (int t = blockIdx.x; t < p.tiles; t += gridDim.x, ++lt) {
            const uint32_t acc = lt & 1u;
            const int64_t m0 = (int64_t)(t / p.tiles_n) * p.BNA;
            const int64_t n = (int64_t)(t % p.tiles_n) * BW + q * 32 + lane;   // channel
            const bool n_ok = n < p.N;
            const float ws = n_ok ? load_scale<ScaleT>(p.w_scale, n) : 0.f;
            const float bs = (p.bias && n_ok) ? load_scale<ScaleT>(p.bias, n) : 0.f;
            const int rows = (int)((p.M - m0) < p.BNA ? (p.M - m0) : p.BNA);
            // the tile's row scales, loaded before the accumulator is ready: lane l of
            // as_r[k] holds a_scale[m0 + 32k + l]
            float as_r[BNA_MAX / 32];
#pragma unroll
            for (int k = 0; k < BNA_MAX / 32; ++k)
                as_r[k] = (32 * k + lane < rows) ? __ldg(p.a_scale + m0 + 32 * k + lane) : 0.f;
            if (!__all_sync(0xffffffffu,
                            mbar_wait(&acc_full[acc], (lt >> 1) & 1u, &abort_flag, p.dev_status)))
                break;
            tc_fence_after();
            const uint32_t tacc = tmem_base + ((uint32_t)(q * 32) << 16) + acc * (uint32_t)p.BNA;
            // the lane's channel's output segment
            int sg = 0;
            while (n_ok && sg + 1 < p.segs.n && n >= p.segs.start[sg + 1]) ++sg;
            OutT* ocol = static_cast<OutT*>(p.segs.ptr[sg]) + (n_ok ? n - p.segs.start[sg] : 0);
            const int64_t ldo = p.segs.ldo[sg];
            // 16-byte stores from a staged chunk when the warp's 32 channels are all present, in
            // one segment, and every 16-byte piece of every row is aligned
            constexpr int PER16 = 16 / (int)sizeof(OutT);          // outputs per 16 bytes
            const int sg0 = __shfl_sync(0xffffffffu, sg, 0);
            // lane 0's column address: the warp's first channel
            const unsigned long long obits =
                __shfl_sync(0xffffffffu, (unsigned long long)reinterpret_cast<uintptr_t>(ocol), 0);
            const bool vec = __all_sync(0xffffffffu, n_ok && sg == sg0) && (obits % 16 == 0) &&
                             (ldo % PER16 == 0);
            OutT* stage = reinterpret_cast<OutT*>(epi_stage + (size_t)(q + 4 * eh) * EPI_STAGE_BYTES);
            OutT* obase = reinterpret_cast<OutT*>(static_cast<uintptr_t>(obits));
#pragma unroll
            for (int k = 0; k < BNA_MAX / 32; ++k) {
                const int c0 = 32 * k + 16 * eh;       // first row of this warp's chunk
                if (c0 < rows) {
                    uint32_t r[16];
                    tc_ld_32x32b_x16(tacc + (uint32_t)c0, r);
                    tc_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float a_s = __shfl_sync(0xffffffffu, as_r[k], 16 * eh + j);
                        const int accv = X16 ? ((int)r[j] >> 4) : (int)r[j];   // exact: 16 | acc
                        float o = __int2float_rn(accv);
                        o = __fmul_rn(o, a_s);
                        o = __fmul_rn(o, ws);
                        if (p.bias) o = __fadd_rn(o, bs);
                        if (vec) {
                            OutStore<OutT>::one(stage + j * 32 + lane, o);   // row j, channel lane
                        } else if (c0 + j < rows && n_ok) {
                            OutStore<OutT>::one(ocol + (m0 + c0 + j) * ldo, o);
                        }
                    }
                    if (vec) {
                        __syncwarp();
                        // 16 rows x 32 channels: 32 / PER16 pieces of 16 bytes a row
                        constexpr int PIECES = 32 / PER16;
                        for (int i = lane; i < 16 * PIECES; i += 32) {
                            const int row = i / PIECES, pc = i % PIECES;
                            if (c0 + row < rows)
                                *reinterpret_cast<uint4*>(obase + (m0 + c0 + row) * ldo + pc * PER16) =
                                    *reinterpret_cast<const uint4*>(stage + row * 32 + pc * PER16);
                        }
                        __syncwarp();
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
static ck_status launch_typed(const CUtensorMap& xmap, const CUtensorMap& wmap,
                              const GemmParams& p, size_t smem, int grid, bool x16, bool w8,
                              bool dependent, cudaStream_t stream) {
    auto kern = w8 ? w4a4_gemm_kernel<OutT, ScaleT, false, true>
                   : x16 ? w4a4_gemm_kernel<OutT, ScaleT, true, false>
                         : w4a4_gemm_kernel<OutT, ScaleT, false, false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return CK_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(gemm::THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = dependent ? 1 : 0;
    if (cudaLaunchKernelEx(&cfg, kern, xmap, wmap, p) != cudaSuccess) return CK_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? CK_OK : CK_ERR_CUDA;
}

template <typename OutT>
static ck_status launch_out(const CUtensorMap& xmap, const CUtensorMap& wmap, const GemmParams& p,
                            size_t smem, int grid, bool x16, bool w8, bool dep, ck_dtype scale_dt,
                            cudaStream_t stream) {
    switch (scale_dt) {
        case CK_F32:
            return launch_typed<OutT, float>(xmap, wmap, p, smem, grid, x16, w8, dep, stream);
        case CK_F16:
            return launch_typed<OutT, __half>(xmap, wmap, p, smem, grid, x16, w8, dep, stream);
        case CK_BF16:
            return launch_typed<OutT, __nv_bfloat16>(xmap, wmap, p, smem, grid, x16, w8, dep,
                                                     stream);
        default: return CK_ERR_INVALID_ARG;
    }
}

// Activation rows per tile: the multiple of 16 (<= 192) that minimises the persistent
// schedule's length, (tiles of the busiest CTA) x (BNA + a small per-tile overhead),
// preferring wider tiles on ties.
static int choose_bna(int64_t M, int64_t N, int sms) {
    const int64_t tiles_n = (N + gemm::BW - 1) / gemm::BW;
    int best = gemm::BNA_MAX;
    int64_t best_cost = -1;
    for (int bna = gemm::BNA_MAX; bna >= 16; bna -= 16) {
        const int64_t tiles = tiles_n * ((M + bna - 1) / bna);
        const int64_t per_cta = (tiles + sms - 1) / sms;
        const int64_t cost = per_cta * (bna + 32);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = bna;
        }
    }
    return best;
}

// The persistent GEMM for packed INT4 weights (w8 false, (N, K/2) bytes) or INT8 weights
// (w8 true, (N, K) bytes); codes and weights with 16-byte-aligned rows.
static ck_status launch_persistent(const int8_t* codes, int64_t ldq, const float* a_scale,
                                   int64_t M, int64_t K, const int8_t* w, int64_t w_ld, int64_t N,
                                   const void* w_scale, ck_dtype scale_dt, const void* bias,
                                   const OutSegs& segs, ck_dtype out_dt, bool w8, bool dep,
                                   int* dev_status, cudaStream_t stream) {
    using namespace gemm;
    const int sms = num_sms();
    GemmParams p;
    p.BNA = choose_bna(M, N, sms);
    const bool box3d = !w8 && K % BK == 0;
    const int num_kb = (int)((K + BK - 1) / BK);
    // weight bytes per row of one k-block: 64 packed (two codes a byte) or 128
    const uint32_t wkb = w8 ? BK : BK / 2;
    const CUtensorMapSwizzle wsw = w8 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    CUtensorMap xmap, wmap;
    // packed weights with whole 128-byte k-blocks: one 3-D box fetches the G = 2 k-blocks of a
    // super-stage, (byte of the k-block, row, k-block); otherwise one 2-D box per k-block, zero
    // past K.  INT8 weights (W8) take super-stages of one k-block: a ring slot then holds 40 KB
    // (codes and weights) instead of 80, five slots instead of two.
    const uint32_t G_box = 2;
    {
        // codes: one 2-D box (128 bytes x BNA rows) per k-block, zero past K and M
        const uint64_t dims[2] = {(uint64_t)K, (uint64_t)M};
        const uint64_t strides[1] = {(uint64_t)ldq};
        const uint32_t box[2] = {BK, (uint32_t)p.BNA};
        ck_status st = encode_tma(&xmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, codes, dims, strides,
                                  box, CU_TENSOR_MAP_SWIZZLE_128B);
        if (st != CK_OK) return st;
    }
    if (box3d) {
        const uint64_t wdims[3] = {(uint64_t)wkb, (uint64_t)N, (uint64_t)num_kb};
        const uint64_t wstrides[2] = {(uint64_t)w_ld, (uint64_t)wkb};
        const uint32_t wbox[3] = {wkb, BW, G_box};
        const ck_status st = encode_tma(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, w, wdims, wstrides,
                                        wbox, wsw);
        if (st != CK_OK) return st;
    } else {
        const uint64_t wdims[2] = {(uint64_t)(w8 ? K : K / 2), (uint64_t)N};
        const uint64_t wstrides[1] = {(uint64_t)w_ld};
        const uint32_t wbox[2] = {wkb, BW};
        const ck_status st = encode_tma(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, w, wdims,
                                        wstrides, wbox, wsw);
        if (st != CK_OK) return st;
    }
    p.M = M;
    p.N = N;
    p.num_kb = num_kb;
    p.box3d = box3d ? 1 : 0;
    p.tiles_n = (int)((N + BW - 1) / BW);
    const int64_t tiles = (int64_t)p.tiles_n * ((M + p.BNA - 1) / p.BNA);
    if (tiles >= (1LL << 31)) return CK_ERR_UNSUPPORTED;
    p.tiles = (int)tiles;
    // TMEM: two accumulators of BNA columns; for packed weights the rest holds the weight
    // buffers of G k-blocks (32 columns each), as many as fit (2..4): the unpack of a
    // super-stage may start once the MMAs of the super-stage nb before it completed
    p.G = w8 ? 1 : (int)G_box;   // the 3-D boxes above hold exactly one super-stage
    p.nb = w8 ? 2 : (int)((TMEM_COLS - 2u * (uint32_t)p.BNA) / ((uint32_t)p.G * A_STAGE_COLS));
    if (p.nb > NB_MAX) p.nb = NB_MAX;
    if (p.nb < 2) return CK_ERR_UNSUPPORTED;
    const size_t xss_bytes = (size_t)p.G * p.BNA * BK;
    size_t w_ring_bytes;
    if (w8) {
        // one INT8 weight super-stage per codes slot
        const size_t wss = (size_t)p.G * BW * BK;
        p.xs = (int)((SMEM_BUDGET - EPI_WARPS * EPI_STAGE_BYTES) / (xss_bytes + wss));
        if (p.xs > XS_MAX) p.xs = XS_MAX;
        w_ring_bytes = (size_t)p.xs * wss;
    } else {
        w_ring_bytes = (size_t)2 * p.G * W_BYTES;
        p.xs = (int)((SMEM_BUDGET - w_ring_bytes - EPI_WARPS * EPI_STAGE_BYTES) / xss_bytes);
        if (p.xs > XS_MAX) p.xs = XS_MAX;
    }
    if (p.G < 1 || p.xs < 2) return CK_ERR_UNSUPPORTED;
    p.nss = (p.num_kb + p.G - 1) / p.G;
    const size_t smem = (size_t)p.xs * xss_bytes + w_ring_bytes + EPI_WARPS * EPI_STAGE_BYTES + 1024;
    p.idesc = idesc_i8(BW, p.BNA);   // signed 8-bit A and B, s32 accumulator, 128 x BNA
    p.a_scale = a_scale;
    p.w_scale = w_scale;
    p.bias = bias;
    p.segs = segs;
    p.dev_status = dev_status;
    const int grid = (int)(p.tiles < sms ? p.tiles : sms);
    const bool x16 = !w8 && K <= SCALED16_MAX_K;
    switch (out_dt) {
        case CK_F32:
            return launch_out<float>(xmap, wmap, p, smem, grid, x16, w8, dep, scale_dt, stream);
        case CK_F16:
            return launch_out<__half>(xmap, wmap, p, smem, grid, x16, w8, dep, scale_dt, stream);
        case CK_BF16:
            return launch_out<__nv_bfloat16>(xmap, wmap, p, smem, grid, x16, w8, dep, scale_dt,
                                             stream);
        default: return CK_ERR_INVALID_ARG;
    }
}

ck_status launch_w4a4_gemm(const int8_t* codes, int64_t ldq, const float* a_scale, int64_t M,
                           int64_t K, const int8_t* w_packed, int64_t w_ld, int64_t N,
                           const void* w_scale, ck_dtype scale_dt, const void* bias,
                           const OutSegs& segs, ck_dtype out_dt, bool after_stage1,
                           int* dev_status, cudaStream_t stream) {
    if (M == 0 || N == 0) return CK_OK;
    if (M <= 64) {   // few rows: split K over clusters so the weights stream on every SM
        const ck_status st = launch_w4a4_splitk(codes, ldq, a_scale, M, K, w_packed, w_ld, N,
                                                w_scale, scale_dt, bias, segs, out_dt,
                                                after_stage1, dev_status, stream);
        if (st != CK_ERR_UNSUPPORTED) return st;
    }
    return launch_persistent(codes, ldq, a_scale, M, K, w_packed, w_ld, N, w_scale, scale_dt,
                             bias, segs, out_dt, false, after_stage1, dev_status, stream);
}

ck_status launch_w8a8_gemm(const int8_t* codes, int64_t ldq, const float* a_scale, int64_t M,
                           int64_t K, const int8_t* w, int64_t w_ld, int64_t N,
                           const void* w_scale, ck_dtype scale_dt, const void* bias,
                           const OutSegs& segs, ck_dtype out_dt, bool after_stage1,
                           int* dev_status, cudaStream_t stream) {
    if (M == 0 || N == 0) return CK_OK;
    return launch_persistent(codes, ldq, a_scale, M, K, w, w_ld, N, w_scale, scale_dt, bias, segs,
                             out_dt, true, after_stage1, dev_status, stream);
}

}  // namespace ck
