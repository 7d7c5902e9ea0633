// ck_device.cuh -- sm_100a device helpers: mbarriers with bounded waits, TMA tile
// loads, tcgen05 (TMEM alloc, MMA, commit, loads) and dtype conversions.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "ck.h"

namespace ck {

// A wait that spins longer than this many SM clock cycles (about a second at the
// B200's clocks) gives up, records CK_ERR_TIMEOUT and lets the kernel exit.
constexpr long long kWaitLimitCycles = 2000000000LL;

// The limit of a role's waits on its ring (every wait given an abort flag); the waits for
// copies and MMAs already in flight keep kWaitLimitCycles.  The library built for the expiry
// test sets it to 0: such a wait then gives up unless its phase is already complete, so the
// kernel takes its timeout path (record the status, stop issuing, drain what is in flight,
// free tensor memory, return) on an ordinary input.
#ifndef CK_ROLE_WAIT_LIMIT_CYCLES
#define CK_ROLE_WAIT_LIMIT_CYCLES 2000000000LL
#endif
constexpr long long kRoleWaitLimitCycles = CK_ROLE_WAIT_LIMIT_CYCLES;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void record_timeout(int* dev_status) {
    if (dev_status) atomicExch(dev_status, (int)CK_ERR_TIMEOUT);
}

// ------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Whether the phase with the given parity has completed, without waiting at all.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// try_wait that may suspend the thread (up to about 20 us) until the phase completes, so a
// waiting warp does not take issue slots from the working ones.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(20000u)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete.  Returns false (after
// recording a timeout) if it does not complete within kWaitLimitCycles, or as soon as
// *abort is seen set by another role of the CTA.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          int* dev_status) {
    const long long limit = abort ? kRoleWaitLimitCycles : kWaitLimitCycles;
    if (limit <= 0) {
        // the expiry-test build: give up unless the phase is already complete (try_wait may
        // suspend the thread for a while, during which most phases complete)
        if (mbar_test_wait(bar, parity)) return true;
        if (abort) *abort = 1;
        record_timeout(dev_status);
        return false;
    }
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait_sleep(bar, parity)) return true;
        if (abort && *abort) return false;
        if (clock64() - t0 > limit) {
            if (abort) *abort = 1;
            record_timeout(dev_status);
            return false;
        }
    }
}

// ------------------------------------------------------------------ Philox4x32-10

// Philox4x32-10 is the counter-based generator of Salmon, Moraes, Dror and Shaw ("Parallel
// random numbers: as easy as 1, 2, 3", SC 2011): ten rounds of two 32 x 32 -> 64-bit products
// mixed with the key, the key bumped by two Weyl constants between rounds.
// Word 0 of Philox4x32-10 of a 128-bit counter under a 64-bit key.
__device__ __forceinline__ uint32_t philox_word0(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                                 uint32_t k0, uint32_t k1) {
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        const uint32_t lo0 = 0xD2511F53u * c0, hi0 = __umulhi(0xD2511F53u, c0);
        const uint32_t lo1 = 0xCD9E8D57u * c2, hi1 = __umulhi(0xCD9E8D57u, c2);
        const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
        c0 = n0;
        c1 = lo1;
        c2 = n2;
        c3 = lo0;
    }
    return c0;
}

// philox_word0 for a run of counters (e, e >> 32, o0, o1) that differ only in e: the ten round
// keys and the first round's product of the fixed third word o0 are computed once per run.
struct PhiloxRun {
    uint32_t k0[10], k1[10];
    uint32_t lo_o0, hi_o0;   // 0xCD9E8D57 o0: its low and high words
    uint32_t o1;
    __device__ __forceinline__ PhiloxRun(uint64_t seed, uint64_t offset) {
        uint32_t a = (uint32_t)seed, b = (uint32_t)(seed >> 32);
#pragma unroll
        for (int r = 0; r < 10; ++r) {
            k0[r] = a;
            k1[r] = b;
            a += 0x9E3779B9u;
            b += 0xBB67AE85u;
        }
        lo_o0 = 0xCD9E8D57u * (uint32_t)offset;
        hi_o0 = __umulhi(0xCD9E8D57u, (uint32_t)offset);
        o1 = (uint32_t)(offset >> 32);
    }
    __device__ __forceinline__ uint32_t word0(uint64_t e) const {
        uint32_t c0 = (uint32_t)e;
        const uint32_t lo = 0xD2511F53u * c0, hi = __umulhi(0xD2511F53u, c0);
        c0 = hi_o0 ^ (uint32_t)(e >> 32) ^ k0[0];
        uint32_t c1 = lo_o0, c2 = hi ^ o1 ^ k1[0], c3 = lo;
#pragma unroll
        for (int r = 1; r < 10; ++r) {
            const uint32_t lo0 = 0xD2511F53u * c0, hi0 = __umulhi(0xD2511F53u, c0);
            const uint32_t lo1 = 0xCD9E8D57u * c2, hi1 = __umulhi(0xCD9E8D57u, c2);
            c0 = hi1 ^ c1 ^ k0[r];
            c2 = hi0 ^ c3 ^ k1[r];
            c1 = lo1;
            c3 = lo0;
        }
        return c0;
    }
};

// ------------------------------------------------------------------ dependent launches

// Programmatic dependent launch.  A kernel launched with programmatic stream serialization may
// start while the kernel before it in the stream still runs (once every CTA of that kernel has
// called grid_dependents_launch() or exited); its grid_dependency_wait() returns when that
// kernel has completed and its memory writes are visible.  Without the launch attribute the
// wait returns at once and the trigger does nothing.
__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dependents_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------------ warps

// True in exactly one lane of the (fully converged) warp, false in the others.
__device__ __forceinline__ bool elect_one() {
    uint32_t chosen;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "elect.sync _|p, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(chosen));
    return chosen != 0;
}

// ------------------------------------------------------------------ thread-block clusters

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_nctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}

// All threads of every CTA of the cluster: shared-memory writes before it are visible to the
// cluster's reads after it.
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// A 32-bit word of CTA `rank`'s shared memory at the address of `local` in this CTA.
__device__ __forceinline__ uint32_t dsmem_load_u32(const void* local, uint32_t rank) {
    uint32_t remote, v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(remote) : "memory");
    return v;
}

// Sixteen bytes of CTA `rank`'s shared memory at the address of `local` in this CTA.
__device__ __forceinline__ uint4 dsmem_load_v4(const void* local, uint32_t rank) {
    uint32_t remote;
    uint4 v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
    asm volatile("ld.shared::cluster.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(remote)
                 : "memory");
    return v;
}

// ------------------------------------------------------------------ TMA

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1, int32_t c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

// Make generic-proxy writes to shared memory visible to the async proxy (TMA, tcgen05).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ tcgen05

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, s8 x s8 -> s32, one CTA.
__device__ __forceinline__ void tc_mma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, s8 x s8 -> s32, one CTA: A is M = 128 rows held in TMEM
// lanes 0-127, each row's K bytes packed four to a 32-bit column in k order (32 bytes = 8
// columns per instruction, starting at column a_tmem).
__device__ __forceinline__ void tc_mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 or fp16 inputs (both the same type), fp32
// accumulator, one CTA.  K = 16 per instruction.
__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Instruction descriptor for tcgen05.mma kind::f16 with an fp32 accumulator, A and B both
// bf16 (bf16 = true) or both fp16, both K-major, shape M x N.  Bits: [4,6) D format (1 =
// f32), [7,10) A format (0 = f16, 1 = bf16), [10,13) B format, [17,23) N >> 3, [24,29) M >> 4.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, bool bf16) {
    return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Arrive on an mbarrier once every tcgen05 operation this thread issued so far completes.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread t gets lane (base + t), columns c..c+31.
__device__ __forceinline__ void tc_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}

// 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tc_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// 32 lanes x 16 consecutive 32-bit columns from registers: thread t writes lane (base + t).
__device__ __forceinline__ void tc_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tc_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tc_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major operand stored in the 128-byte
// swizzled canonical layout: 8-row x 128-byte atoms, atoms 1024 bytes apart along
// M/N.  Bits: [0,14) start >> 4, [16,30) leading offset >> 4 (unused for swizzled
// K-major, set to 1), [32,46) stride offset >> 4, [46,48) version 1 (sm_100),
// [61,64) layout 2 = 128-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc_k_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// Instruction descriptor for tcgen05.mma kind::i8: s32 accumulator, signed A and B,
// both K-major, shape M x N.  Bits: [4,6) D format (2 = s32), [7,10) A format
// (1 = signed 8-bit), [10,13) B format, [15] A major, [16] B major, [17,23) N >> 3,
// [24,29) M >> 4.
__host__ __device__ constexpr uint32_t idesc_i8(int M, int N) {
    return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

// ------------------------------------------------------------------ dtypes

template <typename T> struct Elem;
template <> struct Elem<float> {
    __device__ static __forceinline__ float to_f(float v) { return v; }
    __device__ static __forceinline__ float from_f(float v) { return v; }
};
template <> struct Elem<__half> {
    __device__ static __forceinline__ float to_f(__half v) { return __half2float(v); }
    __device__ static __forceinline__ __half from_f(float v) { return __float2half_rn(v); }
};
template <> struct Elem<__nv_bfloat16> {
    __device__ static __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
    __device__ static __forceinline__ __nv_bfloat16 from_f(float v) {
        return __float2bfloat16_rn(v);
    }
};

// Round an fp32 value to T and back (the rotation result "in x's dtype").
template <typename T>
__device__ __forceinline__ float round_through(float v) {
    return Elem<T>::to_f(Elem<T>::from_f(v));
}

// max that propagates NaN (the row absmax of a row holding NaN is NaN).
__device__ __forceinline__ float fmax_nan(float a, float b) {
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

// Signed code of one value on the grid [-qmax - 1, qmax] (qmax = 7 for INT4, 127 for INT8):
// clamp(round_half_even(y / s), -qmax - 1, qmax); NaN -> 0.
__device__ __forceinline__ int quant_code(float y, float s, int qmax) {
    float t = __fdiv_rn(y, s);
    if (t != t) return 0;
    t = rintf(t);
    t = fminf(fmaxf(t, (float)(-qmax - 1)), (float)qmax);
    return (int)t;
}

// The divisor of one row: s and r = fl(1 / s), the correctly rounded reciprocal.
//
// Division by s uses Markstein's correction step (P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990):
//   t = fl(y r);  e = fl(y - t s) (one FMA, exact);  q = fl(t + e r) (one FMA).
// With r correctly rounded and t within a few ulps of y / s, q is the correctly rounded
// quotient fl(y / s) as long as the remainder e is not subnormal.  The quotients needed
// here are below 2^23 and y is at least 2^-24 |q| s, so s >= 2^-64 keeps e far above the
// subnormal range.  A power of two s (for instance the FLT_MIN of an all-zero row) is fast at
// any size: r = 1 / s exactly, so t = y r is the exact quotient whenever it is a normal
// number (then e = 0 and q = t), and a quotient below the normal range gives code 0 either way.
// Where t overflows or is at least 16 (a caller's scale far below the values), the code
// saturates by the sign of t, which the callers take instead of q (the correction would turn
// an infinite t into NaN).  `fast` is false when s is below 2^-64 and not a power of two, not
// finite, or NaN, or when r is not a normal number; every code of such a row takes the IEEE
// division.
struct RowDivisor {
    float s, r;
    bool fast;
    int qmax;   // the code grid [-qmax - 1, qmax]: 7 (INT4) or 127 (INT8)
    __device__ __forceinline__ RowDivisor(float s_, int qmax_) : s(s_), qmax(qmax_) {
        r = __frcp_rn(s_);
        const bool pow2 = (__float_as_uint(s_) & 0x007FFFFFu) == 0u;
        fast = (s_ >= 0x1p-64f || pow2) && (r >= 1.17549435e-38f) && (r <= 3.40282347e38f);
    }
};

// fl(y / s) for a fast RowDivisor (Markstein's correction, see RowDivisor), or y r where
// |y r| >= 1024, which saturates the code of either grid the same way.
__device__ __forceinline__ float quotient_fast(float y, float s, float r) {
    const float t = __fmul_rn(y, r);
    const float e = __fmaf_rn(-t, s, y);
    const float q = __fmaf_rn(e, r, t);
    return fabsf(t) < 1024.0f ? q : t;
}

// The same code as quant_code(y, d.s): the IEEE quotient from a reciprocal multiply and
// Markstein's correction (RowDivisor), rounded half to even by the conversion.  NaN
// converts to 0 and +-inf saturates, as in quant_code.
__device__ __forceinline__ int quant_code_fast(float y, const RowDivisor& d) {
    if (!d.fast) return quant_code(y, d.s, d.qmax);
    return min(max(__float2int_rn(quotient_fast(y, d.s, d.r)), -d.qmax - 1), d.qmax);
}

// Sixteen codes of one row (divisor d) packed four per word, first code lowest: the
// quotients of quant_code_fast computed two at a time with packed fp32 arithmetic.
__device__ __forceinline__ uint32_t pack4_codes(int q0, int q1, int q2, int q3);
__device__ __forceinline__ unsigned long long f2_pack(float a0, float a1);
__device__ __forceinline__ float2 f2_unpack(unsigned long long x);
__device__ __forceinline__ unsigned long long mul2s_rn(unsigned long long a, float b);
__device__ __forceinline__ unsigned long long fma2_rn(unsigned long long a, unsigned long long b,
                                                      unsigned long long c);
__device__ __forceinline__ void quant16(const float (&y)[16], const RowDivisor& d,
                                        uint32_t (&out)[4]) {
    int q[16];
    if (d.fast) {
        const unsigned long long ns = f2_pack(-d.s, -d.s), r2 = f2_pack(d.r, d.r);
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
            const unsigned long long y2 = f2_pack(y[i], y[i + 1]);
            const unsigned long long t = mul2s_rn(y2, d.r);
            const unsigned long long e = fma2_rn(t, ns, y2);
            const float2 qq = f2_unpack(fma2_rn(e, r2, t));
            const float2 tt = f2_unpack(t);       // |t| >= 1024: the code saturates by sign
            q[i] = __float2int_rn(fabsf(tt.x) < 1024.0f ? qq.x : tt.x);   // NaN -> 0
            q[i + 1] = __float2int_rn(fabsf(tt.y) < 1024.0f ? qq.y : tt.y);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) q[i] = __float2int_rn(__fdiv_rn(y[i], d.s));
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) q[i] = min(max(q[i], -d.qmax - 1), d.qmax);
#pragma unroll
    for (int w = 0; w < 4; ++w) out[w] = pack4_codes(q[4 * w], q[4 * w + 1], q[4 * w + 2], q[4 * w + 3]);
}

// Four codes in [-8, 7] packed into the bytes of one word, first code lowest.
__device__ __forceinline__ uint32_t pack4_codes(int q0, int q1, int q2, int q3) {
    const uint32_t lo = __byte_perm((uint32_t)q0, (uint32_t)q1, 0x0040);
    const uint32_t hi = __byte_perm((uint32_t)q2, (uint32_t)q3, 0x0040);
    return __byte_perm(lo, hi, 0x5410);
}

// Packed fp32 pairs as 64-bit registers for the sm_100 f32x2 instructions.
__device__ __forceinline__ unsigned long long f2_pack(float a0, float a1) {
    unsigned long long x;
    asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(a0), "f"(a1));
    return x;
}
__device__ __forceinline__ float2 f2_unpack(unsigned long long x) {
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(x));
    return r;
}
__device__ __forceinline__ unsigned long long add2_rn(unsigned long long a, unsigned long long b) {
    unsigned long long z;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(z) : "l"(a), "l"(b));
    return z;
}
__device__ __forceinline__ unsigned long long sub2_rn(unsigned long long a, unsigned long long b) {
    unsigned long long z;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(z) : "l"(a), "l"(b));
    return z;
}
__device__ __forceinline__ unsigned long long mul2s_rn(unsigned long long a, float b) {
    unsigned long long y = f2_pack(b, b), z;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(z) : "l"(a), "l"(y));
    return z;
}

__device__ __forceinline__ unsigned long long fma2_rn(unsigned long long a, unsigned long long b,
                                                      unsigned long long c) {
    unsigned long long z;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(z) : "l"(a), "l"(b), "l"(c));
    return z;
}

// quant16 for a row whose scale came from its own absmax (s = max(amax / qmax, FLT_MIN)), with
// the input as eight fp32 pairs.  There every quotient satisfies |y / s| <= qmax <= 127, so no
// code needs the clamp, and adding 1.5 * 2^23 to the quotient rounds it to an integer (half to
// even) that sits in the low byte of the sum's bit pattern as a two's-complement code.
// A row that is not `fast` (NaN, inf, tiny or huge scale) takes quant_code per element.
__device__ __forceinline__ void quant16_dyn2(const unsigned long long (&y2)[8], const RowDivisor& d,
                                             uint32_t (&out)[4]) {
    uint32_t u[16];
    if (d.fast) {
        const unsigned long long magic = f2_pack(0x1.8p23f, 0x1.8p23f);
        const unsigned long long ns = f2_pack(-d.s, -d.s), r2 = f2_pack(d.r, d.r);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const unsigned long long t = mul2s_rn(y2[i], d.r);
            const unsigned long long e = fma2_rn(t, ns, y2[i]);
            const unsigned long long q = fma2_rn(e, r2, t);               // fl(y / s)
            const float2 rr = f2_unpack(add2_rn(q, magic));               // 1.5 * 2^23 + rint
            u[2 * i] = __float_as_uint(rr.x);
            u[2 * i + 1] = __float_as_uint(rr.y);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float2 y = f2_unpack(y2[i]);
            u[2 * i] = (uint32_t)quant_code(y.x, d.s, d.qmax);
            u[2 * i + 1] = (uint32_t)quant_code(y.y, d.s, d.qmax);
        }
    }
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const uint32_t lo = __byte_perm(u[4 * w], u[4 * w + 1], 0x0040);
        const uint32_t hi = __byte_perm(u[4 * w + 2], u[4 * w + 3], 0x0040);
        out[w] = __byte_perm(lo, hi, 0x5410);
    }
}

}  // namespace ck
