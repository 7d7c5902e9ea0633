// ck_rq_packed.cu -- the public packed-activation quantizer: the same rotation and row scale as
// stage 1, codes rounded half to even or stochastically, stored two to a byte.
//
// Operation (comfy-kitchen PR #201 "Avoid activation pack/unpack in ConvRot W4A4", "Summary":
// the W4A4 path stops packing activations, while the public packed quantizer keeps its
// signature, its scales and its stochastic rounding; "Correctness and tests": odd widths are
// rejected):
//   y = rotation of x in its dtype, s = max(fp32(amax |y|) / 7, FLT_MIN) (or the caller's)
//   t = fl(y / s)
//   nearest:    q = clamp(round_half_even(t), -8, 7)
//   stochastic: q = clamp(floor(fl(t + u)), -8, 7),  u = (r >> 8) * 2^-24,
//               r = word 0 of Philox4x32-10(counter {e, e >> 32, offset, offset >> 32},
//                                           key {seed, seed >> 32}),  e = m K + k
//   packed[m, k / 2] = (q[m, k] & 15) | (q[m, k + 1] & 15) << 4        (k even)
// Philox4x32-10 is the counter-based generator of Salmon, Moraes, Dror and Shaw ("Parallel
// random numbers: as easy as 1, 2, 3", SC 2011): ten rounds of two 32 x 32 -> 64-bit products
// mixed with the key, the key bumped by two Weyl constants between rounds.
//
// 16-bit rows of g = 16 or 64 and at most 128 64-channel group-rows, or of g = 256 and at most
// 128 groups, go to the tensor-core stage-1 kernel with a packed epilogue (ck_rotate_quant.cu).
// Every other row here: one row per CTA step (grid-stride over rows): the row is read once into
// shared memory
// (any strides), each thread rotates 4-channel chunks with fp32 FMAs against R in shared
// memory and rounds them to the dtype, the row absmax is reduced through shared memory, and a
// second pass rotates again, quantizes and stores 2 bytes per chunk.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <float.h>
#include <stdint.h>

#include "ck_device.cuh"
#include "ck_internal.h"

namespace ck {

namespace rqp {
constexpr int kThreads = 256;
}

template <typename T>
__device__ __forceinline__ float4 rqp_load4_r(const T* p);
template <>
__device__ __forceinline__ float4 rqp_load4_r<float>(const float* p) {
    return make_float4(p[0], p[1], p[2], p[3]);
}
template <>
__device__ __forceinline__ float4 rqp_load4_r<__half>(const __half* p) {
    return make_float4(__half2float(p[0]), __half2float(p[1]), __half2float(p[2]), __half2float(p[3]));
}
template <>
__device__ __forceinline__ float4 rqp_load4_r<__nv_bfloat16>(const __nv_bfloat16* p) {
    return make_float4(__bfloat162float(p[0]), __bfloat162float(p[1]), __bfloat162float(p[2]),
                       __bfloat162float(p[3]));
}

// Channels c0 .. c0 + 3 of group j0 of the row in shared memory, rounded to T.
template <typename T>
__device__ __forceinline__ void rqp_rotate4(const float* xs, const T* Rs, int g, int64_t k0,
                                            float (&y)[4]) {
    const int64_t j0 = (k0 / g) * g;
    const int c0 = (int)(k0 - j0);
    float a[4] = {0.f, 0.f, 0.f, 0.f};
    for (int i = 0; i < g; ++i) {
        const float xv = xs[j0 + i];
        const float4 r = rqp_load4_r<T>(Rs + (int64_t)i * g + c0);
        a[0] = __fmaf_rn(xv, r.x, a[0]);
        a[1] = __fmaf_rn(xv, r.y, a[1]);
        a[2] = __fmaf_rn(xv, r.z, a[2]);
        a[3] = __fmaf_rn(xv, r.w, a[3]);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) y[e] = round_through<T>(a[e]);
}

template <typename T, bool SR>
__global__ void __launch_bounds__(rqp::kThreads)
    rq_packed_kernel(const T* __restrict__ x, int64_t M, int64_t K, int64_t sm, int64_t sk,
                     const T* __restrict__ R, int g, const float* __restrict__ scale_in,
                     uint8_t* __restrict__ packed, int64_t ldp, float* __restrict__ scales,
                     uint64_t seed, uint64_t offset, int vec) {
    using namespace rqp;
    extern __shared__ __align__(16) unsigned char rqp_smem[];
    float* xs = reinterpret_cast<float*>(rqp_smem);
    T* Rs = reinterpret_cast<T*>(xs + K);
    __shared__ float warp_max[kThreads / 32];
    const int tid = threadIdx.x;
    for (int i = tid; i < g * g; i += kThreads) Rs[i] = R[i];
    const int64_t nchunk = K / 4;
    const uint32_t k0s = (uint32_t)seed, k1s = (uint32_t)(seed >> 32);
    const uint32_t o0 = (uint32_t)offset, o1 = (uint32_t)(offset >> 32);

    for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
        __syncthreads();
        const T* xr = x + m * sm;
        for (int64_t k = tid; k < K; k += kThreads) xs[k] = Elem<T>::to_f(xr[k * sk]);
        __syncthreads();
        float mx = 0.f;
        for (int64_t ci = tid; ci < nchunk; ci += kThreads) {
            float y[4];
            rqp_rotate4<T>(xs, Rs, g, ci * 4, y);
#pragma unroll
            for (int e = 0; e < 4; ++e) mx = fmax_nan(mx, fabsf(y[e]));
        }
        for (int o = 16; o > 0; o >>= 1) mx = fmax_nan(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if ((tid & 31) == 0) warp_max[tid >> 5] = mx;
        __syncthreads();
        float amax = 0.f;
        for (int w = 0; w < kThreads / 32; ++w) amax = fmax_nan(amax, warp_max[w]);
        float s = scale_in ? *scale_in : __fdiv_rn(amax, 7.0f);
        s = (s < FLT_MIN) ? FLT_MIN : s;   // lower clamp; NaN stays NaN
        if (tid == 0) scales[m] = s;
        const RowDivisor dv(s, 7);

        uint8_t* pr = packed + m * ldp;
        for (int64_t ci = tid; ci < nchunk; ci += kThreads) {
            float y[4];
            rqp_rotate4<T>(xs, Rs, g, ci * 4, y);
            int q[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if (!SR) {
                    q[e] = quant_code_fast(y[e], dv);
                } else {
                    // t = fl(y / s): the corrected reciprocal product for a fast row (y r itself
                    // where |y r| >= 1024, which saturates either way), the IEEE divide otherwise
                    const float t = dv.fast ? quotient_fast(y[e], dv.s, dv.r) : __fdiv_rn(y[e], dv.s);
                    if (t != t) {
                        q[e] = 0;
                        continue;
                    }
                    const uint64_t el = (uint64_t)m * (uint64_t)K + (uint64_t)(ci * 4 + e);
                    const uint32_t rnd = philox_word0((uint32_t)el, (uint32_t)(el >> 32), o0, o1, k0s, k1s);
                    const float u = __uint2float_rn(rnd >> 8) * 0x1p-24f;   // exact
                    float v = floorf(__fadd_rn(t, u));
                    v = fminf(fmaxf(v, -8.0f), 7.0f);
                    q[e] = (int)v;
                }
            }
            const uint32_t b0 = ((uint32_t)q[0] & 15u) | (((uint32_t)q[1] & 15u) << 4);
            const uint32_t b1 = ((uint32_t)q[2] & 15u) | (((uint32_t)q[3] & 15u) << 4);
            uint8_t* dst = pr + ci * 2;
            if (vec) {
                *reinterpret_cast<uint16_t*>(dst) = (uint16_t)(b0 | (b1 << 8));
            } else {
                dst[0] = (uint8_t)b0;
                dst[1] = (uint8_t)b1;
            }
        }
    }
}

template <typename T>
static ck_status launch_packed_typed(const void* x, int64_t M, int64_t K, int64_t sm, int64_t sk,
                                     const void* R, int g, const float* scale_in, bool sr,
                                     uint64_t seed, uint64_t offset, uint8_t* packed, int64_t ldp,
                                     float* scales, cudaStream_t stream) {
    using namespace rqp;
    const size_t smem = (size_t)K * sizeof(float) + (size_t)g * g * sizeof(T);
    if (smem > 220 * 1024) return CK_ERR_UNSUPPORTED;
    const int vec = (aligned(packed, 2) && ldp % 2 == 0) ? 1 : 0;
    const int grid = (int)(M < 8LL * num_sms() ? M : 8LL * num_sms());
    auto kern = sr ? rq_packed_kernel<T, true> : rq_packed_kernel<T, false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return CK_ERR_CUDA;
    kern<<<grid, kThreads, smem, stream>>>(static_cast<const T*>(x), M, K, sm, sk,
                                           static_cast<const T*>(R), g, scale_in, packed, ldp,
                                           scales, seed, offset, vec);
    return cudaGetLastError() == cudaSuccess ? CK_OK : CK_ERR_CUDA;
}

ck_status launch_rotate_quant_packed(const void* x, ck_dtype dt, int64_t M, int64_t K, int64_t sm,
                                     int64_t sk, const void* R, int g, const float* scale_in,
                                     bool stochastic, uint64_t seed, uint64_t offset,
                                     uint8_t* packed, int64_t ldp, float* scales,
                                     cudaStream_t stream) {
    if (M == 0) return CK_OK;
    // 16-bit rows of g = 16, 64 (at most 128 64-channel group-rows) or 256 (at most 128 groups):
    // the tensor-core kernel
    const ck_status st = launch_rotate_quant_packed_tc(x, dt, M, K, sm, sk, R, g, scale_in,
                                                       stochastic, seed, offset, packed, ldp,
                                                       scales, stream);
    if (st != CK_ERR_UNSUPPORTED) return st;
    switch (dt) {
        case CK_F32:
            return launch_packed_typed<float>(x, M, K, sm, sk, R, g, scale_in, stochastic, seed,
                                              offset, packed, ldp, scales, stream);
        case CK_F16:
            return launch_packed_typed<__half>(x, M, K, sm, sk, R, g, scale_in, stochastic, seed,
                                               offset, packed, ldp, scales, stream);
        case CK_BF16:
            return launch_packed_typed<__nv_bfloat16>(x, M, K, sm, sk, R, g, scale_in, stochastic,
                                                      seed, offset, packed, ldp, scales, stream);
        default: return CK_ERR_INVALID_ARG;
    }
}

}  // namespace ck
