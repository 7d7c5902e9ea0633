// ck_gemm_common.cuh -- device helpers shared by the W4A4 GEMM kernels: packed-weight
// nibble expansion, weight-scale loads by dtype, output stores by dtype, ring positions.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace ck {

// Eight signed 4-bit codes of one packed word -> eight sign-extended bytes in k order (the
// low nibble of byte i is k = 2i).  Per byte, a nibble x in [0, 15] becomes
// ((x + 0x78) ^ 0x78): x for x < 8 and x + 240 (x - 16 as a signed byte) for x >= 8; the sum
// stays below 0x100, so no carry crosses a byte.
__device__ __forceinline__ void unpack_word_s(uint32_t w, uint32_t& o0, uint32_t& o1) {
    const uint32_t lo = ((w & 0x0F0F0F0Fu) + 0x78787878u) ^ 0x78787878u;          // k even
    const uint32_t hi = (((w >> 4) & 0x0F0F0F0Fu) + 0x78787878u) ^ 0x78787878u;   // k odd
    o0 = __byte_perm(lo, hi, 0x5140);                                             // k0 k1 k2 k3
    o1 = __byte_perm(lo, hi, 0x7362);                                             // k4 k5 k6 k7
}

// The same eight codes as the bytes 16 w: a signed nibble placed in the high half of a byte
// reads as 16 times its value.
__device__ __forceinline__ void unpack_word_x16(uint32_t w, uint32_t& o0, uint32_t& o1) {
    const uint32_t lo = (w << 4) & 0xF0F0F0F0u;   // k even
    const uint32_t hi = w & 0xF0F0F0F0u;          // k odd
    o0 = __byte_perm(lo, hi, 0x5140);
    o1 = __byte_perm(lo, hi, 0x7362);
}

// A ring position: slot index and the parity of the slot's current fill.
struct RingPos {
    uint32_t idx = 0, phase = 0;
    __device__ __forceinline__ void step(uint32_t n) {
        if (++idx == n) {
            idx = 0;
            phase ^= 1u;
        }
    }
};

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

}  // namespace ck
