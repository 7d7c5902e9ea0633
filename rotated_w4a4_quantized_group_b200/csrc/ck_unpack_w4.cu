// ck_unpack_w4.cu -- W4 weight unpack to INT8 (comfy-kitchen PR #198 "Consolidate INT8,
// RotateQuant, RoPE and ConvRot W4A4 backends", "W4A4 correctness and performance scope":
// the W4 codes are unpacked to INT8; PR #201: only weights are unpacked) and a byte-matrix
// re-pitch used to align inputs for TMA.
//
// Packed layout: (N, K/2) bytes, byte i of a row holds the code of k = 2i in its low
// nibble and k = 2i + 1 in its high nibble, each a 4-bit two's-complement value.
#include <stdint.h>

#include "ck_device.cuh"
#include "ck_internal.h"

namespace ck {

__device__ __forceinline__ int8_t sext4(uint32_t v) { return (int8_t)((int)(v << 28) >> 28); }

// One thread per 8 packed bytes (16 codes) when rows are 8-byte / 16-byte aligned,
// otherwise one thread per packed byte.
__global__ void unpack_w4_vec_kernel(const int8_t* __restrict__ packed, int64_t N, int64_t K,
                                     int64_t ld_packed, int8_t* __restrict__ out, int64_t ld_out) {
    const int64_t per_row = K / 16;    // 8-byte packed chunks per row
    const int64_t total = N * per_row;
    for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total;
         t += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = t / per_row, c = t - n * per_row;
        const uint2 v = *reinterpret_cast<const uint2*>(packed + n * ld_packed + c * 8);
        uint32_t o[4];
        const uint32_t w[2] = {v.x, v.y};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint32_t lo = 0, hi = 0;
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const uint32_t byte = (w[h] >> (8 * b)) & 0xFFu;
                const uint32_t e0 = (uint32_t)(uint8_t)sext4(byte & 0xFu);
                const uint32_t e1 = (uint32_t)(uint8_t)sext4(byte >> 4);
                const uint32_t pair = e0 | (e1 << 8);
                if (b < 2) lo |= pair << (16 * b);
                else hi |= pair << (16 * (b - 2));
            }
            o[2 * h] = lo;
            o[2 * h + 1] = hi;
        }
        *reinterpret_cast<uint4*>(out + n * ld_out + c * 16) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

__global__ void unpack_w4_scalar_kernel(const int8_t* __restrict__ packed, int64_t N, int64_t K,
                                        int64_t ld_packed, int8_t* __restrict__ out,
                                        int64_t ld_out) {
    const int64_t half = K / 2;
    const int64_t total = N * half;
    for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total;
         t += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = t / half, i = t - n * half;
        const uint32_t byte = (uint8_t)packed[n * ld_packed + i];
        out[n * ld_out + 2 * i] = sext4(byte & 0xFu);
        out[n * ld_out + 2 * i + 1] = sext4(byte >> 4);
    }
}

__global__ void copy_rows_kernel(const int8_t* __restrict__ src, int64_t ld_src,
                                 int8_t* __restrict__ dst, int64_t ld_dst, int64_t rows,
                                 int64_t cols) {
    const int64_t total = rows * cols;
    for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total;
         t += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = t / cols, c = t - r * cols;
        dst[r * ld_dst + c] = src[r * ld_src + c];
    }
}

static int grid_for(int64_t work, int threads) {
    int64_t b = (work + threads - 1) / threads;
    const int64_t cap = 8LL * num_sms();
    if (b > cap) b = cap;
    return (int)(b < 1 ? 1 : b);
}

ck_status launch_unpack_w4(const int8_t* packed, int64_t N, int64_t K, int64_t ld_packed,
                           int8_t* out, int64_t ld_out, cudaStream_t stream) {
    if (N == 0) return CK_OK;
    const bool vec = K % 16 == 0 && aligned(packed, 8) && ld_packed % 8 == 0 &&
                     aligned(out, 16) && ld_out % 16 == 0;
    if (vec) {
        const int64_t work = N * (K / 16);
        unpack_w4_vec_kernel<<<grid_for(work, 256), 256, 0, stream>>>(packed, N, K, ld_packed, out,
                                                                       ld_out);
    } else {
        const int64_t work = N * (K / 2);
        unpack_w4_scalar_kernel<<<grid_for(work, 256), 256, 0, stream>>>(packed, N, K, ld_packed,
                                                                         out, ld_out);
    }
    return cudaGetLastError() == cudaSuccess ? CK_OK : CK_ERR_CUDA;
}

ck_status launch_copy_rows(const int8_t* src, int64_t ld_src, int8_t* dst, int64_t ld_dst,
                           int64_t rows, int64_t cols, cudaStream_t stream) {
    if (rows == 0 || cols == 0) return CK_OK;
    copy_rows_kernel<<<grid_for(rows * cols, 256), 256, 0, stream>>>(src, ld_src, dst, ld_dst, rows,
                                                                     cols);
    return cudaGetLastError() == cudaSuccess ? CK_OK : CK_ERR_CUDA;
}

}  // namespace ck
