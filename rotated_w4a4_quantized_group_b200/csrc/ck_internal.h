// ck_internal.h -- host-side declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime_api.h>
#include <stdint.h>

#include "ck.h"

namespace ck {

// Encode a tiled TMA descriptor through the driver entry point (no -lcuda link).
// Returns CK_ERR_CUDA if the driver call fails.
ck_status encode_tma(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base,
                     const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                     CUtensorMapSwizzle swizzle);

int num_sms();

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Where stage 2 writes its outputs: channels [start[s], start[s + 1]) go to segment s, whose
// column 0 is channel start[s], with row pitch ldo[s] (elements).  A plain linear is one
// segment; a grouped linear has one per group.
constexpr int kMaxOutSegs = 8;
struct OutSegs {
    int n;
    int64_t start[kMaxOutSegs + 1];
    void* ptr[kMaxOutSegs];
    int64_t ldo[kMaxOutSegs];
};

inline OutSegs single_segment(void* out, int64_t N, int64_t ldo) {
    OutSegs s = {};
    s.n = 1;
    s.start[0] = 0;
    s.start[1] = N;
    s.ptr[0] = out;
    s.ldo[0] = ldo;
    return s;
}

// Stage 1 launch (arguments already validated); qmax = 7 gives signed-INT4 codes, 127 the
// INT8 codes of the W8A8 variant.
ck_status launch_rotate_quant(const void* x, ck_dtype dt, int64_t M, int64_t K, int64_t sm,
                              int64_t sk, const void* R, int g, const float* scale_in,
                              int8_t* codes, int64_t ldq, float* scales, int qmax,
                              int* dev_status, cudaStream_t stream);

// fp32 stage-1 kernels; each returns CK_ERR_UNSUPPORTED for shapes or layouts it does not take:
//   launch_rq_tf32         g = 64, row-major, split TF32 on the tensor cores (ck_rq_tf32.cu)
//   launch_rq_f32_ffma256  g = 256, row-major, K <= 16384, FFMA (ck_rq_f32_256.cu)
//   launch_rq_f32_g16      g = 16, row-major or column-major, FP64 tensor-core rotation
//                          (ck_rq_f32.cu)
ck_status launch_rq_tf32(const void* x, int64_t M, int64_t K, int64_t sm, int64_t sk,
                         const void* R, const float* scale_in, int8_t* codes, int64_t ldq,
                         float* scales, int qmax, int* dev_status, cudaStream_t stream);
ck_status launch_rq_f32_ffma256(const void* x, int64_t M, int64_t K, int64_t sm, int64_t sk,
                                const void* R, const float* scale_in, int8_t* codes, int64_t ldq,
                                float* scales, int qmax, int* dev_status, cudaStream_t stream);
// fp32 stage 1 at g = 64 or 256 on row-major rows (ck_rq_tf32.cu picks the kernel);
// CK_ERR_UNSUPPORTED for shapes no kernel there takes.
ck_status launch_rq_f32_wide(const void* x, int64_t M, int64_t K, int64_t sm, int64_t sk,
                             const void* R, int g, const float* scale_in, int8_t* codes,
                             int64_t ldq, float* scales, int qmax, int* dev_status,
                             cudaStream_t stream);
ck_status launch_rq_f32_g16(const void* x, int64_t M, int64_t K, int64_t sm, int64_t sk,
                            const void* R, const float* scale_in, int8_t* codes, int64_t ldq,
                            float* scales, int qmax, int* dev_status, cudaStream_t stream);

// Stage 2 launch: codes (M, K) int8 with 16-byte-aligned rows (ldq % 16 == 0), packed
// weights with 16-byte-aligned rows (w_ld % 16 == 0).  after_stage1: the kernel just before
// this one on the stream is the stage-1 launch that writes the codes and row scales (and
// nothing this GEMM reads besides them); the GEMM is then launched as its programmatic
// dependent, so it may start (set up, load and expand its weights) while stage 1 finishes,
// and reads the codes and scales only after stage 1 has completed.
ck_status launch_w4a4_gemm(const int8_t* codes, int64_t ldq, const float* a_scale, int64_t M,
                           int64_t K, const int8_t* w_packed, int64_t w_ld, int64_t N,
                           const void* w_scale, ck_dtype scale_dt, const void* bias,
                           const OutSegs& segs, ck_dtype out_dt, bool after_stage1,
                           int* dev_status, cudaStream_t stream);

// The W8A8 variant's stage 2: INT8 weights (N, K) with 16-byte-aligned rows (w_ld % 16 == 0),
// the same codes, epilogue and outputs as launch_w4a4_gemm.
ck_status launch_w8a8_gemm(const int8_t* codes, int64_t ldq, const float* a_scale, int64_t M,
                           int64_t K, const int8_t* w, int64_t w_ld, int64_t N,
                           const void* w_scale, ck_dtype scale_dt, const void* bias,
                           const OutSegs& segs, ck_dtype out_dt, bool after_stage1,
                           int* dev_status, cudaStream_t stream);

// Stage 2 for M <= 64 with K split over a thread-block cluster (ck_w4a4_splitk.cu); same
// arguments as launch_w4a4_gemm.  Returns CK_ERR_UNSUPPORTED for shapes it does not take.
ck_status launch_w4a4_splitk(const int8_t* codes, int64_t ldq, const float* a_scale, int64_t M,
                             int64_t K, const int8_t* w_packed, int64_t w_ld, int64_t N,
                             const void* w_scale, ck_dtype scale_dt, const void* bias,
                             const OutSegs& segs, ck_dtype out_dt, bool after_stage1,
                             int* dev_status, cudaStream_t stream);

ck_status launch_unpack_w4(const int8_t* packed, int64_t N, int64_t K, int64_t ld_packed,
                           int8_t* out, int64_t ld_out, cudaStream_t stream);

// Scratch bytes one ck_w4a4_linear call needs (0 when it needs none): the stage-1 codes and
// row scales for floating-point input, or a 16-byte-pitched copy of int8 codes whose rows are
// not 16-byte aligned, then (offset past them) a 16-byte-pitched copy of packed weights that
// are not 16-byte aligned and pitched.  Arguments as in ck_w4a4_linear, already validated.
size_t linear_scratch_need(const void* x, ck_dtype x_dtype, int64_t M, int64_t K,
                           int64_t stride_m, const int8_t* w_packed, int64_t N, int64_t w_ld,
                           bool w8 = false);

// The public packed quantizer (ck_rq_packed.cu), arguments already validated.
// The packed quantizer on the tensor-core stage-1 kernel (ck_rotate_quant.cu): bf16/fp16, unit K
// stride, g = 16 or 64 with at most 128 64-channel group-rows, or g = 256 with at most 128
// groups; CK_ERR_UNSUPPORTED otherwise.
ck_status launch_rotate_quant_packed_tc(const void* x, ck_dtype dt, int64_t M, int64_t K,
                                        int64_t sm, int64_t sk, const void* R, int g,
                                        const float* scale_in, bool stochastic, uint64_t seed,
                                        uint64_t offset, uint8_t* packed, int64_t ldp,
                                        float* scales, cudaStream_t stream);
ck_status launch_rotate_quant_packed(const void* x, ck_dtype dt, int64_t M, int64_t K, int64_t sm,
                                     int64_t sk, const void* R, int g, const float* scale_in,
                                     bool stochastic, uint64_t seed, uint64_t offset,
                                     uint8_t* packed, int64_t ldp, float* scales,
                                     cudaStream_t stream);

// Copy a (rows, cols) byte matrix between pitches (used to re-pitch misaligned inputs).
ck_status launch_copy_rows(const int8_t* src, int64_t ld_src, int8_t* dst, int64_t ld_dst,
                           int64_t rows, int64_t cols, cudaStream_t stream);

}  // namespace ck
