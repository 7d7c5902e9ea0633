// ck_noalloc.cu -- ck_w4a4_linear_noalloc: the whole W4A4 linear without a caller-provided
// workspace, for callers that cannot allocate device memory.
//
// ck_w4a4_linear needs scratch memory for the stage-1 codes and row scales (and, for weight
// rows that are not 16-byte pitched, a re-pitched weight copy).  Some callers cannot obtain
// it: a plugin running inside a host framework that owns all device memory through its own
// allocator and exposes no allocation hook, or a latency-critical loop that must not call
// cudaMalloc (which may synchronise the device).  This entry point uses a scratch array
// compiled into the library instead: a file-scope __device__ array of kNoAllocScratchBytes,
// which every GPU that loads the library holds until the process exits.
#include <cuda_runtime_api.h>
#include <stdint.h>

#include <mutex>

#include "ck.h"

namespace ck {

// 32 MiB: the int8 codes and fp32 row scales of up to about 33 million activation
// elements (for example 8192 rows x 3840 channels).
constexpr size_t kNoAllocScratchBytes = 32u << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};
}  // namespace

// Device address of the scratch array on the current device.  In host code the array's name
// is only a host-side stand-in, so the address is looked up once per device (with that
// device current) and cached.
static ck_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CK_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return CK_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return CK_OK;
}

}  // namespace ck

extern "C" ck_status ck_w4a4_linear_noalloc(const void* x, ck_dtype x_dtype, int64_t M,
                                            int64_t K, int64_t stride_m, int64_t stride_k,
                                            const void* R, int g, const float* a_scale,
                                            const int8_t* w_packed, int64_t N, int64_t w_ld,
                                            const void* w_scale, ck_dtype scale_dtype,
                                            const void* bias, void* out, ck_dtype out_dtype,
                                            int64_t ldo, int* dev_status, cudaStream_t stream) {
    // scratch is used for the stage-1 result of activation input, for int8 codes whose rows
    // are not 16-byte aligned, and for weight rows that are not 16-byte pitched
    const bool codes_direct = x_dtype == CK_I8 && (reinterpret_cast<uintptr_t>(x) % 16) == 0 &&
                              stride_m % 16 == 0;
    const bool w_direct = (reinterpret_cast<uintptr_t>(w_packed) % 16) == 0 && w_ld % 16 == 0;
    const size_t need = (codes_direct && w_direct) ? 0 : ck_w4a4_linear_workspace_bytes(M, N, K, w_ld);
    if (need > ck::kNoAllocScratchBytes) return CK_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (M > 0 && N > 0) {
        const ck_status st = ck::scratch_address(&scratch);
        if (st != CK_OK) return st;
    }
    return ck_w4a4_linear(x, x_dtype, M, K, stride_m, stride_k, R, g, a_scale, w_packed, N, w_ld,
                          w_scale, scale_dtype, bias, out, out_dtype, ldo, scratch,
                          ck::kNoAllocScratchBytes, dev_status, stream);
}
