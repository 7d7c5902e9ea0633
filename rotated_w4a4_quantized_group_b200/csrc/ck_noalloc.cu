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
#include <cuda.h>
#include <cuda_runtime_api.h>
#include <stdint.h>

#include <mutex>

#include "ck.h"
#include "ck_internal.h"

namespace ck {

// 32 MiB: the int8 codes and fp32 row scales of up to about 33 million activation
// elements (for example 8192 rows x 3840 channels).
constexpr size_t kNoAllocScratchBytes = 32u << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context (0 if the driver cannot say).  A device
// reset ends the context and reloads the module, which may move the array; the new context has
// a new id, so an address cached under the old one is looked up again.
unsigned long long current_context_id() {
    static CtxGetCurrentFn get_ctx = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_ctx = reinterpret_cast<CtxGetCurrentFn>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_ctx && get_id && get_ctx(&ctx) == CUDA_SUCCESS && ctx && get_id(ctx, &id) == CUDA_SUCCESS)
        return id;
    return 0;
}
}  // namespace

// Device address of the scratch array on the current device.  In host code the array's name
// is only a host-side stand-in, so the address is looked up (with that device current) once
// per device and context, and cached.
static ck_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CK_ERR_CUDA;
    unsigned long long ctx = current_context_id();
    if (ctx == 0) {   // no context current yet: make the device's primary context current
        if (cudaSetDevice(dev) != cudaSuccess) return CK_ERR_CUDA;
        ctx = current_context_id();
    }
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_addr[dev] || g_scratch_ctx[dev] != ctx) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return CK_ERR_CUDA;
        g_scratch_addr[dev] = p;
        g_scratch_ctx[dev] = ctx;
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
    // the same scratch calculation ck_w4a4_linear enforces (pointer alignments included);
    // sizes it would reject are passed on for it to reject
    if (M > 0 && N > 0 && K > 0 && K % 2 == 0 && w_ld >= K / 2) {
        const size_t need =
            ck::linear_scratch_need(x, x_dtype, M, K, stride_m, w_packed, N, w_ld);
        if (need > ck::kNoAllocScratchBytes) return CK_ERR_WORKSPACE;
    }
    void* scratch = nullptr;
    if (M > 0 && N > 0) {
        const ck_status st = ck::scratch_address(&scratch);
        if (st != CK_OK) return st;
    }
    return ck_w4a4_linear(x, x_dtype, M, K, stride_m, stride_k, R, g, a_scale, w_packed, N, w_ld,
                          w_scale, scale_dtype, bias, out, out_dtype, ldo, scratch,
                          ck::kNoAllocScratchBytes, dev_status, stream);
}
