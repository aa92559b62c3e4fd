// scan_noalloc.cu -- mamba_selective_scan_fwd_noalloc: the selective scan for callers
// that cannot allocate device memory.
//
// Some callers are not allowed to allocate: extension code running inside a host
// framework that owns the whole device-memory budget (an inference engine with a
// preallocated pool, say), or latency-sensitive code that cannot afford cudaMalloc /
// cudaFree, which may synchronise the device.  The regular entry point needs a
// caller-provided workspace whenever a long sequence is split into segments; this
// variant takes its scratch from a fixed array compiled into the library instead.
//
// The array lives in device global memory on every GPU that loads the library and
// stays allocated until the process exits.  Its device address is looked up once per
// device and context (cudaGetSymbolAddress on the first call made with that device and
// context current; a call under another context, such as one the caller made current
// with the driver API, looks it up again); host code never passes the array's name
// itself, which on the host side is only a stand-in.  After cudaDeviceReset the
// runtime may load the module again at a new address under a context whose handle
// equals the old one, so callers that reset a device must not use this entry point
// on that device afterwards.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/mamba_s6.h"

namespace {

// Largest scratch the no-allocation path can provide: 2.25 MiB.  The million-length
// layer (batch 1, dim 2048, N 16, L 2^20) needs 2.125 MiB; a split needs
// segments x batch x dim x (dstate + 1) x 4 bytes.
constexpr size_t kNoAllocScratchBytes = size_t(9) << 18;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_lock;
struct CachedAddr {
    CUcontext ctx;  // the context the address was looked up under
    void* addr;
};
CachedAddr g_scratch[kMaxDevices] = {};

using CtxGetCurrent = CUresult (*)(CUcontext*);

// cuCtxGetCurrent through the runtime's driver entry-point query (no link to libcuda).
CtxGetCurrent ctx_get_current() {
    static CtxGetCurrent fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrent>(ptr);
    });
    return fn;
}

// Device address of the scratch array on the current device and context (looked up on
// the first use there).
int scratch_on_current_device(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MAMBA_ERR_CUDA;
    const CtxGetCurrent get_ctx = ctx_get_current();
    if (!get_ctx) return MAMBA_ERR_CUDA;
    CUcontext ctx = nullptr;
    if (get_ctx(&ctx) != CUDA_SUCCESS) return MAMBA_ERR_CUDA;
    std::lock_guard<std::mutex> guard(g_lock);
    if (!ctx || g_scratch[dev].ctx != ctx || !g_scratch[dev].addr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return MAMBA_ERR_CUDA;
        // the lookup makes the runtime's context current on this thread if none was
        if (get_ctx(&ctx) != CUDA_SUCCESS || !ctx) return MAMBA_ERR_CUDA;
        g_scratch[dev].ctx = ctx;
        g_scratch[dev].addr = p;
    }
    *out = g_scratch[dev].addr;
    return MAMBA_OK;
}

}  // namespace

extern "C" int mamba_selective_scan_fwd_noalloc(const void* u, const void* delta, const float* A,
                                                const void* B, const void* C, const float* D,
                                                const void* z, const float* delta_bias,
                                                int delta_softplus, void* y, float* last_state,
                                                mamba_scan_dims dims, mamba_dtype in_dtype,
                                                mamba_dtype out_dtype, void* stream) {
    const size_t need = mamba_selective_scan_workspace_size(dims);
    void* scratch = nullptr;
    if (need > 0) {
        if (need > kNoAllocScratchBytes) return MAMBA_ERR_WORKSPACE;
        const int rc = scratch_on_current_device(&scratch);
        if (rc != MAMBA_OK) return rc;
    }
    // The split scan writes every scratch entry before it reads it, so nothing in the
    // array has to start at zero and the previous call's contents are harmless.
    return mamba_selective_scan_fwd(u, delta, A, B, C, D, z, delta_bias, delta_softplus, y,
                                    last_state, dims, in_dtype, out_dtype, scratch, need, stream);
}
