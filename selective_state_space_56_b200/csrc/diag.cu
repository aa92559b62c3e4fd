// diag.cu -- diagnostic entry points: the kernels' exponential paths on given inputs, and
// a throughput probe of the pipes the scan's roofline is stated against.
#include "../../include/mamba_s6.h"
#include "s6_device.cuh"

namespace {

__global__ void exp2_paths_kernel(const float* x, float* out_fma, float* out_sfu, float* out_lib,
                                  int64_t n) {
    const int64_t i = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
    if (i >= n) return;
    const float a = x[i], b = i + 1 < n ? x[i + 1] : 0.f;
    float f0, f1;
    s6::unpack2(s6::exp2_fma2(s6::pack2(a, b)), f0, f1);
    out_fma[i] = f0;
    out_sfu[i] = s6::ex2(a);
    out_lib[i] = exp2f(a);
    if (i + 1 < n) {
        out_fma[i + 1] = f1;
        out_sfu[i + 1] = s6::ex2(b);
        out_lib[i + 1] = exp2f(b);
    }
}

// Throughput probe: 8 independent chains per thread of one instruction kind, so every
// pipe stays fed (64 resident warps per SM at 256 threads x 8 CTAs).  kind 0: SFU
// ex2.approx (x <- 2^-x stays in [1/2, 1)); 1: fp32 FMA; 2: packed fp32x2 FMA.
__global__ void __launch_bounds__(256) throughput_kernel(int kind, int64_t iters, float* sink) {
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = 0.25f + 0.01f * i + 1e-7f * (threadIdx.x & 31);
    if (kind == 0) {
#pragma unroll 8
        for (int64_t it = 0; it < iters; ++it)
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = s6::ex2(-v[i]);
    } else if (kind == 1) {
#pragma unroll 8
        for (int64_t it = 0; it < iters; ++it)
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = fmaf(v[i], 0.9999f, 1e-4f);
    } else {
        s6::f2 w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = s6::pack2(v[i], v[i] + 0.5f);
        const s6::f2 a = s6::pack2(0.9999f, 0.9999f), c = s6::pack2(1e-4f, 1e-4f);
#pragma unroll 8
        for (int64_t it = 0; it < iters; ++it)
#pragma unroll
            for (int i = 0; i < 8; ++i) w[i] = s6::fma2(w[i], a, c);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float lo, hi;
            s6::unpack2(w[i], lo, hi);
            v[i] = lo + hi;
        }
    }
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) acc += v[i];
    sink[tid] = acc;
}

}  // namespace

extern "C" int mamba_diag_throughput(int kind, int64_t blocks, int64_t iters, float* sink,
                                     void* stream) {
    if (!sink) return MAMBA_ERR_NULL;
    // blocks x iters <= 2^28 keeps one launch well under a second on a B200
    if (kind < 0 || kind > 2 || blocks < 1 || blocks > (1LL << 20) || iters < 1 ||
        iters > (1LL << 24) || blocks * iters > (1LL << 28))
        return MAMBA_ERR_DIMS;
    throughput_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(kind, iters,
                                                                                      sink);
    return cudaGetLastError() == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA;
}

extern "C" int mamba_diag_exp2(const float* x, float* out_fma, float* out_sfu, float* out_lib,
                               int64_t n, void* stream) {
    if (!x || !out_fma || !out_sfu || !out_lib) return MAMBA_ERR_NULL;
    if (n < 0) return MAMBA_ERR_DIMS;
    if (n == 0) return MAMBA_OK;
    const int64_t pairs = (n + 1) / 2;
    exp2_paths_kernel<<<(unsigned)((pairs + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        x, out_fma, out_sfu, out_lib, n);
    return cudaGetLastError() == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA;
}
