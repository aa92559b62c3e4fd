// diag.cu -- diagnostic entry point: the kernels' exponential paths on given inputs.
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

}  // namespace

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
