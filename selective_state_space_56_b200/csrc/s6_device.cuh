// s6_device.cuh -- small device helpers shared by the sm_100a selective-scan kernels.
//
// The SFU (MUFU) instructions are issued directly through inline PTX so the
// instruction mix is explicit: ex2.approx / lg2.approx / rcp.approx are single
// hardware instructions with documented error bounds (PTX ISA: relative error of
// ex2.approx.f32 about 2^-22, lg2.approx.f32 absolute error about 2^-22, rcp.approx
// within 1 ulp).  No CUDA math-library routine is reproduced here.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace s6 {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float lg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float rcp(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// softplus(x) = log(1 + e^x) from one ex2 and one lg2.
//  * x > 15: log(1 + e^x) - x < e^-15, below half an fp32 ulp of x; return x.
//  * x < -5: e = e^x < 6.8e-3 and log1p(e) = e - e^2/2 + e^3/3 - ...; three terms
//    leave a relative error under 1e-7, where forming 1 + e in fp32 would lose
//    up to 1e-5 of the result.
//  * otherwise log2(1 + e) * ln 2, with 1 + e >= 1.0067 so its rounding is benign.
__device__ __forceinline__ float softplus(float x) {
    float e = ex2(x * kLog2e);
    float small = e * (1.f - e * (0.5f - e * (1.f / 3.f)));
    float mid = lg2(1.f + e) * kLn2;
    float r = x < -5.f ? small : mid;
    return x > 15.f ? x : r;
}

// z * sigmoid(z) = z / (1 + e^-z); e^-z = +inf for very negative z gives z * 0.
__device__ __forceinline__ float silu(float z) { return z * rcp(1.f + ex2(-z * kLog2e)); }

template <typename T> struct io;
template <> struct io<float> {
    __device__ __forceinline__ static float load(const float* p) { return *p; }
    __device__ __forceinline__ static float to_f(float v) { return v; }
    __device__ __forceinline__ static float from_f(float v) { return v; }
};
template <> struct io<__nv_bfloat16> {
    __device__ __forceinline__ static float load(const __nv_bfloat16* p) {
        return __bfloat162float(*p);
    }
    __device__ __forceinline__ static float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
    __device__ __forceinline__ static __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};

// 16-byte global -> shared async copy (Ampere+ LDGSTS); src_bytes = 0 zero-fills.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src, int src_bytes) {
    uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem_src),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

}  // namespace s6
