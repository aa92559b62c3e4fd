// conv1d.cu -- causal depthwise conv1d + SiLU (the Mamba block's producer of the scan's
// input u) and its one-token decode update, for sm_100a.
//
// Mamba block ("Mamba: Linear-Time Sequence Modeling with Selective State Spaces", Mamba
// Block; the "Mamba" Q&A on the convolution before the SSM): the projected input x of
// every channel passes a short causal 1-D convolution and an activation before the SSM:
//
//   out[b, d, t] = silu(bias[d] + sum_{k<K} w[d, k] * x[b, d, t - (K-1) + k])
//
// with the K-1 inputs before the sequence taken from an optional initial state.  The step
// is a pure stream (2 bytes in, 2 bytes out per element in bf16), so the kernel is laid out
// for HBM: a thread owns two consecutive 16-byte vectors of outputs of one row, issues
// its loads first (the two vectors and the one before them, whose last K-1 inputs form the
// halo -- that vector is also another thread's, so the extra read mostly hits L1), carries
// the halo of the second vector in registers, computes in fp32 and stores 16 bytes per
// vector.  The grid is (vector blocks, dim, batch), so no thread divides to find its row.
// Rows whose length is not a multiple of the vector take an element-wise path.
#include <cstring>

#include "s6_device.cuh"
#include "s6_launch.h"

namespace s6 {
namespace {

struct CParams {
    const void* x;
    const float* w;
    const float* bias;
    const void* init;
    void* out;
    void* fin;
    int64_t rows, dim, L;
    int K;
    int silu;
};

template <typename T>
__device__ __forceinline__ float ldf(const T* p) {
    return io<T>::to_f(*p);
}

// Input at position s of row r of the extended sequence init ++ x (zero before init).
template <typename T>
__device__ __forceinline__ float x_at(const CParams& p, int64_t r, int64_t s) {
    if (s >= 0) return ldf(static_cast<const T*>(p.x) + r * p.L + s);
    if (!p.init) return 0.f;
    return ldf(static_cast<const T*>(p.init) + r * (p.K - 1) + (p.K - 1) + s);
}

// One thread per kVPT consecutive 16-byte output vectors of one row; the grid is
// (vector blocks, dim, batch), so a thread finds its row and channel without division.
constexpr int kVPT = 2;

template <typename T, int K>
__global__ void __launch_bounds__(256) conv1d_vec_kernel(const CParams p) {
    constexpr int E = 16 / sizeof(T);  // outputs per 16-byte vector
    const int64_t vpr = p.L / E;
    const int64_t v0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * kVPT;
    if (v0 >= vpr) return;
    const int64_t d = blockIdx.y;
    const int64_t r = (int64_t)blockIdx.z * p.dim + d;
    const T* xr = static_cast<const T*>(p.x) + r * p.L;
    // every load first: the vectors of this thread and the one before them
    uint4 cur[kVPT], prev = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int i = 0; i < kVPT; ++i)
        if (v0 + i < vpr) cur[i] = *reinterpret_cast<const uint4*>(xr + (v0 + i) * E);
    if (K > 1 && v0 > 0) prev = *reinterpret_cast<const uint4*>(xr + (v0 - 1) * E);
    float w[K];
#pragma unroll
    for (int k = 0; k < K; ++k) w[k] = __ldg(p.w + d * K + k);
    const float bias = p.bias ? __ldg(p.bias + d) : 0.f;

    float hist[K > 1 ? K - 1 : 1];  // the K-1 inputs before the current vector
    if (K > 1) {
        if (v0 > 0) {
            const T* c = reinterpret_cast<const T*>(&prev);
#pragma unroll
            for (int j = 0; j < K - 1; ++j) hist[j] = io<T>::to_f(c[E - (K - 1) + j]);
        } else {
#pragma unroll
            for (int j = 0; j < K - 1; ++j) hist[j] = x_at<T>(p, r, j - (K - 1));
        }
    }
#pragma unroll
    for (int i = 0; i < kVPT; ++i) {
        if (v0 + i >= vpr) break;
        float xv[K - 1 + E];
#pragma unroll
        for (int j = 0; j < K - 1; ++j) xv[j] = hist[j];
        const T* c = reinterpret_cast<const T*>(&cur[i]);
#pragma unroll
        for (int j = 0; j < E; ++j) xv[K - 1 + j] = io<T>::to_f(c[j]);
        alignas(16) T o[E];
#pragma unroll
        for (int j = 0; j < E; ++j) {
            float acc = bias;
#pragma unroll
            for (int k = 0; k < K; ++k) acc = fmaf(w[k], xv[j + k], acc);
            o[j] = io<T>::from_f(p.silu ? silu(acc) : acc);
        }
        *reinterpret_cast<uint4*>(static_cast<T*>(p.out) + r * p.L + (v0 + i) * E) =
            *reinterpret_cast<const uint4*>(o);
        if (K > 1) {
#pragma unroll
            for (int j = 0; j < K - 1; ++j) hist[j] = xv[E + j];
        }
    }
}

// Rows too many for the grid's y/z extent: one thread per 16-byte vector, row found by
// division.
template <typename T, int K>
__global__ void __launch_bounds__(256) conv1d_vec1d_kernel(const CParams p) {
    constexpr int E = 16 / sizeof(T);
    const int64_t vpr = p.L / E;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= p.rows * vpr) return;
    const int64_t r = gid / vpr, t0 = (gid - r * vpr) * E;
    const int64_t d = r % p.dim;
    float xv[K - 1 + E];
#pragma unroll
    for (int j = 0; j < K - 1; ++j) xv[j] = x_at<T>(p, r, t0 - (K - 1) + j);
    const uint4 cur = *reinterpret_cast<const uint4*>(static_cast<const T*>(p.x) + r * p.L + t0);
    const T* c = reinterpret_cast<const T*>(&cur);
#pragma unroll
    for (int j = 0; j < E; ++j) xv[K - 1 + j] = io<T>::to_f(c[j]);
    const float bias = p.bias ? __ldg(p.bias + d) : 0.f;
    alignas(16) T o[E];
#pragma unroll
    for (int j = 0; j < E; ++j) {
        float acc = bias;
#pragma unroll
        for (int k = 0; k < K; ++k) acc = fmaf(__ldg(p.w + d * K + k), xv[j + k], acc);
        o[j] = io<T>::from_f(p.silu ? silu(acc) : acc);
    }
    *reinterpret_cast<uint4*>(static_cast<T*>(p.out) + r * p.L + t0) =
        *reinterpret_cast<const uint4*>(o);
}

template <typename T, int K>
__global__ void __launch_bounds__(256) conv1d_elem_kernel(const CParams p) {
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= p.rows * p.L) return;
    const int64_t r = gid / p.L, t = gid - r * p.L;
    const int64_t d = r % p.dim;
    float acc = p.bias ? __ldg(p.bias + d) : 0.f;
#pragma unroll
    for (int k = 0; k < K; ++k) acc = fmaf(__ldg(p.w + d * K + k), x_at<T>(p, r, t - (K - 1) + k), acc);
    static_cast<T*>(p.out)[r * p.L + t] = io<T>::from_f(p.silu ? silu(acc) : acc);
}

// final[r, k] = input K-1-k steps before the end of init ++ x (thread per (row, k)).
template <typename T>
__global__ void conv1d_final_kernel(const CParams p) {
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int km1 = p.K - 1;
    if (gid >= p.rows * km1) return;
    const int64_t r = gid / km1;
    const int k = (int)(gid - r * km1);
    const float v = x_at<T>(p, r, p.L - km1 + k);
    static_cast<T*>(p.fin)[r * km1 + k] = io<T>::from_f(v);
}

// Decode: state (rows, K-1) holds the previous K-1 inputs, oldest first.  Grid (channel
// blocks, batch): thread (d, b) owns row b * dim + d.
template <typename T, int K>
__global__ void __launch_bounds__(256) conv1d_update_kernel(T* state, const T* x, const float* w,
                                                            const float* bias, T* out,
                                                            int64_t dim, int silu_on) {
    const int64_t d = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (d >= dim) return;
    const int64_t r = (int64_t)blockIdx.y * dim + d;
    float win[K];
#pragma unroll
    for (int k = 0; k < K - 1; ++k) win[k] = io<T>::to_f(state[r * (K - 1) + k]);
    win[K - 1] = io<T>::to_f(x[r]);
    float acc = bias ? __ldg(bias + d) : 0.f;
#pragma unroll
    for (int k = 0; k < K; ++k) acc = fmaf(__ldg(w + d * K + k), win[k], acc);
    out[r] = io<T>::from_f(silu_on ? silu(acc) : acc);
#pragma unroll
    for (int k = 0; k < K - 1; ++k) state[r * (K - 1) + k] = io<T>::from_f(win[k + 1]);
}

unsigned blocks_for(int64_t threads) { return (unsigned)((threads + 255) / 256); }

template <typename T, int K>
cudaError_t launch_conv_k(const CParams& p, cudaStream_t s) {
    constexpr int E = 16 / sizeof(T);
    if (p.L > 0) {
        const int64_t vpr = p.L / E;
        const int64_t batch = p.rows / p.dim;
        if (p.L % E == 0 && K - 1 <= E && p.dim <= 65535 && batch <= 65535 &&
            (vpr + 256 * kVPT - 1) / (256 * kVPT) <= 0x7fffffff) {
            const dim3 grid((unsigned)((vpr + 256 * kVPT - 1) / (256 * kVPT)), (unsigned)p.dim,
                            (unsigned)batch);
            conv1d_vec_kernel<T, K><<<grid, 256, 0, s>>>(p);
        } else if (p.L % E == 0 && K - 1 <= E) {
            conv1d_vec1d_kernel<T, K><<<blocks_for(p.rows * vpr), 256, 0, s>>>(p);
        } else {
            conv1d_elem_kernel<T, K><<<blocks_for(p.rows * p.L), 256, 0, s>>>(p);
        }
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (p.fin && K > 1) {
        conv1d_final_kernel<T><<<blocks_for(p.rows * (K - 1)), 256, 0, s>>>(p);
        return cudaGetLastError();
    }
    return cudaSuccess;
}

template <typename T>
cudaError_t launch_conv_t(const CParams& p, cudaStream_t s) {
    switch (p.K) {
        case 1: return launch_conv_k<T, 1>(p, s);
        case 2: return launch_conv_k<T, 2>(p, s);
        case 3: return launch_conv_k<T, 3>(p, s);
        case 4: return launch_conv_k<T, 4>(p, s);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T>
cudaError_t launch_update_t(const ConvUpdateArgs& a, cudaStream_t s) {
    T* st = static_cast<T*>(a.state);
    const T* x = static_cast<const T*>(a.x);
    T* out = static_cast<T*>(a.out);
    if (a.batch > 65535) return cudaErrorInvalidConfiguration;
    const dim3 grid(blocks_for(a.dim), (unsigned)a.batch);
    switch (a.width) {
        case 1: conv1d_update_kernel<T, 1><<<grid, 256, 0, s>>>(st, x, a.weight, a.bias, out, a.dim, a.silu); break;
        case 2: conv1d_update_kernel<T, 2><<<grid, 256, 0, s>>>(st, x, a.weight, a.bias, out, a.dim, a.silu); break;
        case 3: conv1d_update_kernel<T, 3><<<grid, 256, 0, s>>>(st, x, a.weight, a.bias, out, a.dim, a.silu); break;
        case 4: conv1d_update_kernel<T, 4><<<grid, 256, 0, s>>>(st, x, a.weight, a.bias, out, a.dim, a.silu); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_conv1d(const ConvArgs& a, cudaStream_t stream) {
    CParams p;
    memset(&p, 0, sizeof(p));
    p.x = a.x;
    p.w = a.weight;
    p.bias = a.bias;
    p.init = a.initial_state;
    p.out = a.out;
    p.fin = a.final_state;
    p.rows = a.batch * a.dim;
    p.dim = a.dim;
    p.L = a.L;
    p.K = a.width;
    p.silu = a.silu ? 1 : 0;
    if (a.dtype == DType::BF16) return launch_conv_t<__nv_bfloat16>(p, stream);
    return launch_conv_t<float>(p, stream);
}

cudaError_t launch_conv1d_update(const ConvUpdateArgs& a, cudaStream_t stream) {
    if (a.dtype == DType::BF16) return launch_update_t<__nv_bfloat16>(a, stream);
    return launch_update_t<float>(a, stream);
}

}  // namespace s6
