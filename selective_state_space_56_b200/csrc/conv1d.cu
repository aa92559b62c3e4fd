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
#include <algorithm>
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

// Decode over several batch rows per thread: thread (d, row slice) takes rows b = by, by +
// gridDim.y, ... of channel d (up to R of them), loading the channel's weights and bias
// once and every row's state and input before any arithmetic; per row the arithmetic is
// that of conv1d_update_kernel.  Used when batch >= R.  Measured on (256, 5120), K = 4,
// bf16, L2 flushed: 12.3 us with one row per thread, 10.2 us with 4 (identical results),
// 8 no better (median 12.3 us).
#ifndef S6_CONVU_ROWS
#define S6_CONVU_ROWS 4
#endif
template <typename T, int K, int R>
__global__ void __launch_bounds__(256) conv1d_update_rows_kernel(T* state, const T* x, const float* w,
                                                                 const float* bias, T* out,
                                                                 int64_t dim, int64_t batch,
                                                                 int silu_on) {
    const int64_t d = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (d >= dim) return;
    float wk[K];
#pragma unroll
    for (int k = 0; k < K; ++k) wk[k] = __ldg(w + d * K + k);
    const float bv = bias ? __ldg(bias + d) : 0.f;
    float win[R][K];
    bool ok[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int64_t b = (int64_t)blockIdx.y + (int64_t)r * gridDim.y;
        ok[r] = b < batch;
        const int64_t row = (ok[r] ? b : 0) * dim + d;
#pragma unroll
        for (int k = 0; k < K - 1; ++k) win[r][k] = ok[r] ? io<T>::to_f(state[row * (K - 1) + k]) : 0.f;
        win[r][K - 1] = ok[r] ? io<T>::to_f(x[row]) : 0.f;
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
        if (!ok[r]) continue;
        const int64_t row = ((int64_t)blockIdx.y + (int64_t)r * gridDim.y) * dim + d;
        float acc = bv;
#pragma unroll
        for (int k = 0; k < K; ++k) acc = fmaf(wk[k], win[r][k], acc);
        out[row] = io<T>::from_f(silu_on ? silu(acc) : acc);
#pragma unroll
        for (int k = 0; k < K - 1; ++k) state[row * (K - 1) + k] = io<T>::from_f(win[r][k + 1]);
    }
}

// ---- Backward ------------------------------------------------------------------------
// Gradients of sum_t out[t] * dout[t] (the chain rule of the definition above): with
// pre[t] the value before the activation and g[t] = dout[t] * act'(pre[t]),
//   dx[s] = sum_k w[k] g[s + (K-1) - k],  dw[k] = sum_t g[t] xe[t - (K-1) + k],
//   dbias = sum_t g[t],  dinit[j] = sum_{k <= j} w[k] g[j - k]  (xe = init ++ x).
// Also a stream: x and dout read, dx written, 6 bytes per element in bf16.  A thread owns
// kVPT consecutive 16-byte vectors of dx of one row: it loads the x vectors before, over
// and after them and the dout vectors over and after them, recomputes pre and g over its
// steps plus the K-1 after them, correlates, and stores.  dw and dbias are summed over the
// CTA (one row per CTA) and added to global memory once per CTA.

struct CBParams {
    const void* x;
    const float* w;
    const float* bias;
    const void* init;
    const void* dout;
    void* dx;
    float* dw;
    float* db;
    void* dinit;
    int64_t dim, batch, L;
    int silu;
};

// act'(p) for SiLU: sigmoid(p) (1 + p (1 - sigmoid(p))).
__device__ __forceinline__ float dsilu(float p) {
    const float sg = rcp(1.f + ex2(-p * kLog2e));
    return sg * fmaf(p, 1.f - sg, 1.f);
}
// The same on a packed pair (each half rounded exactly as dsilu rounds it).
__device__ __forceinline__ f2 dsilu2(f2 p) {
    const f2 e = ex2x2(mul2(p, pack2(-kLog2e, -kLog2e)));
    float d0, d1;
    unpack2(add2(e, pack2(1.f, 1.f)), d0, d1);
    const f2 sg = pack2(rcp(d0), rcp(d1));
    return mul2(sg, fma2(p, sub2(pack2(1.f, 1.f), sg), pack2(1.f, 1.f)));
}

// Input at position s of row r of init ++ x (zero before init).
template <typename T>
__device__ __forceinline__ float xb_at(const CBParams& p, int64_t r, int64_t s, int K) {
    if (s >= 0) return io<T>::to_f(static_cast<const T*>(p.x)[r * p.L + s]);
    if (!p.init) return 0.f;
    return io<T>::to_f(static_cast<const T*>(p.init)[r * (K - 1) + (K - 1) + s]);
}

// Sum of the K + 1 partial sums (dw[0..K-1], dbias) over the CTA, added to row d's entries.
template <int K>
__device__ __forceinline__ void cta_add(const CBParams& p, int64_t d, float (&part)[K + 1],
                                        float* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int k = 0; k <= K; ++k)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part[k] += __shfl_xor_sync(0xffffffffu, part[k], o);
    if (lane == 0)
#pragma unroll
        for (int k = 0; k <= K; ++k) red[warp * (K + 1) + k] = part[k];
    __syncthreads();
    if ((int)threadIdx.x <= K) {
        float v = 0.f;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) v += red[w * (K + 1) + threadIdx.x];
        if ((int)threadIdx.x < K)
            atomicAdd(p.dw + d * K + threadIdx.x, v);
        else if (p.db)
            atomicAdd(p.db + d, v);
    }
    __syncthreads();  // red is reused by the next row
}

// Rows of 16-byte multiples.  Grid (vector blocks, min(dim, 65535), batch slices); each CTA
// walks channels d with stride gridDim.y and, for each, the batch rows b with stride
// gridDim.z, carrying its dweight / dbias partial sums across those rows and reducing them
// once per channel.  Steps go in packed pairs (two independent fp32 lanes per instruction,
// so every element is rounded as in the scalar form; only the order in which a thread's
// partial sums are added differs).
#ifndef S6_CONVB_VPT
#define S6_CONVB_VPT 2
#endif
constexpr int kVPTB = S6_CONVB_VPT;  // 16-byte dx vectors per thread in the backward

// Register budget of the vector kernel: four CTAs of 256 threads per SM (64 registers, a
// 24-byte spill) measured faster than the compiler's own choice (76 registers, three CTAs):
// 125.3 against 129.4 us for the 2.8B-shaped layer's conv (149.9 us before the packed
// pairs and the per-channel reduction).  0 leaves the choice to the compiler.
#ifndef S6_CONVB_MINB
#define S6_CONVB_MINB 4
#endif
#if S6_CONVB_MINB > 0
#define S6_CONVB_BOUNDS __launch_bounds__(256, S6_CONVB_MINB)
#else
#define S6_CONVB_BOUNDS __launch_bounds__(256)
#endif
template <typename T, int K, bool SILU>
__global__ void S6_CONVB_BOUNDS conv1d_bwd_vec_kernel(const CBParams p) {
    constexpr int kVPT = kVPTB;
    constexpr int E = 16 / sizeof(T);
    constexpr int NT = kVPT * E;  // steps of this thread
    __shared__ float red[8 * (K + 1)];
    const int64_t vpr = p.L / E;
    const int64_t v0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * kVPT;
    const bool active = v0 < vpr;
    for (int64_t d = blockIdx.y; d < p.dim; d += gridDim.y) {
        float w[K];
        f2 w2[K];
#pragma unroll
        for (int k = 0; k < K; ++k) {
            w[k] = __ldg(p.w + d * K + k);
            w2[k] = pack2(w[k], w[k]);
        }
        const float bias = p.bias ? __ldg(p.bias + d) : 0.f;
        const f2 bias2 = pack2(bias, bias);
        f2 part2[K + 1];  // even and odd steps of every batch row of this channel
#pragma unroll
        for (int k = 0; k <= K; ++k) part2[k] = pack2(0.f, 0.f);
        for (int64_t b = blockIdx.z; b < p.batch; b += gridDim.z) {
            const int64_t r = b * p.dim + d;
            if (active) {
                const T* xr = static_cast<const T*>(p.x) + r * p.L;
                const T* gr = static_cast<const T*>(p.dout) + r * p.L;
                const int64_t s0 = v0 * E;
                // x over [s0 - E, s0 + NT + E) and dout over [s0, s0 + NT + E): loads first
                uint4 xv[kVPT + 2], gv[kVPT + 1];
                const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                for (int i = 0; i < kVPT; ++i) {
                    const bool in = v0 + i < vpr;
                    xv[i + 1] = in ? *reinterpret_cast<const uint4*>(xr + (v0 + i) * E) : zero;
                    gv[i] = in ? *reinterpret_cast<const uint4*>(gr + (v0 + i) * E) : zero;
                }
                const bool nxt = v0 + kVPT < vpr;
                xv[kVPT + 1] = (K > 1 && nxt) ? *reinterpret_cast<const uint4*>(xr + (v0 + kVPT) * E) : zero;
                gv[kVPT] = (K > 1 && nxt) ? *reinterpret_cast<const uint4*>(gr + (v0 + kVPT) * E) : zero;
                xv[0] = (K > 1 && v0 > 0) ? *reinterpret_cast<const uint4*>(xr + (v0 - 1) * E) : zero;
                // xe[s0 - (K-1) + j] for j < NT + 2 (K-1), and dout[s0 + j] for j < NT + K - 1
                float xs[NT + 2 * (K - 1)];
                float gs[NT + K - 1];
#pragma unroll
                for (int j = 0; j < K - 1; ++j)
                    xs[j] = v0 > 0 ? io<T>::to_f(reinterpret_cast<const T*>(&xv[0])[E - (K - 1) + j])
                                   : xb_at<T>(p, r, j - (K - 1), K);
#pragma unroll
                for (int i = 0; i < kVPT; ++i)
#pragma unroll
                    for (int j = 0; j < E; ++j) {
                        xs[K - 1 + i * E + j] = io<T>::to_f(reinterpret_cast<const T*>(&xv[i + 1])[j]);
                        gs[i * E + j] = io<T>::to_f(reinterpret_cast<const T*>(&gv[i])[j]);
                    }
#pragma unroll
                for (int j = 0; j < K - 1; ++j) {
                    xs[K - 1 + NT + j] = io<T>::to_f(reinterpret_cast<const T*>(&xv[kVPT + 1])[j]);
                    gs[NT + j] = io<T>::to_f(reinterpret_cast<const T*>(&gv[kVPT])[j]);
                }
                // g over steps s0 .. s0 + NT + K - 2 (zero past the row: those dout are zero),
                // two steps per packed pair
                constexpr int NG = NT + K - 1;
                float g[NG];
#pragma unroll
                for (int j = 0; j + 1 < NG; j += 2) {
                    f2 pre = bias2;
#pragma unroll
                    for (int k = 0; k < K; ++k) pre = fma2(w2[k], pack2(xs[j + k], xs[j + k + 1]), pre);
                    f2 gg = pack2(gs[j], gs[j + 1]);
                    if (SILU) gg = mul2(gg, dsilu2(pre));
                    unpack2(gg, g[j], g[j + 1]);
                }
                if constexpr (NG % 2 == 1) {
                    float pre = bias;
#pragma unroll
                    for (int k = 0; k < K; ++k) pre = fmaf(w[k], xs[NG - 1 + k], pre);
                    g[NG - 1] = SILU ? gs[NG - 1] * dsilu(pre) : gs[NG - 1];
                }
                // this thread's share of dw and dbias (its own steps; past the row g and x
                // are zero and add nothing)
#pragma unroll
                for (int t = 0; t < NT; t += 2) {
                    const f2 gg = pack2(g[t], g[t + 1]);
#pragma unroll
                    for (int k = 0; k < K; ++k) part2[k] = fma2(gg, pack2(xs[t + k], xs[t + k + 1]), part2[k]);
                    part2[K] = add2(part2[K], gg);
                }
                // dx[s0 + t] = sum_k w[k] g[t + K-1-k]
#pragma unroll
                for (int i = 0; i < kVPT; ++i) {
                    if (v0 + i >= vpr) break;
                    alignas(16) T o[E];
#pragma unroll
                    for (int j = 0; j < E; j += 2) {
                        const int t = i * E + j;
                        f2 acc = pack2(0.f, 0.f);
#pragma unroll
                        for (int k = 0; k < K; ++k)
                            acc = fma2(w2[k], pack2(g[t + K - 1 - k], g[t + K - k]), acc);
                        float a0, a1;
                        unpack2(acc, a0, a1);
                        o[j] = io<T>::from_f(a0);
                        o[j + 1] = io<T>::from_f(a1);
                    }
                    *reinterpret_cast<uint4*>(static_cast<T*>(p.dx) + r * p.L + (v0 + i) * E) =
                        *reinterpret_cast<const uint4*>(o);
                }
                // the inputs before the sequence: dinit[j] = sum_{k <= j} w[k] g[j - k]
                if (K > 1 && v0 == 0 && p.init && p.dinit) {
#pragma unroll
                    for (int j = 0; j < K - 1; ++j) {
                        float acc = 0.f;
#pragma unroll
                        for (int k = 0; k <= j; ++k) acc = fmaf(w[k], g[j - k], acc);
                        static_cast<T*>(p.dinit)[r * (K - 1) + j] = io<T>::from_f(acc);
                    }
                }
            }
        }
        float part[K + 1];
#pragma unroll
        for (int k = 0; k <= K; ++k) {
            float lo, hi;
            unpack2(part2[k], lo, hi);
            part[k] = lo + hi;
        }
        cta_add<K>(p, d, part, red);
    }
}

// Any row length: one step per thread, the K values of g it needs formed from K x each;
// dweight / dbias partial sums carried across the batch rows of a channel as above.
template <typename T, int K, bool SILU>
__global__ void __launch_bounds__(256) conv1d_bwd_elem_kernel(const CBParams p) {
    __shared__ float red[8 * (K + 1)];
    const int64_t s = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const bool active = s < p.L;
    for (int64_t d = blockIdx.y; d < p.dim; d += gridDim.y) {
        float w[K];
#pragma unroll
        for (int k = 0; k < K; ++k) w[k] = __ldg(p.w + d * K + k);
        const float bias = p.bias ? __ldg(p.bias + d) : 0.f;
        float part[K + 1];
#pragma unroll
        for (int k = 0; k <= K; ++k) part[k] = 0.f;
        for (int64_t b = blockIdx.z; b < p.batch; b += gridDim.z) {
            const int64_t r = b * p.dim + d;
            if (active) {
                // g at steps s .. s + K - 1 (zero past the row)
                float g[K];
#pragma unroll
                for (int m = 0; m < K; ++m) {
                    const int64_t t = s + m;
                    g[m] = 0.f;
                    if (t < p.L) {
                        float pre = bias;
#pragma unroll
                        for (int k = 0; k < K; ++k) pre = fmaf(w[k], xb_at<T>(p, r, t - (K - 1) + k, K), pre);
                        const float dv = io<T>::to_f(static_cast<const T*>(p.dout)[r * p.L + t]);
                        g[m] = SILU ? dv * dsilu(pre) : dv;
                    }
                }
#pragma unroll
                for (int k = 0; k < K; ++k) part[k] = fmaf(g[0], xb_at<T>(p, r, s - (K - 1) + k, K), part[k]);
                part[K] += g[0];
                float acc = 0.f;
#pragma unroll
                for (int k = 0; k < K; ++k) acc = fmaf(w[k], g[K - 1 - k], acc);
                static_cast<T*>(p.dx)[r * p.L + s] = io<T>::from_f(acc);
                if (K > 1 && s == 0 && p.init && p.dinit) {
#pragma unroll
                    for (int j = 0; j < K - 1; ++j) {
                        float a = 0.f;
#pragma unroll
                        for (int k = 0; k <= j; ++k) a = fmaf(w[k], g[j - k], a);
                        static_cast<T*>(p.dinit)[r * (K - 1) + j] = io<T>::from_f(a);
                    }
                }
            }
        }
        cta_add<K>(p, d, part, red);
    }
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
    if (S6_CONVU_ROWS > 1 && a.batch >= S6_CONVU_ROWS) {
        constexpr int R = S6_CONVU_ROWS > 1 ? S6_CONVU_ROWS : 2;
        const dim3 rgrid(blocks_for(a.dim), (unsigned)((a.batch + R - 1) / R));
        switch (a.width) {
            case 1: conv1d_update_rows_kernel<T, 1, R><<<rgrid, 256, 0, s>>>(st, x, a.weight, a.bias, out, a.dim, a.batch, a.silu); break;
            case 2: conv1d_update_rows_kernel<T, 2, R><<<rgrid, 256, 0, s>>>(st, x, a.weight, a.bias, out, a.dim, a.batch, a.silu); break;
            case 3: conv1d_update_rows_kernel<T, 3, R><<<rgrid, 256, 0, s>>>(st, x, a.weight, a.bias, out, a.dim, a.batch, a.silu); break;
            case 4: conv1d_update_rows_kernel<T, 4, R><<<rgrid, 256, 0, s>>>(st, x, a.weight, a.bias, out, a.dim, a.batch, a.silu); break;
            default: return cudaErrorInvalidValue;
        }
        return cudaGetLastError();
    }
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

namespace {

// Batch slices of the grid: one (each CTA walks every batch row of its channels, reducing
// dweight / dbias once per channel) unless the channels and row blocks alone give fewer
// than 8 CTAs per SM.
unsigned batch_slices(int64_t xy_ctas, int64_t batch) {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
        sms = 148;
    const int64_t want = 8 * (int64_t)sms;
    int64_t gz = xy_ctas >= want ? 1 : (want + xy_ctas - 1) / xy_ctas;
    gz = std::min<int64_t>(std::min<int64_t>(gz, batch), 65535);
    return (unsigned)std::max<int64_t>(gz, 1);
}

template <typename T, int K, bool SILU>
cudaError_t launch_conv_bwd_ks(const CBParams& p, int64_t L, cudaStream_t s) {
    constexpr int E = 16 / sizeof(T);
    const unsigned gy = (unsigned)(p.dim < 65535 ? p.dim : 65535);
    if (L % E == 0 && K - 1 <= E) {
        const int64_t vpr = L / E;
        const unsigned gx = (unsigned)((vpr + 256 * kVPTB - 1) / (256 * kVPTB));
        const dim3 grid(gx, gy, batch_slices((int64_t)gx * gy, p.batch));
        conv1d_bwd_vec_kernel<T, K, SILU><<<grid, 256, 0, s>>>(p);
    } else {
        const unsigned gx = (unsigned)((L + 255) / 256);
        const dim3 grid(gx, gy, batch_slices((int64_t)gx * gy, p.batch));
        conv1d_bwd_elem_kernel<T, K, SILU><<<grid, 256, 0, s>>>(p);
    }
    return cudaGetLastError();
}

template <typename T, int K>
cudaError_t launch_conv_bwd_k(const CBParams& p, int64_t L, cudaStream_t s) {
    return p.silu ? launch_conv_bwd_ks<T, K, true>(p, L, s) : launch_conv_bwd_ks<T, K, false>(p, L, s);
}

template <typename T>
cudaError_t launch_conv_bwd_t(const CBParams& p, int K, cudaStream_t s) {
    switch (K) {
        case 1: return launch_conv_bwd_k<T, 1>(p, p.L, s);
        case 2: return launch_conv_bwd_k<T, 2>(p, p.L, s);
        case 3: return launch_conv_bwd_k<T, 3>(p, p.L, s);
        case 4: return launch_conv_bwd_k<T, 4>(p, p.L, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_conv1d_bwd(const ConvBwdArgs& a, cudaStream_t stream) {
    cudaError_t e = cudaMemsetAsync(a.dweight, 0, (size_t)a.dim * a.width * sizeof(float), stream);
    if (e == cudaSuccess && a.dbias)
        e = cudaMemsetAsync(a.dbias, 0, (size_t)a.dim * sizeof(float), stream);
    if (e != cudaSuccess || a.L == 0) {
        // an empty sequence: the gradients of the initial state are zero as well
        if (e == cudaSuccess && a.L == 0 && a.initial_state && a.dinitial_state && a.width > 1)
            e = cudaMemsetAsync(a.dinitial_state, 0,
                                (size_t)a.batch * a.dim * (a.width - 1) *
                                    (a.dtype == DType::BF16 ? 2 : 4), stream);
        return e;
    }
    CBParams p;
    memset(&p, 0, sizeof(p));
    p.x = a.x;
    p.w = a.weight;
    p.bias = a.bias;
    p.init = a.width > 1 ? a.initial_state : nullptr;
    p.dout = a.dout;
    p.dx = a.dx;
    p.dw = a.dweight;
    p.db = a.dbias;
    p.dinit = a.width > 1 ? a.dinitial_state : nullptr;
    p.dim = a.dim;
    p.batch = a.batch;
    p.L = a.L;
    p.silu = a.silu ? 1 : 0;
    if (a.dtype == DType::BF16) return launch_conv_bwd_t<__nv_bfloat16>(p, a.width, stream);
    return launch_conv_bwd_t<float>(p, a.width, stream);
}

}  // namespace s6
