// s6_launch.h -- internal (C++) launch interface between the C ABI and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace s6 {

enum class DType : int { F32 = 0, BF16 = 1 };

// Everything one selective-scan call needs, already validated by the ABI layer.
struct ScanArgs {
    const void* u;
    const void* delta;
    const void* z;  // may be null
    const float* A;
    const void* B;
    const void* C;
    const float* D;           // may be null
    const float* delta_bias;  // may be null
    void* y;
    float* last_state;  // may be null
    int64_t batch, dim, N, L;
    int softplus;
    DType in_dtype, out_dtype;
    // sequence split (nseg == 1: single pass, no workspace)
    int64_t nseg, seg_len;
    float* seg_h;    // (nseg, batch, dim, N)
    float* seg_sum;  // (nseg, batch, dim)
};

struct StateUpdateArgs {
    float* state;
    const void* u;
    const void* delta;
    const void* z;
    const float* A;
    const void* B;
    const void* C;
    const float* D;
    const float* delta_bias;
    void* y;
    int64_t batch, dim, N;
    int softplus;
    DType io_dtype;
};

// A split sequence's segments are multiples of this many steps (a multiple of every
// chunk length a scan kernel stages at once).
constexpr int kChunk = 128;

// Split plan for a problem: number of segments and their length (a multiple of kChunk).
void plan_segments(int64_t batch, int64_t dim, int64_t L, int64_t* nseg, int64_t* seg_len);

// Each returns a cudaError_t from the launches (cudaSuccess when all were enqueued).
cudaError_t launch_scan(const ScanArgs& a, cudaStream_t stream);
cudaError_t launch_state_update(const StateUpdateArgs& a, cudaStream_t stream);

// Reads (and optionally clears) the device error word on `stream`, synchronising it.
// Bit 0: a bounded device-side wait gave up.
cudaError_t read_device_error(unsigned* out, bool clear, cudaStream_t stream);

}  // namespace s6
