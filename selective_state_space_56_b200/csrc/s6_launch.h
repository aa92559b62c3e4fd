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
    int zoh;  // nonzero: exact zero-order-hold Bbar = (exp(Delta A) - 1) / A * B
    DType in_dtype, out_dtype;
    // sequence split (nseg == 1: single pass, no workspace)
    int64_t nseg, seg_len;
    float* seg_h;    // (nseg, batch, dim, N)
    float* seg_sum;  // (nseg, batch, dim)
    const float* h0;  // (batch, dim, N) initial state or null (zero)
    float* ckpt;      // backward checkpoints to record, or null (layout of launch_scan_checkpoints)
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
    int zoh;  // as in ScanArgs
    DType io_dtype;
};

// A split sequence's segments are multiples of this many steps (a multiple of every
// chunk length a scan kernel stages at once).
constexpr int kChunk = 128;

// Split plan for a problem: number of segments and their length (a multiple of kChunk),
// no more segments than one wave of the current device's CTAs holds for the input type.
void plan_segments(int64_t batch, int64_t dim, int64_t dstate, int64_t L, int64_t* nseg,
                   int64_t* seg_len, bool fp32_in);
// Most segments plan_segments can return for these sizes (what the workspace is sized for).
int64_t split_segments_bound(int64_t batch, int64_t dim, int64_t L);

// Each returns a cudaError_t from the launches (cudaSuccess when all were enqueued).
cudaError_t launch_scan(const ScanArgs& a, cudaStream_t stream);
cudaError_t launch_state_update(const StateUpdateArgs& a, cudaStream_t stream);

// Summary of the whole sequence in `a` (its plan's segments folded): the end state from
// h = 0 into h_end (batch, dim, N) and the summed step into dsum (batch, dim).  With
// a.nseg > 1 the segment aggregates go through a.seg_h / a.seg_sum.
cudaError_t launch_scan_summary(const ScanArgs& a, float* h_end, float* dsum, cudaStream_t stream);

// Inclusive fold of `count` summaries (hend (count, batch, dim, N), dsum (count, batch, dim))
// applied to h0 (or zero): the state after them and (when dsum_out) their total step.
cudaError_t launch_fold(const float* hend, const float* dsum, const float* A, const float* h0,
                        int64_t count, int64_t batch, int64_t dim, int64_t N, float* h_out,
                        float* dsum_out, cudaStream_t stream);

// Steps per chunk of the forward kernel for state width N.
int scan_chunk_steps(int64_t N);

// Steps between the backward's checkpoints: the state entering every group of 4 steps,
// the unit the reverse sweep recomputes from (so it runs no forward pass of its own).
constexpr int kCkptSteps = 4;
int checkpoint_steps(int64_t N);
// Two layouts of the checkpoints (blocks = ceil(L / kCkptSteps)):
//   per channel  ckpt[((b * dim + d) * blocks + g) * N + n]: a channel's groups contiguous;
//   tile-major   ckpt[(((b * ntiles + d / kCkptTile) * blocks + g) * kCkptTile + d % kCkptTile)
//                * N + n], ntiles = ceil(dim / kCkptTile): the kCkptTile channels of the
//                sweep's CTA tile contiguous for each group, its groups one after another.
// Tile-major is used once a channel's checkpoints reach 1 MB (L * N >= 2^20): a block of the
// sweep then reads one contiguous piece instead of 32 pieces a channel's checkpoints apart
// (measured on the million-length layer (1, 2048, 16, 2^20): backward 131.3 -> 124.2 ms).
// Shorter sequences keep the per-channel layout (the 2.8B-shaped layer's backward 2.93 ms
// against 2.97 tile-major, its exact-ZOH backward 4.85 against 4.97).  Writer and reader
// both take the choice from ckpt_tiled(L, N).
constexpr int kCkptTile = 32;
__host__ __device__ inline bool ckpt_tiled(int64_t L, int64_t N) { return L * N >= (int64_t(1) << 20); }
__host__ __device__ inline int64_t ckpt_index(int64_t b, int64_t d, int64_t g, int64_t dim,
                                              int64_t blocks, int64_t N, bool tiled) {
    if (!tiled) return ((b * dim + d) * blocks + g) * N;
    const int64_t ntiles = (dim + kCkptTile - 1) / kCkptTile;
    return (((b * ntiles + d / kCkptTile) * blocks + g) * kCkptTile + d % kCkptTile) * N;
}
// Floats of the checkpoints of a (batch, dim, L, N) scan (the tile-major size, which covers
// the per-channel one).
inline int64_t ckpt_floats(int64_t batch, int64_t dim, int64_t L, int64_t N) {
    return batch * ((dim + kCkptTile - 1) / kCkptTile) * kCkptTile *
           ((L + kCkptSteps - 1) / kCkptSteps) * N;
}

// Forward pass that writes the state entering every checkpoint group to ckpt (the layout
// of ckpt_index), and no output.  Uses a.u, delta, A, B, C, delta_bias, softplus, dims and in_dtype.
// With a.nseg > 1 (a.seg_len a multiple of 64) the segments run side by side from their
// true starts, formed first in a.seg_h / a.seg_sum (nseg x batch x dim x N, and
// nseg x batch x dim floats).
cudaError_t launch_scan_checkpoints(const ScanArgs& a, float* ckpt, cudaStream_t stream);

// The backward's split of a long sequence over few channels into nseg segments of seg_len
// steps (a multiple of 64; nseg = 1 when it does not split).  Its workspace then holds,
// after the checkpoints (rounded up to 64 floats), nseg x batch x dim x (N + 1) floats.
void backward_segments(int64_t batch, int64_t dim, int64_t L, int64_t* nseg, int64_t* seg_len);

// Gradients of the scan (outputs of the backward); dy is read, the rest written.
struct BackwardArgs {
    const void* dy;     // (batch, dim, L) in_dtype
    void* du;           // (batch, dim, L) in_dtype
    void* ddelta;       // (batch, dim, L) in_dtype, gradient of the raw delta
    void* dz;           // (batch, dim, L) in_dtype, null when there is no gate
    float* dA;          // (dim, N)
    float* dB;          // (batch, N, L)
    float* dC;          // (batch, N, L)
    float* dD;          // (dim), null when there is no skip term
    float* ddelta_bias; // (dim), null when there is no bias
};

// Backward of the scan described by `a` (its y, last_state and segment fields are
// unused): zeroes the accumulated outputs, runs the checkpointing forward into
// `ckpt` (batch * dim * ceil(L / checkpoint_steps(N)) * N floats) -- unless ckpt_ready,
// when a training forward has recorded them already -- and then the reverse sweep.
cudaError_t launch_scan_backward(const ScanArgs& a, const BackwardArgs& g, float* ckpt,
                                 cudaStream_t stream, bool ckpt_ready = false);

// Causal depthwise conv1d (+ SiLU) over (batch, dim, L) rows, 1 <= width <= 4.
struct ConvArgs {
    const void* x;
    const float* weight;        // (dim, width)
    const float* bias;          // (dim) or null
    const void* initial_state;  // (batch, dim, width - 1) or null
    void* out;
    void* final_state;          // (batch, dim, width - 1) or null
    int64_t batch, dim, L;
    int width;
    int silu;
    DType dtype;
};

struct ConvUpdateArgs {
    void* state;  // (batch, dim, width - 1), updated in place
    const void* x;
    const float* weight;
    const float* bias;
    void* out;
    int64_t batch, dim;
    int width;
    int silu;
    DType dtype;
};

// Gradients of sum(out * dout) for the convolution above.
struct ConvBwdArgs {
    const void* x;
    const float* weight;        // (dim, width)
    const float* bias;          // (dim) or null
    const void* initial_state;  // (batch, dim, width - 1) or null
    const void* dout;           // (batch, dim, L)
    void* dx;                   // (batch, dim, L)
    float* dweight;             // (dim, width), zeroed here, then accumulated
    float* dbias;               // (dim) or null, likewise
    void* dinitial_state;       // (batch, dim, width - 1) or null (written with initial_state)
    int64_t batch, dim, L;
    int width;
    int silu;
    DType dtype;
};

cudaError_t launch_conv1d(const ConvArgs& a, cudaStream_t stream);
cudaError_t launch_conv1d_update(const ConvUpdateArgs& a, cudaStream_t stream);
cudaError_t launch_conv1d_bwd(const ConvBwdArgs& a, cudaStream_t stream);

// One bounded device wait that nothing completes: sets bit 0 of the device error word
// after limit_cycles SM clocks.
cudaError_t launch_wait_timeout_probe(long long limit_cycles, cudaStream_t stream);

// Reads (and optionally clears) the device error word on `stream`, synchronising it.
// Bit 0: a bounded device-side wait gave up.
cudaError_t read_device_error(unsigned* out, bool clear, cudaStream_t stream);

}  // namespace s6
