// api.cu -- the extern "C" boundary declared in include/mamba_s6.h.
//
// Host-side only: validates every argument before anything is enqueued, turns
// the plain pointers and sizes into launch arguments and forwards to the kernel
// launchers.  No allocation, no synchronisation, no state kept between calls.
#include <stdint.h>

#include "../../include/mamba_s6.h"
#include "s6_launch.h"

namespace {

constexpr int64_t kMaxDstate = 16;
constexpr int64_t kMaxGridYZ = 65535;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool dtype_ok(int dt) { return dt == MAMBA_F32 || dt == MAMBA_BF16; }

s6::DType to_dtype(int dt) { return dt == MAMBA_BF16 ? s6::DType::BF16 : s6::DType::F32; }

bool mul_ok(int64_t a, int64_t b) { return a == 0 || b <= INT64_MAX / a; }

// Shared size checks: positive batch/dim, dstate in [1, 16], L >= 0, and every
// element count representable.
bool dims_ok(int64_t batch, int64_t dim, int64_t dstate, int64_t L) {
    if (batch < 1 || dim < 1 || dstate < 1 || dstate > kMaxDstate || L < 0) return false;
    if (batch > kMaxGridYZ) return false;
    if (!mul_ok(batch, dim)) return false;
    const int64_t bd = batch * dim;
    if (!mul_ok(bd, L) || !mul_ok(bd, dstate) || !mul_ok(bd * dstate, 8)) return false;
    if (!mul_ok(batch * dstate, L) || !mul_ok(bd * (L > 0 ? L : 1), 8)) return false;
    return (bd + 31) / 32 <= (int64_t)0x7fffffff;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA; }

constexpr unsigned kKnownFlags = MAMBA_FLAG_EXACT_ZOH;

int scan_fwd(const void* u, const void* delta, const float* A, const void* B, const void* C,
             const float* D, const void* z, const float* delta_bias, int delta_softplus,
             const float* h0, void* y, float* last_state, mamba_scan_dims dims,
             mamba_dtype in_dtype, mamba_dtype out_dtype, void* workspace,
             size_t workspace_bytes, unsigned flags, void* stream, float* ckpt = nullptr,
             size_t ckpt_bytes = 0);

int scan_bwd(const void* u, const void* delta, const float* A, const void* B, const void* C,
             const float* D, const void* z, const float* delta_bias, int delta_softplus,
             const void* dy, void* du, void* ddelta, void* dz, float* dA, float* dB, float* dC,
             float* dD, float* ddelta_bias, mamba_scan_dims dims, mamba_dtype in_dtype,
             void* ckpt, size_t ckpt_bytes, bool ckpt_ready, unsigned flags, void* stream);

int state_update(float* state, const void* u, const void* delta, const float* A, const void* B,
                 const void* C, const float* D, const void* z, const float* delta_bias,
                 int delta_softplus, void* y, int64_t batch, int64_t dim, int64_t dstate,
                 mamba_dtype io_dtype, unsigned flags, void* stream);

}  // namespace

extern "C" {

size_t mamba_selective_scan_workspace_size(mamba_scan_dims dims) {
    if (!dims_ok(dims.batch, dims.dim, dims.dstate, dims.seqlen)) return 0;
    // sized for the most segments the plan can take, so the size depends on the sizes alone
    const int64_t nseg = s6::split_segments_bound(dims.batch, dims.dim, dims.seqlen);
    if (nseg <= 1) return 0;
    const int64_t rows = nseg * dims.batch * dims.dim;
    // seg_h (rows x N) then seg_sum (rows), fp32; the tail rounded to 256 bytes
    const int64_t bytes = rows * (dims.dstate + 1) * 4;
    return (size_t)((bytes + 255) / 256 * 256);
}

int mamba_selective_scan_fwd(const void* u, const void* delta, const float* A, const void* B,
                             const void* C, const float* D, const void* z,
                             const float* delta_bias, int delta_softplus, void* y,
                             float* last_state, mamba_scan_dims dims, mamba_dtype in_dtype,
                             mamba_dtype out_dtype, void* workspace, size_t workspace_bytes,
                             void* stream) {
    return scan_fwd(u, delta, A, B, C, D, z, delta_bias, delta_softplus, nullptr, y, last_state,
                    dims, in_dtype, out_dtype, workspace, workspace_bytes, 0u, stream);
}

int mamba_selective_scan_fwd_ex(const void* u, const void* delta, const float* A, const void* B,
                                const void* C, const float* D, const void* z,
                                const float* delta_bias, int delta_softplus, void* y,
                                float* last_state, mamba_scan_dims dims, mamba_dtype in_dtype,
                                mamba_dtype out_dtype, void* workspace, size_t workspace_bytes,
                                unsigned flags, void* stream) {
    return scan_fwd(u, delta, A, B, C, D, z, delta_bias, delta_softplus, nullptr, y, last_state,
                    dims, in_dtype, out_dtype, workspace, workspace_bytes, flags, stream);
}

int mamba_selective_scan_fwd_init(const void* u, const void* delta, const float* A,
                                  const void* B, const void* C, const float* D, const void* z,
                                  const float* delta_bias, int delta_softplus,
                                  const float* initial_state, void* y, float* last_state,
                                  mamba_scan_dims dims, mamba_dtype in_dtype,
                                  mamba_dtype out_dtype, void* workspace, size_t workspace_bytes,
                                  unsigned flags, void* stream) {
    if (!initial_state) return MAMBA_ERR_NULL;
    return scan_fwd(u, delta, A, B, C, D, z, delta_bias, delta_softplus, initial_state, y,
                    last_state, dims, in_dtype, out_dtype, workspace, workspace_bytes, flags,
                    stream);
}

int mamba_selective_scan_summary(const void* u, const void* delta, const float* A, const void* B,
                                 const void* C, const float* delta_bias, int delta_softplus,
                                 float* h_end, float* delta_sum, mamba_scan_dims dims,
                                 mamba_dtype in_dtype, void* workspace, size_t workspace_bytes,
                                 unsigned flags, void* stream) {
    if (flags & ~kKnownFlags) return MAMBA_ERR_FLAGS;
    const bool empty = dims.seqlen == 0;
    if (!A || !h_end || !delta_sum || (!empty && (!u || !delta || !B || !C)))
        return MAMBA_ERR_NULL;
    if (!dtype_ok(in_dtype)) return MAMBA_ERR_DTYPE;
    if (!dims_ok(dims.batch, dims.dim, dims.dstate, dims.seqlen)) return MAMBA_ERR_DIMS;
    const void* ptrs[] = {u, delta, A, B, C, delta_bias, h_end, delta_sum};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return MAMBA_ERR_ALIGN;
    int64_t nseg = 1, seg_len = 0;
    s6::plan_segments(dims.batch, dims.dim, dims.dstate, dims.seqlen, &nseg, &seg_len,
                      in_dtype == MAMBA_F32);
    if (nseg > kMaxGridYZ) return MAMBA_ERR_DIMS;
    const size_t need = mamba_selective_scan_workspace_size(dims);
    if (need > 0) {
        if (!workspace || workspace_bytes < need) return MAMBA_ERR_WORKSPACE;
        if (!aligned16(workspace)) return MAMBA_ERR_ALIGN;
    }
    s6::ScanArgs a;
    a.u = u;
    a.delta = delta;
    a.z = nullptr;
    a.A = A;
    a.B = B;
    a.C = C;
    a.D = nullptr;
    a.delta_bias = delta_bias;
    a.y = nullptr;
    a.last_state = nullptr;
    a.batch = dims.batch;
    a.dim = dims.dim;
    a.N = dims.dstate;
    a.L = dims.seqlen;
    a.softplus = delta_softplus;
    a.zoh = (flags & MAMBA_FLAG_EXACT_ZOH) ? 1 : 0;
    a.in_dtype = to_dtype(in_dtype);
    a.out_dtype = a.in_dtype;
    a.nseg = nseg;
    a.seg_len = seg_len;
    a.seg_h = nullptr;
    a.seg_sum = nullptr;
    a.h0 = nullptr;
    a.ckpt = nullptr;
    if (nseg > 1) {
        a.seg_h = static_cast<float*>(workspace);
        a.seg_sum = a.seg_h + nseg * dims.batch * dims.dim * dims.dstate;
    }
    return cuda_status(s6::launch_scan_summary(a, h_end, delta_sum, static_cast<cudaStream_t>(stream)));
}

int mamba_selective_scan_fold(const float* h_ends, const float* delta_sums, const float* A,
                              const float* h0, int64_t count, int64_t batch, int64_t dim,
                              int64_t dstate, float* h_out, float* delta_sum_out, void* stream) {
    if (!A || !h_out || (count > 0 && (!h_ends || !delta_sums))) return MAMBA_ERR_NULL;
    if (count < 0 || !dims_ok(batch, dim, dstate, 0) || !mul_ok(batch * dim * dstate, count + 1))
        return MAMBA_ERR_DIMS;
    const void* ptrs[] = {h_ends, delta_sums, A, h0, h_out, delta_sum_out};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return MAMBA_ERR_ALIGN;
    return cuda_status(s6::launch_fold(h_ends, delta_sums, A, h0, count, batch, dim, dstate, h_out,
                                       delta_sum_out, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {

int scan_fwd(const void* u, const void* delta, const float* A, const void* B, const void* C,
             const float* D, const void* z, const float* delta_bias, int delta_softplus,
             const float* h0, void* y, float* last_state, mamba_scan_dims dims,
             mamba_dtype in_dtype, mamba_dtype out_dtype, void* workspace,
             size_t workspace_bytes, unsigned flags, void* stream, float* ckpt,
             size_t ckpt_bytes) {
    if (flags & ~kKnownFlags) return MAMBA_ERR_FLAGS;
    // With seqlen == 0 the (batch, dim, 0) and (batch, dstate, 0) arrays are empty and
    // may be NULL; only last_state (zeros) is written.
    const bool empty = dims.seqlen == 0;
    if (!A || (!empty && (!u || !delta || !B || !C || !y))) return MAMBA_ERR_NULL;
    if (!dtype_ok(in_dtype) || !dtype_ok(out_dtype)) return MAMBA_ERR_DTYPE;
    if (!dims_ok(dims.batch, dims.dim, dims.dstate, dims.seqlen)) return MAMBA_ERR_DIMS;
    const void* ptrs[] = {u, delta, A, B, C, D, z, delta_bias, y, last_state, h0, ckpt};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return MAMBA_ERR_ALIGN;
    if (ckpt && ckpt_bytes < mamba_selective_scan_bwd_workspace_size(dims))
        return MAMBA_ERR_WORKSPACE;

    int64_t nseg = 1, seg_len = 0;
    s6::plan_segments(dims.batch, dims.dim, dims.dstate, dims.seqlen, &nseg, &seg_len,
                      in_dtype == MAMBA_F32);
    if (nseg > kMaxGridYZ) return MAMBA_ERR_DIMS;
    const size_t need = mamba_selective_scan_workspace_size(dims);
    if (need > 0) {
        if (!workspace || workspace_bytes < need) return MAMBA_ERR_WORKSPACE;
        if (!aligned16(workspace)) return MAMBA_ERR_ALIGN;
    }

    s6::ScanArgs a;
    a.u = u;
    a.delta = delta;
    a.z = z;
    a.A = A;
    a.B = B;
    a.C = C;
    a.D = D;
    a.delta_bias = delta_bias;
    a.y = y;
    a.last_state = last_state;
    a.batch = dims.batch;
    a.dim = dims.dim;
    a.N = dims.dstate;
    a.L = dims.seqlen;
    a.softplus = delta_softplus;
    a.zoh = (flags & MAMBA_FLAG_EXACT_ZOH) ? 1 : 0;
    a.in_dtype = to_dtype(in_dtype);
    a.out_dtype = to_dtype(out_dtype);
    a.nseg = nseg;
    a.seg_len = seg_len;
    a.seg_h = nullptr;
    a.seg_sum = nullptr;
    a.h0 = h0;
    a.ckpt = ckpt;
    if (nseg > 1) {
        a.seg_h = static_cast<float*>(workspace);
        a.seg_sum = a.seg_h + nseg * dims.batch * dims.dim * dims.dstate;
    }
    return cuda_status(s6::launch_scan(a, static_cast<cudaStream_t>(stream)));
}

int state_update(float* state, const void* u, const void* delta, const float* A, const void* B,
                 const void* C, const float* D, const void* z, const float* delta_bias,
                 int delta_softplus, void* y, int64_t batch, int64_t dim, int64_t dstate,
                 mamba_dtype io_dtype, unsigned flags, void* stream) {
    if (flags & ~kKnownFlags) return MAMBA_ERR_FLAGS;
    if (!state || !u || !delta || !A || !B || !C || !y) return MAMBA_ERR_NULL;
    if (!dtype_ok(io_dtype)) return MAMBA_ERR_DTYPE;
    if (!dims_ok(batch, dim, dstate, 1)) return MAMBA_ERR_DIMS;
    const void* ptrs[] = {state, u, delta, A, B, C, D, z, delta_bias, y};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return MAMBA_ERR_ALIGN;
    s6::StateUpdateArgs a;
    a.state = state;
    a.u = u;
    a.delta = delta;
    a.z = z;
    a.A = A;
    a.B = B;
    a.C = C;
    a.D = D;
    a.delta_bias = delta_bias;
    a.y = y;
    a.batch = batch;
    a.dim = dim;
    a.N = dstate;
    a.softplus = delta_softplus;
    a.zoh = (flags & MAMBA_FLAG_EXACT_ZOH) ? 1 : 0;
    a.io_dtype = to_dtype(io_dtype);
    return cuda_status(s6::launch_state_update(a, static_cast<cudaStream_t>(stream)));
}

}  // namespace

extern "C" {

int mamba_selective_state_update(float* state, const void* u, const void* delta, const float* A,
                                 const void* B, const void* C, const float* D, const void* z,
                                 const float* delta_bias, int delta_softplus, void* y,
                                 int64_t batch, int64_t dim, int64_t dstate,
                                 mamba_dtype io_dtype, void* stream) {
    return state_update(state, u, delta, A, B, C, D, z, delta_bias, delta_softplus, y, batch, dim,
                        dstate, io_dtype, 0u, stream);
}

int mamba_selective_state_update_ex(float* state, const void* u, const void* delta,
                                    const float* A, const void* B, const void* C, const float* D,
                                    const void* z, const float* delta_bias, int delta_softplus,
                                    void* y, int64_t batch, int64_t dim, int64_t dstate,
                                    mamba_dtype io_dtype, unsigned flags, void* stream) {
    return state_update(state, u, delta, A, B, C, D, z, delta_bias, delta_softplus, y, batch, dim,
                        dstate, io_dtype, flags, stream);
}

size_t mamba_selective_scan_bwd_workspace_size(mamba_scan_dims dims) {
    if (!dims_ok(dims.batch, dims.dim, dims.dstate, dims.seqlen)) return 0;
    // checkpoints: sized for the tile-major layout (the channel count padded to whole
    // tiles), which also holds the per-channel one used for shorter sequences
    const int64_t dpad = (dims.dim + s6::kCkptTile - 1) / s6::kCkptTile * s6::kCkptTile;
    const int64_t T = s6::checkpoint_steps(dims.dstate);
    const int64_t chunks = (dims.seqlen + T - 1) / T;
    if (!mul_ok(dims.batch * dpad, chunks) || !mul_ok(dims.batch * dpad * chunks, dims.dstate * 4))
        return 0;
    int64_t floats = (s6::ckpt_floats(dims.batch, dims.dim, dims.seqlen, dims.dstate) + 63) / 64 * 64;
    int64_t nseg = 1, seg_len = 0;
    s6::backward_segments(dims.batch, dims.dim, dims.seqlen, &nseg, &seg_len);
    if (nseg > 1) {  // the segments' adjoint summaries and summed steps
        if (!mul_ok(nseg * dims.batch * dims.dim, dims.dstate + 1)) return 0;
        floats += nseg * dims.batch * dims.dim * (dims.dstate + 1);
    }
    const int64_t bytes = floats * 4;
    return (size_t)((bytes + 255) / 256 * 256);
}

int mamba_selective_scan_bwd(const void* u, const void* delta, const float* A, const void* B,
                             const void* C, const float* D, const void* z,
                             const float* delta_bias, int delta_softplus, const void* dy,
                             void* du, void* ddelta, void* dz, float* dA, float* dB, float* dC,
                             float* dD, float* ddelta_bias, mamba_scan_dims dims,
                             mamba_dtype in_dtype, void* workspace, size_t workspace_bytes,
                             void* stream) {
    return scan_bwd(u, delta, A, B, C, D, z, delta_bias, delta_softplus, dy, du, ddelta, dz, dA,
                    dB, dC, dD, ddelta_bias, dims, in_dtype, workspace, workspace_bytes, false, 0u,
                    stream);
}

int mamba_selective_scan_bwd_ex(const void* u, const void* delta, const float* A, const void* B,
                                const void* C, const float* D, const void* z,
                                const float* delta_bias, int delta_softplus, const void* dy,
                                void* du, void* ddelta, void* dz, float* dA, float* dB, float* dC,
                                float* dD, float* ddelta_bias, mamba_scan_dims dims,
                                mamba_dtype in_dtype, void* workspace, size_t workspace_bytes,
                                unsigned flags, void* stream) {
    return scan_bwd(u, delta, A, B, C, D, z, delta_bias, delta_softplus, dy, du, ddelta, dz, dA,
                    dB, dC, dD, ddelta_bias, dims, in_dtype, workspace, workspace_bytes, false,
                    flags, stream);
}

int mamba_selective_scan_fwd_train(const void* u, const void* delta, const float* A,
                                   const void* B, const void* C, const float* D, const void* z,
                                   const float* delta_bias, int delta_softplus, void* y,
                                   float* last_state, mamba_scan_dims dims, mamba_dtype in_dtype,
                                   mamba_dtype out_dtype, void* workspace,
                                   size_t workspace_bytes, float* checkpoints,
                                   size_t checkpoint_bytes, void* stream) {
    if (!checkpoints && dims.seqlen > 0) return MAMBA_ERR_NULL;
    return scan_fwd(u, delta, A, B, C, D, z, delta_bias, delta_softplus, nullptr, y, last_state,
                    dims, in_dtype, out_dtype, workspace, workspace_bytes, 0u, stream,
                    dims.seqlen > 0 ? checkpoints : nullptr, checkpoint_bytes);
}

int mamba_selective_scan_bwd_from_checkpoints(
    const void* u, const void* delta, const float* A, const void* B, const void* C,
    const float* D, const void* z, const float* delta_bias, int delta_softplus, const void* dy,
    void* du, void* ddelta, void* dz, float* dA, float* dB, float* dC, float* dD,
    float* ddelta_bias, mamba_scan_dims dims, mamba_dtype in_dtype, const float* checkpoints,
    size_t checkpoint_bytes, void* stream) {
    return scan_bwd(u, delta, A, B, C, D, z, delta_bias, delta_softplus, dy, du, ddelta, dz, dA,
                    dB, dC, dD, ddelta_bias, dims, in_dtype, const_cast<float*>(checkpoints),
                    checkpoint_bytes, true, 0u, stream);
}

int mamba_selective_scan_fwd_train_ex(const void* u, const void* delta, const float* A,
                                      const void* B, const void* C, const float* D, const void* z,
                                      const float* delta_bias, int delta_softplus, void* y,
                                      float* last_state, mamba_scan_dims dims, mamba_dtype in_dtype,
                                      mamba_dtype out_dtype, void* workspace,
                                      size_t workspace_bytes, float* checkpoints,
                                      size_t checkpoint_bytes, unsigned flags, void* stream) {
    if (!checkpoints && dims.seqlen > 0) return MAMBA_ERR_NULL;
    return scan_fwd(u, delta, A, B, C, D, z, delta_bias, delta_softplus, nullptr, y, last_state,
                    dims, in_dtype, out_dtype, workspace, workspace_bytes, flags, stream,
                    dims.seqlen > 0 ? checkpoints : nullptr, checkpoint_bytes);
}

int mamba_selective_scan_bwd_from_checkpoints_ex(
    const void* u, const void* delta, const float* A, const void* B, const void* C,
    const float* D, const void* z, const float* delta_bias, int delta_softplus, const void* dy,
    void* du, void* ddelta, void* dz, float* dA, float* dB, float* dC, float* dD,
    float* ddelta_bias, mamba_scan_dims dims, mamba_dtype in_dtype, const float* checkpoints,
    size_t checkpoint_bytes, unsigned flags, void* stream) {
    return scan_bwd(u, delta, A, B, C, D, z, delta_bias, delta_softplus, dy, du, ddelta, dz, dA,
                    dB, dC, dD, ddelta_bias, dims, in_dtype, const_cast<float*>(checkpoints),
                    checkpoint_bytes, true, flags, stream);
}

}  // extern "C"

namespace {

int scan_bwd(const void* u, const void* delta, const float* A, const void* B, const void* C,
             const float* D, const void* z, const float* delta_bias, int delta_softplus,
             const void* dy, void* du, void* ddelta, void* dz, float* dA, float* dB, float* dC,
             float* dD, float* ddelta_bias, mamba_scan_dims dims, mamba_dtype in_dtype,
             void* workspace, size_t workspace_bytes, bool ckpt_ready, unsigned flags,
             void* stream) {
    if (flags & ~kKnownFlags) return MAMBA_ERR_FLAGS;
    const bool empty = dims.seqlen == 0;
    if (!A || !dA) return MAMBA_ERR_NULL;
    if (!empty && (!u || !delta || !B || !C || !dy || !du || !ddelta || !dB || !dC))
        return MAMBA_ERR_NULL;
    // a gradient is present exactly when its input is
    if ((D == nullptr) != (dD == nullptr) || (delta_bias == nullptr) != (ddelta_bias == nullptr))
        return MAMBA_ERR_NULL;
    if (!empty && (z == nullptr) != (dz == nullptr)) return MAMBA_ERR_NULL;
    if (!dtype_ok(in_dtype)) return MAMBA_ERR_DTYPE;
    if (!dims_ok(dims.batch, dims.dim, dims.dstate, dims.seqlen)) return MAMBA_ERR_DIMS;
    const void* ptrs[] = {u, delta, A, B, C, D, z, delta_bias, dy, du, ddelta, dz,
                          dA, dB, dC, dD, ddelta_bias};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return MAMBA_ERR_ALIGN;
    const size_t need = mamba_selective_scan_bwd_workspace_size(dims);
    if (need > 0) {
        if (!workspace || workspace_bytes < need) return MAMBA_ERR_WORKSPACE;
        if (!aligned16(workspace)) return MAMBA_ERR_ALIGN;
    }
    s6::ScanArgs a;
    a.u = u;
    a.delta = delta;
    a.z = z;
    a.A = A;
    a.B = B;
    a.C = C;
    a.D = D;
    a.delta_bias = delta_bias;
    a.y = nullptr;
    a.last_state = nullptr;
    a.batch = dims.batch;
    a.dim = dims.dim;
    a.N = dims.dstate;
    a.L = dims.seqlen;
    a.softplus = delta_softplus;
    a.zoh = (flags & MAMBA_FLAG_EXACT_ZOH) ? 1 : 0;
    a.in_dtype = to_dtype(in_dtype);
    a.out_dtype = a.in_dtype;
    a.nseg = 1;
    a.seg_len = dims.seqlen;
    a.seg_h = nullptr;
    a.seg_sum = nullptr;
    a.h0 = nullptr;
    a.ckpt = nullptr;
    s6::BackwardArgs g;
    g.dy = dy;
    g.du = du;
    g.ddelta = ddelta;
    g.dz = dz;
    g.dA = dA;
    g.dB = dB;
    g.dC = dC;
    g.dD = dD;
    g.ddelta_bias = ddelta_bias;
    return cuda_status(s6::launch_scan_backward(a, g, static_cast<float*>(workspace),
                                                static_cast<cudaStream_t>(stream), ckpt_ready));
}

}  // namespace

extern "C" {

int mamba_causal_conv1d_fwd(const void* x, const float* weight, const float* bias,
                            const void* initial_state, void* out, void* final_state,
                            int64_t batch, int64_t dim, int64_t seqlen, int width, int silu,
                            mamba_dtype dtype, void* stream) {
    if (!weight || (seqlen > 0 && (!x || !out))) return MAMBA_ERR_NULL;
    if (!dtype_ok(dtype)) return MAMBA_ERR_DTYPE;
    if (width < 1 || width > 4 || batch < 1 || dim < 1 || seqlen < 0) return MAMBA_ERR_DIMS;
    if (!mul_ok(batch, dim) || !mul_ok(batch * dim, seqlen > 0 ? seqlen : 1) ||
        !mul_ok(batch * dim * (seqlen > 0 ? seqlen : 1), 8))
        return MAMBA_ERR_DIMS;
    const void* ptrs[] = {x, weight, bias, initial_state, out, final_state};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return MAMBA_ERR_ALIGN;
    s6::ConvArgs a;
    a.x = x;
    a.weight = weight;
    a.bias = bias;
    a.initial_state = width > 1 ? initial_state : nullptr;
    a.out = out;
    a.final_state = width > 1 ? final_state : nullptr;
    a.batch = batch;
    a.dim = dim;
    a.L = seqlen;
    a.width = width;
    a.silu = silu;
    a.dtype = to_dtype(dtype);
    return cuda_status(s6::launch_conv1d(a, static_cast<cudaStream_t>(stream)));
}

int mamba_causal_conv1d_update(void* conv_state, const void* x, const float* weight,
                               const float* bias, void* out, int64_t batch, int64_t dim,
                               int width, int silu, mamba_dtype dtype, void* stream) {
    if (!x || !weight || !out || (width > 1 && !conv_state)) return MAMBA_ERR_NULL;
    if (!dtype_ok(dtype)) return MAMBA_ERR_DTYPE;
    if (width < 1 || width > 4 || batch < 1 || dim < 1 || batch > kMaxGridYZ ||
        !mul_ok(batch, dim) || !mul_ok(batch * dim, 8))
        return MAMBA_ERR_DIMS;
    const void* ptrs[] = {conv_state, x, weight, bias, out};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return MAMBA_ERR_ALIGN;
    s6::ConvUpdateArgs a;
    a.state = conv_state;
    a.x = x;
    a.weight = weight;
    a.bias = bias;
    a.out = out;
    a.batch = batch;
    a.dim = dim;
    a.width = width;
    a.silu = silu;
    a.dtype = to_dtype(dtype);
    return cuda_status(s6::launch_conv1d_update(a, static_cast<cudaStream_t>(stream)));
}

int mamba_causal_conv1d_bwd(const void* x, const float* weight, const float* bias,
                            const void* initial_state, const void* dout, void* dx,
                            float* dweight, float* dbias, void* dinitial_state, int64_t batch,
                            int64_t dim, int64_t seqlen, int width, int silu, mamba_dtype dtype,
                            void* stream) {
    if (!weight || !dweight || (seqlen > 0 && (!x || !dout || !dx))) return MAMBA_ERR_NULL;
    if (!dtype_ok(dtype)) return MAMBA_ERR_DTYPE;
    if (width < 1 || width > 4 || batch < 1 || dim < 1 || seqlen < 0) return MAMBA_ERR_DIMS;
    if (!mul_ok(batch, dim) || !mul_ok(batch * dim, seqlen > 0 ? seqlen : 1) ||
        !mul_ok(batch * dim * (seqlen > 0 ? seqlen : 1), 8))
        return MAMBA_ERR_DIMS;
    const void* ptrs[] = {x, weight, bias, initial_state, dout, dx, dweight, dbias, dinitial_state};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return MAMBA_ERR_ALIGN;
    s6::ConvBwdArgs a;
    a.x = x;
    a.weight = weight;
    a.bias = bias;
    a.initial_state = width > 1 ? initial_state : nullptr;
    a.dout = dout;
    a.dx = dx;
    a.dweight = dweight;
    a.dbias = dbias;
    a.dinitial_state = width > 1 ? dinitial_state : nullptr;
    a.batch = batch;
    a.dim = dim;
    a.L = seqlen;
    a.width = width;
    a.silu = silu;
    a.dtype = to_dtype(dtype);
    return cuda_status(s6::launch_conv1d_bwd(a, static_cast<cudaStream_t>(stream)));
}

int mamba_diag_wait_timeout(int64_t limit_cycles, void* stream) {
    if (limit_cycles < 1 || limit_cycles > 4000000000LL) return MAMBA_ERR_DIMS;
    return cuda_status(s6::launch_wait_timeout_probe((long long)limit_cycles,
                                                     static_cast<cudaStream_t>(stream)));
}

int mamba_check_device_error(int clear, void* stream) {
    unsigned word = 0;
    if (s6::read_device_error(&word, clear != 0, static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return MAMBA_ERR_CUDA;
    return word ? MAMBA_ERR_TIMEOUT : MAMBA_OK;
}

const char* mamba_status_string(int status) {
    switch (status) {
        case MAMBA_OK: return "ok";
        case MAMBA_ERR_NULL: return "a required pointer is NULL";
        case MAMBA_ERR_DIMS: return "invalid sizes (batch, dim >= 1; 1 <= dstate <= 16; seqlen >= 0)";
        case MAMBA_ERR_ALIGN: return "a pointer is not 16-byte aligned";
        case MAMBA_ERR_DTYPE: return "unknown dtype";
        case MAMBA_ERR_WORKSPACE: return "workspace missing or too small";
        case MAMBA_ERR_CUDA: return "CUDA runtime error";
        case MAMBA_ERR_TIMEOUT: return "a bounded device wait timed out";
        case MAMBA_ERR_FLAGS: return "unknown flag bits";
        default: return "unknown status";
    }
}

int mamba_abi_version(void) { return 105; }

}  // extern "C"
