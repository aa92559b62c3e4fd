/*
 * mamba_s6.h -- C ABI of the B200 (sm_100a) selective-scan library.
 *
 * Operations, each a hand-written CUDA kernel sequence launched on the caller's stream:
 *
 *   mamba_selective_scan_fwd      the fused S6 forward scan over a whole sequence
 *   mamba_selective_state_update  one decode token, updating a carried state in place
 *   mamba_selective_scan_bwd      gradients of the forward scan, states recomputed
 *                                 (_ex: also for the exact zero-order-hold forward)
 *   mamba_causal_conv1d_fwd       the block's causal conv1d + SiLU producing the scan's u
 *   mamba_causal_conv1d_update    its one-token decode step on a rolling conv state
 *   mamba_causal_conv1d_bwd       the gradients of that convolution (training)
 *
 * Definitions (Mamba: Linear-Time Sequence Modeling with Selective State Spaces,
 * page "xyznot.com/ar/paper/2312.00752", sections "Method", "Selection mechanism
 * (S6)" and "Hardware-aware state expansion"; page "yongjin360.com/news/29389",
 * serial scan, parallel-scan derivation steps 1-4 and the Q&A):
 *
 *   Delta_t  = softplus(delta[t] + delta_bias)   (or delta[t] + delta_bias when
 *                                                 delta_softplus == 0)
 *   Abar_t,n = exp(Delta_t * A[n])                ZOH discretisation of a diagonal A
 *   h_t,n    = Abar_t,n * h_{t-1},n + Delta_t * B[n,t] * u[t]     (h_{-1} = 0)
 *   y[t]     = (sum_n C[n,t] * h_t,n + D * u[t]) * silu(z[t]),  silu(x) = x / (1 + e^-x)
 *
 * per independent (batch, channel) lane.  B and C are per token and shared by
 * all channels of a batch; A, D and delta_bias are per channel.  The expanded
 * (batch, L, dim, N) state never reaches device memory: it lives in registers.
 *
 * Conventions for every entry point:
 *   - All array pointers are DEVICE pointers owned by the caller, contiguous in
 *     the layouts stated below (last dimension fastest), 16-byte aligned.  The
 *     library keeps no pointer after a call returns and allocates nothing.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls are
 *     asynchronous: they enqueue kernels and return without synchronising.
 *   - Argument errors are detected on the host before anything is launched and
 *     return a negative mamba_status; nothing is written in that case.
 *   - A launch failure reported by the CUDA runtime returns MAMBA_ERR_CUDA.
 *   - Outputs must not alias inputs (except `state`, which is updated in place).
 */
#ifndef MAMBA_S6_H
#define MAMBA_S6_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { MAMBA_F32 = 0, MAMBA_BF16 = 1 } mamba_dtype;

typedef enum {
    MAMBA_OK = 0,
    MAMBA_ERR_NULL = -1,      /* a required pointer is NULL                         */
    MAMBA_ERR_DIMS = -2,      /* a size is negative, too large, or dstate not 1..16 */
    MAMBA_ERR_ALIGN = -3,     /* a pointer is not 16-byte aligned                   */
    MAMBA_ERR_DTYPE = -4,     /* an unknown dtype enum                              */
    MAMBA_ERR_WORKSPACE = -5, /* workspace missing or smaller than required          */
    MAMBA_ERR_CUDA = -6,      /* the CUDA runtime reported an error                 */
    MAMBA_ERR_TIMEOUT = -7,   /* a bounded device-side wait gave up                 */
    MAMBA_ERR_FLAGS = -8      /* unknown bits in a flags argument                   */
} mamba_status;

/*
 * Flags of the _ex entry points.
 *
 * MAMBA_FLAG_EXACT_ZOH: discretise B with the exact zero-order hold of the "Method"
 * section, Bbar = (Delta A)^-1 (exp(Delta A) - I) Delta B -- for the diagonal A, per
 * state Bbar_n = (exp(Delta A_n) - 1) / A_n * B_n (Delta B_n when A_n = 0) -- instead of
 * Bbar = Delta * B.  The kernels form (exp(Delta A_n) - 1) / A_n from the same
 * exponential as Abar where |Delta A_n| >= 1/16 and from the series of expm1(y) / y
 * below, so the weight stays accurate as Delta A_n -> 0.
 */
#define MAMBA_FLAG_EXACT_ZOH 1u

/* Problem sizes: batch >= 1, dim >= 1, 1 <= dstate <= 16, seqlen >= 0. */
typedef struct {
    int64_t batch;
    int64_t dim;    /* d_inner: channels */
    int64_t dstate; /* N: state width per channel */
    int64_t seqlen; /* L */
} mamba_scan_dims;

/*
 * Bytes of device workspace mamba_selective_scan_fwd needs for `dims`.
 *
 * Zero unless the sequence is split into segments (few channels, long L: the
 * "million-length" regime).  Then the scan runs as three launches -- per-segment
 * aggregates (the segment's state from h = 0 and its summed step), the exclusive
 * prefix of the associative combine (Abar_j Abar_i, Abar_j b_i + b_j) across
 * segments (parallel-scan derivation, steps 2-4), and a final pass from each
 * segment's true initial state -- and the workspace holds the aggregates.  The size
 * covers the most segments a plan for `dims` may take (segments x batch x dim x
 * (dstate + 1) x 4 bytes); a launch may use fewer, e.g. to keep its CTAs in one wave.
 * Depends on `dims` only.  Returns 0 for invalid dims.
 */
size_t mamba_selective_scan_workspace_size(mamba_scan_dims dims);

/*
 * Fused selective-scan forward.
 *
 *   u, delta, z : (batch, dim, seqlen)  in_dtype       z may be NULL (no gate)
 *   A           : (dim, dstate)         float32        any real values (Mamba uses A < 0)
 *   B, C        : (batch, dstate, seqlen) in_dtype
 *   D           : (dim) float32 or NULL (no skip term)
 *   delta_bias  : (dim) float32 or NULL (no bias)
 *   delta_softplus : nonzero applies softplus to delta + delta_bias
 *   y           : (batch, dim, seqlen)  out_dtype      written
 *   last_state  : (batch, dim, dstate)  float32 or NULL; receives h_{L-1} (zeros when L = 0)
 *   (when seqlen == 0, u, delta, z, B, C and y hold no elements and may be NULL)
 *   workspace   : device buffer of at least mamba_selective_scan_workspace_size(dims)
 *                 bytes, or NULL when that size is 0; its contents on entry do not matter
 *
 * Accumulation and state are float32; exp/log run on the SFU (ex2/lg2/rcp).
 * Errors: NULL (required pointer), DIMS, ALIGN, DTYPE, WORKSPACE, CUDA.
 */
int mamba_selective_scan_fwd(const void* u, const void* delta, const float* A, const void* B,
                             const void* C, const float* D, const void* z,
                             const float* delta_bias, int delta_softplus, void* y,
                             float* last_state, mamba_scan_dims dims, mamba_dtype in_dtype,
                             mamba_dtype out_dtype, void* workspace, size_t workspace_bytes,
                             void* stream);

/*
 * mamba_selective_scan_fwd with a flags word (MAMBA_FLAG_EXACT_ZOH, or 0 for exactly
 * mamba_selective_scan_fwd).  Same arguments, layouts, workspace and errors, plus
 * MAMBA_ERR_FLAGS for unknown bits.
 */
int mamba_selective_scan_fwd_ex(const void* u, const void* delta, const float* A, const void* B,
                                const void* C, const float* D, const void* z,
                                const float* delta_bias, int delta_softplus, void* y,
                                float* last_state, mamba_scan_dims dims, mamba_dtype in_dtype,
                                mamba_dtype out_dtype, void* workspace, size_t workspace_bytes,
                                unsigned flags, void* stream);

/*
 * mamba_selective_scan_fwd_ex starting from a given state instead of h_{-1} = 0.
 *
 *   initial_state : (batch, dim, dstate) float32, required; read only
 *
 * Everything else as mamba_selective_scan_fwd_ex (last_state receives the state after
 * the sequence; with seqlen == 0 that is initial_state).  With the two calls below this
 * lets a sequence be split over devices: the segment of device r starts from the fold of
 * the summaries of segments 0..r-1.
 */
int mamba_selective_scan_fwd_init(const void* u, const void* delta, const float* A,
                                  const void* B, const void* C, const float* D, const void* z,
                                  const float* delta_bias, int delta_softplus,
                                  const float* initial_state, void* y, float* last_state,
                                  mamba_scan_dims dims, mamba_dtype in_dtype,
                                  mamba_dtype out_dtype, void* workspace, size_t workspace_bytes,
                                  unsigned flags, void* stream);

/*
 * Summary of a sequence (segment) for the associative combine of the parallel-scan
 * derivation (page "yongjin360.com/news/29389", steps 1-4): the segment as one
 * transformation T = (prod_t Abar_t, h_end) with h_end the state after the segment from
 * h = 0.  For the diagonal A, prod_t Abar_t,n = exp(A_n * sum_t Delta_t), so the summary is
 *
 *   h_end     : (batch, dim, dstate) float32   state after the segment from zero
 *   delta_sum : (batch, dim) float32           sum over the segment of Delta_t
 *
 * Inputs as mamba_selective_scan_fwd (D and z do not enter the state and are not taken).
 * workspace: at least mamba_selective_scan_workspace_size(dims) bytes (long segments with
 * few channels are themselves split).  flags: MAMBA_FLAG_EXACT_ZOH or 0.
 * Errors: NULL, DIMS, ALIGN, DTYPE, WORKSPACE, FLAGS, CUDA.
 */
int mamba_selective_scan_summary(const void* u, const void* delta, const float* A, const void* B,
                                 const void* C, const float* delta_bias, int delta_softplus,
                                 float* h_end, float* delta_sum, mamba_scan_dims dims,
                                 mamba_dtype in_dtype, void* workspace, size_t workspace_bytes,
                                 unsigned flags, void* stream);

/*
 * Applies `count` consecutive segment summaries, in order, to h0 (NULL = zero): the
 * combine (prod Abar_j, h_j) (+) state = prod Abar_j * state + h_j, folded left to right
 * (page "yongjin360.com/news/29389", steps 2-4).
 *
 *   h_ends     : (count, batch, dim, dstate) float32     summaries' end states
 *   delta_sums : (count, batch, dim) float32             summaries' summed steps
 *   A          : (dim, dstate) float32
 *   h_out      : (batch, dim, dstate) float32            the state after the segments
 *   delta_sum_out : (batch, dim) float32 or NULL         the total summed step
 *
 * count == 0 gives h_out = h0 (or zero).  Errors: NULL, DIMS, ALIGN, CUDA.
 */
int mamba_selective_scan_fold(const float* h_ends, const float* delta_sums, const float* A,
                              const float* h0, int64_t count, int64_t batch, int64_t dim,
                              int64_t dstate, float* h_out, float* delta_sum_out, void* stream);

/*
 * One decode token (selective_state_update): the recurrence above for a single
 * t, applied in place to a carried state (the generation mode keeps only a
 * fixed dim x dstate state per layer and costs O(1) per token).
 *
 *   state       : (batch, dim, dstate) float32, read and overwritten in place
 *   u, delta, z : (batch, dim)   io_dtype       z may be NULL
 *   A           : (dim, dstate)  float32
 *   B, C        : (batch, dstate) io_dtype
 *   D, delta_bias : (dim) float32 or NULL
 *   y           : (batch, dim)   io_dtype       written
 *
 * Errors: NULL, DIMS (batch, dim >= 1; 1 <= dstate <= 16), ALIGN, DTYPE, CUDA.
 */
int mamba_selective_state_update(float* state, const void* u, const void* delta, const float* A,
                                 const void* B, const void* C, const float* D, const void* z,
                                 const float* delta_bias, int delta_softplus, void* y,
                                 int64_t batch, int64_t dim, int64_t dstate,
                                 mamba_dtype io_dtype, void* stream);

/*
 * mamba_selective_state_update with a flags word (MAMBA_FLAG_EXACT_ZOH, or 0).  Same
 * arguments and errors, plus MAMBA_ERR_FLAGS for unknown bits.
 */
int mamba_selective_state_update_ex(float* state, const void* u, const void* delta,
                                    const float* A, const void* B, const void* C, const float* D,
                                    const void* z, const float* delta_bias, int delta_softplus,
                                    void* y, int64_t batch, int64_t dim, int64_t dstate,
                                    mamba_dtype io_dtype, unsigned flags, void* stream);

/*
 * mamba_selective_scan_fwd for callers that cannot allocate device memory.  (This
 * entry point has no counterpart in the method's description; it only changes where
 * scratch memory comes from.)
 *
 * Some callers may not allocate: extension code inside a host framework that owns the
 * whole device-memory budget, or latency-sensitive code that cannot afford cudaMalloc /
 * cudaFree, which may synchronise the device.  mamba_selective_scan_fwd needs a
 * caller-provided workspace whenever it splits a long sequence into segments; this
 * variant instead uses a fixed 2.25 MiB scratch array compiled into the library and
 * calls no allocator.  Arguments, layouts and results are those of
 * mamba_selective_scan_fwd (without the workspace arguments).
 *
 *   - Limit: when the split plan needs more than 2.25 MiB (segments x batch x dim x
 *     (dstate + 1) x 4 bytes) the call returns MAMBA_ERR_WORKSPACE and launches
 *     nothing.  The million-length layer (1, 2048, 16, 2^20) needs 2.125 MiB.
 *   - The array exists on every GPU that loads the library and stays allocated until
 *     the process exits.  The first call on a device (with that device current) looks
 *     up the array's device address; make that first call before any stream capture.
 *     The address is kept per device and driver context: a call under a different
 *     current context looks it up again.  After cudaDeviceReset the module may be
 *     loaded at a new address under an identical context handle, so do not use this
 *     entry point on a device after resetting it.
 *   - Every call shares the one array and it keeps the last call's contents; the scan
 *     writes each entry before reading it, so nothing needs clearing.  Calls whose
 *     kernels overlap on the GPU (e.g. on two streams at once) race on the array:
 *     serialise them.
 */
int mamba_selective_scan_fwd_noalloc(const void* u, const void* delta, const float* A,
                                     const void* B, const void* C, const float* D, const void* z,
                                     const float* delta_bias, int delta_softplus, void* y,
                                     float* last_state, mamba_scan_dims dims,
                                     mamba_dtype in_dtype, mamba_dtype out_dtype, void* stream);

/*
 * Bytes of device workspace mamba_selective_scan_bwd needs for `dims`: the checkpoints,
 * the state entering every group of 4 steps, batch x dim' x ceil(seqlen / 4) x dstate
 * floats with dim' = dim rounded up to a multiple of 32 (16 bytes per (batch, channel,
 * step) at dstate = 16; stored [batch][dim][group][dstate] while seqlen * dstate < 2^20,
 * tile-major [batch][dim' / 32][group][32][dstate] beyond), rounded up to 64 floats; plus,
 * when a long sequence over few channels is
 * swept in S segments side by side (seqlen >= 16384 and fewer CTAs of 32 channels than two
 * per SM of the current device; S up to five CTAs per SM, segments of at least 4096 steps),
 * S x batch x dim x (dstate + 1) floats for the segments' summaries.  Rounded up to 256
 * bytes (0 when seqlen == 0).  Returns 0 for invalid dims.
 */
size_t mamba_selective_scan_bwd_workspace_size(mamba_scan_dims dims);

/*
 * Backward of mamba_selective_scan_fwd: given dy = dLoss/dy, writes the gradients of
 * every input.  The intermediate states are not read from memory (the forward never
 * stored them); as the method's hardware-aware algorithm prescribes, they are
 * recomputed: a forward pass records the state entering every T-step block in the
 * workspace, and a reverse sweep rebuilds each chunk's states from its record
 * before propagating the adjoint state backwards through it (Mamba, section
 * "Hardware-aware state expansion").  A long sequence over few channels (see the
 * workspace size above) is swept in segments side by side: the checkpoints from each
 * segment's true start, then each segment's adjoint summary and their fold (the
 * adjoint obeys a linear recurrence backwards in time, so segments combine as the
 * forward's do), then every segment's sweep from the adjoint entering it.
 *
 *   u, delta, A, B, C, D, z, delta_bias, delta_softplus, dims, in_dtype
 *               : exactly the forward's inputs (same layouts and rules)
 *   dy          : (batch, dim, seqlen)  in_dtype       gradient of y
 *   du, ddelta  : (batch, dim, seqlen)  in_dtype       written; ddelta is the gradient
 *                                                      of the raw delta (before the
 *                                                      bias and softplus)
 *   dz          : (batch, dim, seqlen)  in_dtype       written; NULL iff z is NULL
 *   dA          : (dim, dstate)         float32        written (summed over batch, t)
 *   dB, dC      : (batch, dstate, seqlen) float32      written (summed over channels)
 *   dD          : (dim) float32                        written; NULL iff D is NULL
 *   ddelta_bias : (dim) float32                        written; NULL iff delta_bias is NULL
 *   workspace   : at least mamba_selective_scan_bwd_workspace_size(dims) bytes; its
 *                 contents on entry do not matter
 *
 * The backward is that of the Bbar = Delta * B discretisation (the forward without
 * flags); mamba_selective_scan_bwd_ex below takes the flags word of the forward.
 * dA, dB, dC, dD and ddelta_bias are sums over many CTAs, formed with float32
 * atomics: their last bits may differ between runs.  With seqlen == 0 the
 * per-token arrays may be NULL and dA, dD, ddelta_bias are set to zero.
 * Errors: NULL (a required pointer, or a gradient whose presence does not match its
 * input's), DIMS, ALIGN, DTYPE, WORKSPACE, CUDA.
 */
int mamba_selective_scan_bwd(const void* u, const void* delta, const float* A, const void* B,
                             const void* C, const float* D, const void* z,
                             const float* delta_bias, int delta_softplus, const void* dy,
                             void* du, void* ddelta, void* dz, float* dA, float* dB, float* dC,
                             float* dD, float* ddelta_bias, mamba_scan_dims dims,
                             mamba_dtype in_dtype, void* workspace, size_t workspace_bytes,
                             void* stream);

/*
 * Training forward: mamba_selective_scan_fwd that also records the backward's checkpoints
 * (the state entering every group of 4 steps -- the layout the backward's own
 * recomputing pass writes), so that a following
 * mamba_selective_scan_bwd_from_checkpoints needs no forward pass of its own.
 *
 *   checkpoints      : device buffer of at least mamba_selective_scan_bwd_workspace_size(dims)
 *                      bytes, written (may be NULL when seqlen == 0)
 *   everything else  : as mamba_selective_scan_fwd (no flags: the Delta * B form; the _ex
 *                      form below takes the flags word)
 *
 * Errors: as mamba_selective_scan_fwd, plus WORKSPACE when checkpoint_bytes is too small.
 */
int mamba_selective_scan_fwd_train(const void* u, const void* delta, const float* A,
                                   const void* B, const void* C, const float* D, const void* z,
                                   const float* delta_bias, int delta_softplus, void* y,
                                   float* last_state, mamba_scan_dims dims, mamba_dtype in_dtype,
                                   mamba_dtype out_dtype, void* workspace,
                                   size_t workspace_bytes, float* checkpoints,
                                   size_t checkpoint_bytes, void* stream);

/*
 * mamba_selective_scan_bwd with the flags word of the forward: with MAMBA_FLAG_EXACT_ZOH
 * the gradients are those of the exact zero-order-hold forward (Mamba, section "Method":
 * Bbar = (Delta A)^-1 (exp(Delta A) - I) Delta B, per state w = expm1(Delta A_n) / A_n
 * times B_n, the weight Delta where A_n = 0), its states recomputed the same way.  The
 * weight's own derivatives enter: dB gains g w u instead of g Delta u, du the sum over
 * states of g w B, dDelta the sum of g B u dw/dDelta (dw/dDelta = exp(Delta A)), dA the sum
 * of g B u dw/dA (dw/dA = Delta^2 psi(Delta A), psi(y) = (y e^y - expm1(y)) / y^2, taken
 * from its series where |Delta A| < 1/2).  flags = 0 is exactly mamba_selective_scan_bwd.
 * Errors: as mamba_selective_scan_bwd, and FLAGS for unknown flag bits.
 */
int mamba_selective_scan_bwd_ex(const void* u, const void* delta, const float* A, const void* B,
                                const void* C, const float* D, const void* z,
                                const float* delta_bias, int delta_softplus, const void* dy,
                                void* du, void* ddelta, void* dz, float* dA, float* dB, float* dC,
                                float* dD, float* ddelta_bias, mamba_scan_dims dims,
                                mamba_dtype in_dtype, void* workspace, size_t workspace_bytes,
                                unsigned flags, void* stream);

/*
 * mamba_selective_scan_bwd from the checkpoints a mamba_selective_scan_fwd_train call
 * recorded for the same inputs (read only): the same gradients, without the backward's
 * own checkpointing forward pass.  Arguments as mamba_selective_scan_bwd with the
 * checkpoints in place of the workspace.
 */
int mamba_selective_scan_bwd_from_checkpoints(
    const void* u, const void* delta, const float* A, const void* B, const void* C,
    const float* D, const void* z, const float* delta_bias, int delta_softplus, const void* dy,
    void* du, void* ddelta, void* dz, float* dA, float* dB, float* dC, float* dD,
    float* ddelta_bias, mamba_scan_dims dims, mamba_dtype in_dtype, const float* checkpoints,
    size_t checkpoint_bytes, void* stream);

/*
 * The training pair with the flags word: mamba_selective_scan_fwd_train_ex records the
 * checkpoints of the forward the flags select (MAMBA_FLAG_EXACT_ZOH: the exact zero-order
 * hold of mamba_selective_scan_fwd_ex, states and checkpoints with the weight
 * w = expm1(Delta A) / A), and mamba_selective_scan_bwd_from_checkpoints_ex returns the
 * gradients of mamba_selective_scan_bwd_ex with the same flags from them.  Both calls of a
 * pair take the same flags; flags = 0 is exactly the plain pair.
 * Errors: as mamba_selective_scan_fwd_train / mamba_selective_scan_bwd_from_checkpoints,
 * and FLAGS for unknown flag bits.
 */
int mamba_selective_scan_fwd_train_ex(const void* u, const void* delta, const float* A,
                                      const void* B, const void* C, const float* D, const void* z,
                                      const float* delta_bias, int delta_softplus, void* y,
                                      float* last_state, mamba_scan_dims dims, mamba_dtype in_dtype,
                                      mamba_dtype out_dtype, void* workspace,
                                      size_t workspace_bytes, float* checkpoints,
                                      size_t checkpoint_bytes, unsigned flags, void* stream);
int mamba_selective_scan_bwd_from_checkpoints_ex(
    const void* u, const void* delta, const float* A, const void* B, const void* C,
    const float* D, const void* z, const float* delta_bias, int delta_softplus, const void* dy,
    void* du, void* ddelta, void* dz, float* dA, float* dB, float* dC, float* dD,
    float* ddelta_bias, mamba_scan_dims dims, mamba_dtype in_dtype, const float* checkpoints,
    size_t checkpoint_bytes, unsigned flags, void* stream);

/*
 * Causal depthwise conv1d with an optional SiLU: the Mamba block's step between the input
 * projection and the SSM (Mamba, section "Mamba Block": input projections, a 1-D
 * convolution, the selective SSM and gating; page "yongjin360.com/news/29389", Q&A on
 * the convolution before the SSM and the activation after it).  Per (batch, channel) row:
 *
 *   out[t] = act(bias[d] + sum_{k=0}^{width-1} weight[d, k] * x[t - (width-1) + k])
 *
 * where positions before the sequence read initial_state (the width-1 preceding inputs,
 * oldest first) or zero when it is NULL, and act is SiLU when silu != 0.
 *
 *   x, out        : (batch, dim, seqlen) dtype     out must not alias x
 *   weight        : (dim, width) float32           1 <= width <= 4
 *   bias          : (dim) float32 or NULL
 *   initial_state : (batch, dim, width-1) dtype or NULL
 *   final_state   : (batch, dim, width-1) dtype or NULL; receives the last width-1 inputs
 *                   of initial_state ++ x, oldest first (the state decode continues from)
 *   (with seqlen == 0, x and out may be NULL)
 *
 * fp32 arithmetic; results rounded to dtype.  Errors: NULL, DIMS, ALIGN, DTYPE, CUDA.
 */
int mamba_causal_conv1d_fwd(const void* x, const float* weight, const float* bias,
                            const void* initial_state, void* out, void* final_state,
                            int64_t batch, int64_t dim, int64_t seqlen, int width, int silu,
                            mamba_dtype dtype, void* stream);

/*
 * One decode token of the convolution above: conv_state (batch, dim, width-1) holds the
 * previous width-1 inputs, oldest first, and is updated in place (oldest dropped, x
 * appended); out (batch, dim) = act(bias + weight . [conv_state, x]).  x, out: (batch,
 * dim) dtype; conv_state may be NULL only when width == 1; batch <= 65535.
 * Errors: NULL, DIMS, ALIGN, DTYPE, CUDA.
 */
int mamba_causal_conv1d_update(void* conv_state, const void* x, const float* weight,
                               const float* bias, void* out, int64_t batch, int64_t dim,
                               int width, int silu, mamba_dtype dtype, void* stream);

/*
 * Gradients of sum_t out[b, d, t] * dout[b, d, t] for mamba_causal_conv1d_fwd with the same
 * x, weight, bias, initial_state, width and silu (the training side of the Mamba block's
 * convolution step; Mamba, section "Mamba Block", and the chain rule of the definition
 * above).  With pre[t] the value before the activation and g[t] = dout[t] * act'(pre[t])
 * (act' = 1 without SiLU, else sigmoid(p) (1 + p (1 - sigmoid(p)))):
 *
 *   dx[s]             = sum_k weight[d, k] * g[s + (width-1) - k]    (terms with t in [0, L))
 *   dweight[d, k]     = sum_{b,t} g[t] * xe[t - (width-1) + k]       (xe = initial_state ++ x)
 *   dbias[d]          = sum_{b,t} g[t]
 *   dinitial_state[j] = sum_{k <= j} weight[d, k] * g[j - k]         (j < width-1)
 *
 *   x, dout, dx     : (batch, dim, seqlen) dtype       dx must not alias x or dout
 *   weight          : (dim, width) float32             1 <= width <= 4
 *   bias            : (dim) float32 or NULL
 *   initial_state   : (batch, dim, width-1) dtype or NULL (zeros before the sequence)
 *   dweight         : (dim, width) float32, overwritten (the library zeroes, then sums)
 *   dbias           : (dim) float32 or NULL, overwritten likewise
 *   dinitial_state  : (batch, dim, width-1) dtype or NULL; written only when initial_state
 *                     is given (the zeros used without it have no gradient)
 *   (with seqlen == 0, x, dout and dx may be NULL; dweight and dbias become zero)
 *
 * fp32 arithmetic; dx and dinitial_state rounded to dtype; dweight and dbias are sums
 * formed with atomic adds, so their last bits may vary from call to call.
 * Errors: NULL, DIMS, ALIGN, DTYPE, CUDA.
 */
int mamba_causal_conv1d_bwd(const void* x, const float* weight, const float* bias,
                            const void* initial_state, const void* dout, void* dx,
                            float* dweight, float* dbias, void* dinitial_state, int64_t batch,
                            int64_t dim, int64_t seqlen, int width, int silu, mamba_dtype dtype,
                            void* stream);

/*
 * Reads the library's device error word on `stream`, synchronising that stream.
 * Every device-side wait in the kernels (on the completion barrier of an
 * asynchronous tile copy) is bounded to about a second; a wait that gives up sets
 * the word and its CTA stops instead of hanging the GPU.  With `clear` nonzero the
 * word is reset.  Returns MAMBA_OK, MAMBA_ERR_TIMEOUT if a wait gave up since the
 * last clear (outputs of that call are then undefined), or MAMBA_ERR_CUDA.
 */
int mamba_check_device_error(int clear, void* stream);

/*
 * Diagnostic for the failure-detection path: launches one bounded device-side wait on a
 * barrier that nothing completes.  It gives up after limit_cycles SM clocks (1 to 4e9;
 * about 2e6 per millisecond) and sets the device error word exactly as a lost transfer
 * in the scan would, so mamba_check_device_error then returns MAMBA_ERR_TIMEOUT.  No
 * fault, trap or unbounded wait is involved and the context stays usable.
 * Errors: DIMS (limit out of range), CUDA.
 */
int mamba_diag_wait_timeout(int64_t limit_cycles, void* stream);

/*
 * Diagnostic: evaluates 2^x for n floats three ways on the device -- the FMA-pipe
 * polynomial the scan uses for part of its Abar factors (out_fma), the SFU
 * ex2.approx instruction (out_sfu) and CUDA's exp2f (out_lib) -- so tests can bound
 * the polynomial's error.  All pointers are device arrays of n floats.
 * Errors: NULL, DIMS (n < 0), CUDA.
 */
int mamba_diag_exp2(const float* x, float* out_fma, float* out_sfu, float* out_lib, int64_t n,
                    void* stream);

/*
 * Diagnostic: throughput probe of the pipes the scan's roofline is stated against.
 * Launches `blocks` CTAs of 256 threads (1 to 2^20); every thread runs `iters` rounds
 * (1 to 2^24, with blocks * iters at most 2^28 so that one launch stays well under a
 * second) of 8 independent chains of one instruction: kind 0 = SFU ex2.approx.f32,
 * 1 = fp32 FMA, 2 = packed fp32x2 FMA (two fp32 results each).  The caller times the
 * launch on `stream`; results per launch = blocks * 256 * iters * 8 (kind 2: * 16).
 * sink: device array of blocks * 256 floats (caller-owned) that receives one value per
 * thread, so no chain is optimised away.  Reads nothing.
 * Errors: NULL, DIMS (kind, blocks or iters out of range), CUDA.
 */
int mamba_diag_throughput(int kind, int64_t blocks, int64_t iters, float* sink, void* stream);

/* A static, human-readable name for a status code. */
const char* mamba_status_string(int status);

/* ABI version of this library (major * 100 + minor). */
int mamba_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MAMBA_S6_H */
