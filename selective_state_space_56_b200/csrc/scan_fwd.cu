// scan_fwd.cu -- fused selective-scan (S6) forward for sm_100a.
//
// One CTA owns a tile of CH channels of one batch row (and, for a split sequence,
// one segment of L) and walks L in chunks of T steps:
//
//   stage     one thread issues 3-D TMA bulk-tensor loads of the chunk's u, delta, z
//             rows and the batch's B, C rows into shared memory (double-buffered,
//             completion on an mbarrier; the tensor edges are zero-filled by the
//             copy engine).  Rows whose length is not a multiple of 16 bytes cannot
//             be described to TMA and are staged element-wise instead;
//   convert   B, C of the chunk -> fp32, time-major, through 4x4 register blocks;
//   phase A   per (channel, t): Delta = softplus(delta + bias), Delta*u  (each warp
//             on its own channels, four steps per lane);
//   phase B   the recurrence.  P lanes share a channel, each holding NS = N/P states
//             in registers: Abar = 2^(Delta * A log2 e) on the SFU,
//             h = Abar h + (Delta u) B, partial y = sum C h, two states per packed
//             fp32x2 instruction.  The P partial sums of each t are combined by a
//             transpose-reduce over lanes (P - 1 shuffles per P steps), leaving one
//             lane with the complete C.h for one t;
//   phase C   y = (C.h + D u) * silu(z), rounded to the output type into a shared
//             tile that one thread writes back with a TMA bulk-tensor store.
//
// The expanded state (batch, L, dim, N) exists only in registers (Mamba,
// "Hardware-aware state expansion": load Delta, A, B, C to on-chip memory,
// discretise and scan there, contract with C to (batch, L, dim) before writing
// back).  The cross-chunk carry is the register state itself.
//
// A split sequence (few channels, long L) runs three launches that use the
// associative combine of the parallel-scan derivation: (1) each segment but the
// last scans from h = 0 and records its end state and its summed step size;
// (2) a carry kernel folds segments left to right, start_{s+1} =
// exp(A * sum Delta_s) * start_s + end_s (the pair (prod Abar, h_end) of segment s
// combined with the prefix before it); (3) every segment rescans from its true
// start state and writes y.
//
// Every wait on an mbarrier is bounded (about a second of SM clocks); a wait that
// gives up sets bit 0 of the device error word and the CTA leaves its loop.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>
#include <cstring>

#include "s6_device.cuh"
#include "s6_launch.h"

namespace s6 {

// Bit 0: a bounded device wait gave up (read and cleared through read_device_error).
__device__ unsigned int g_device_error = 0;

namespace {

constexpr long long kWaitLimitCycles = 2000000000LL;  // ~1 s at the SM clock

struct KParams {
    const void* u;
    const void* delta;
    const void* z;
    const float* A;
    const void* B;
    const void* C;
    const float* D;
    const float* delta_bias;
    void* y;
    float* last_state;
    float* seg_h;
    float* seg_sum;
    float* ckpt;  // checkpoint modes: the state entering every 4-step group (ckpt_index)
    int ck_tiled;  // ckpt_tiled(L, N): the checkpoints' layout
    int64_t batch, dim, L, seg_len;
    int N;
    int nseg;
    int softplus;
    int y_vec;  // L % 4 == 0: four outputs per vector store
    int y_tma;  // output rows are 16-byte multiples: tiles go back by TMA store
    int seg_first;  // kCorr: the segment of blockIdx.z = 0
};

// TMA descriptors of the operands (unused when rows are not 16-byte multiples).
struct TMaps {
    CUtensorMap u, dr, z, B, C, y;
};

// Four outputs as one 8-byte (bf16) or 16-byte (fp32) store.
__device__ __forceinline__ void store4(float* dst, const float (&o)[4]) {
    *reinterpret_cast<float4*>(dst) = make_float4(o[0], o[1], o[2], o[3]);
}
__device__ __forceinline__ void store4(__nv_bfloat16* dst, const float (&o)[4]) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(o[0], o[1]);
    __nv_bfloat162 hi = __floats2bfloat162_rn(o[2], o[3]);
    uint2 v;
    v.x = *reinterpret_cast<uint32_t*>(&lo);
    v.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(dst) = v;
}

// kFull: the scan itself; kAggregate: split-sequence pass 1 (end state and summed step
// per segment, no output); kCheckpoint: the backward's forward pass (the state at the
// start of every checkpoint block, no output); kFullAgg: the one-pass split -- every
// segment scanned from h = 0, writing y and its end state and summed step; kCorr: its
// correction -- from the segment's true start state with no input (h = Abar h), adding
// (C.h) * silu(z) to y until the state has decayed below fp32 resolution; kFullCkpt: the
// scan that also records
// those checkpoints (a training forward, so the backward needs no pass of its own).
enum Mode : int { kFull = 0, kAggregate = 1, kCheckpoint = 2, kFullCkpt = 3, kFullAgg = 4, kCorr = 5 };

// Tuning of the N = 16 instantiation: lanes per channel, warps per CTA, chunk length.
#ifndef S6_P16
#define S6_P16 4
#endif
#ifndef S6_WARPS16
#define S6_WARPS16 6
#endif
#ifndef S6_CHUNK
#define S6_CHUNK 32
#endif
// Coefficient tile format for bf16 inputs: 0 = B and C widened to fp32; 1 = B and C kept
// as bf16 pairs (half the shared-memory bytes, widened in registers); 2 = B in fp32, C as
// bf16 pairs.  fp32 inputs always use format 0.
#ifndef S6_BC_MODE
#define S6_BC_MODE 2
#endif
// Abar pairs evaluated on the FMA pipe (exp2_fma2) instead of the SFU: 0 = none,
// 1 = the second pair of every other step (a quarter of them), 2 = the second pair of
// every step (half).
#ifndef S6_PREEXP
#define S6_PREEXP 1  // Abar of a whole 4-step group before its updates (measured +1.7%)
#endif
// TMA path, producer warps: 0 = none (one CTA barrier per chunk); 1 = one producer warp
// stages every chunk and converts its coefficients; 2 = S6_WSP producer warps also form
// Delta and Delta u for every channel into a double-buffered ring.  With 1 or 2 the
// compute warps wait only on mbarriers and never for one another.  S6_WS forces a form
// for every plain forward; by default the plan picks form 2 for a grid of one wave at
// 2.5 to 3 CTAs per SM and form 0 otherwise (measured on one B200: the 2.8B-shaped layer,
// 428 CTAs, 609.8 -> 584.2 us with form 2; at batch 12, 1284 CTAs, 1602 -> 1640 us).
#ifndef S6_WSP
#define S6_WSP 2
#endif
// The checkpoint-recording forwards (the backward's own pass and the training forward)
// with the same plan-based producer form: measured neutral on the 2.8B-shaped layer
// (backward 3120 -> 3131 us, training step 3287 -> 3267 us with 16-step checkpoints;
// 2908 -> 2900 us and 3096 -> 3087 us with 4-step groups), so off.
#ifndef S6_WS_CKPT
#define S6_WS_CKPT 0
#endif
// The exact-ZOH forward with the same plan-based producer form.
#ifndef S6_ZOH_WS
#define S6_ZOH_WS 0
#endif
#ifndef S6_POLY
#define S6_POLY 0
#endif
// Channels per lane of the plain N = 16 forward: 2 lets one load and widening of a step's
// B and C serve two channels, halving the coefficient traffic through shared memory.
#ifndef S6_CPL16
#define S6_CPL16 1
#endif
#ifndef S6_WARPS16F
#define S6_WARPS16F S6_WARPS16
#endif
// Delta * A log2(e) formed for two consecutive steps of one state at once (the pair
// (Delta_t, Delta_t+1) is already adjacent in registers) instead of for two states of one
// step, which needs Delta copied into both halves of a pair first.  Measured 1.5% slower
// on the 2.8B-shaped layer (no fewer instructions, six more registers): off, except for
// the correction pass, which has no input term and always uses this form.
#ifndef S6_TPX
#define S6_TPX 0
#endif
// Abar of the next 4-step group computed while the current group's states update (one
// step's worth of exponentials before each step), instead of all of a group's before its
// own updates.
#ifndef S6_PIPE
#define S6_PIPE 0
#endif
// SiLU of four outputs with one shared reciprocal (silu4) instead of one each.
#ifndef S6_SILU4
#define S6_SILU4 1
#endif

constexpr size_t align128(size_t x) { return (x + 127) / 128 * 128; }

// Shared-memory carve-up for one instantiation.
template <int NMAX, int P, int WARPS_, int T_, typename Tin, typename Tout, int CPL_ = 1,
          int DQ = 1>
struct Layout {
    static constexpr int T = T_;
    static constexpr int CPL = CPL_;           // channels per lane
    static constexpr int NS = NMAX / P;        // states per lane and channel
    static constexpr int G = 32 / P;           // lane groups per warp
    static constexpr int CW = G * CPL;         // channels per warp
    static constexpr int WARPS = WARPS_;
    static constexpr int CH = WARPS * CW;      // channels per CTA
    static constexpr int THREADS = WARPS * 32;
    static constexpr int RS = T + 4;           // fp32 row stride: rows land 16 B apart in banks
    static constexpr size_t rows_bytes = (size_t)CH * T * sizeof(Tin);    // one of u, delta, z
    static constexpr size_t coef_bytes = (size_t)NMAX * T * sizeof(Tin);  // one of B, C
    static constexpr size_t off_dr = align128(rows_bytes);
    static constexpr size_t off_z = 2 * off_dr;
    static constexpr size_t off_B = 3 * off_dr;
    static constexpr size_t off_C = off_B + align128(coef_bytes);
    static constexpr size_t stage_bytes = off_C + align128(coef_bytes);
    // Per-step coefficients for the recurrence (format S6_BC_MODE for bf16 inputs, 0 for
    // fp32 inputs).  Two buffers (chunk parity), so a chunk's coefficients can be written
    // while the previous chunk's are still being read.
    static constexpr int kBC = sizeof(Tin) == 2 ? S6_BC_MODE : 0;
    static constexpr size_t coef_fp32_bytes = (size_t)T * NMAX * 4;
    static constexpr size_t coef_bytes_all =
        kBC == 0 ? 2 * coef_fp32_bytes : (kBC == 1 ? coef_fp32_bytes : coef_fp32_bytes * 3 / 2);
    static constexpr size_t off_coef = 2 * stage_bytes;
    static constexpr size_t off_del = off_coef + 2 * coef_bytes_all;   // float [CH][RS]
    static constexpr size_t dq_stride = (size_t)CH * RS;                // floats per Delta buffer
    static constexpr size_t off_du = off_del + DQ * (size_t)CH * RS * 4;
    static constexpr size_t off_y = off_du + DQ * (size_t)CH * RS * 4;
    static constexpr size_t off_out = align128(off_y + (size_t)CH * RS * 4);  // Tout [CH][T]
    static constexpr size_t out_bytes = align128((size_t)CH * T * sizeof(Tout));
    static constexpr size_t off_par = off_out + out_bytes;               // bias[CH], D[CH]
    // mbarriers: full[2] (TMA bytes landed), then, for the producer-warp variant,
    // ready[2] (coefficients converted) and empty[2] (compute warps done with a stage)
    static constexpr size_t off_bar = align128(off_par + (size_t)2 * CH * 4);
    static constexpr size_t bytes = off_bar + 6 * 8;
    static_assert(NS % 4 == 0 || NS == 2, "states per lane: a multiple of 4, or 2");
    static_assert(T % 4 == 0 && kChunk % T == 0, "chunks of whole 4-step groups");
    static_assert(T * sizeof(Tin) % 16 == 0 && T * sizeof(Tout) % 16 == 0, "TMA rows");
    static_assert(T <= 256 && CH <= 256, "TMA box extents");
};

// Transpose-reduce of P partial sums over the P lanes of a channel: afterwards
// lane pp holds the complete sum of entry pp (P - 1 shuffles in total).
template <int P>
__device__ __forceinline__ float transpose_reduce(const float* v, int pp) {
    if constexpr (P == 1) {
        return v[0];
    } else if constexpr (P == 2) {
        const bool hi = pp & 1;
        float keep = hi ? v[1] : v[0];
        float send = hi ? v[0] : v[1];
        return keep + __shfl_xor_sync(0xffffffffu, send, 1);
    } else if constexpr (P == 4) {
        const bool hi2 = pp & 2;
        float w0 = (hi2 ? v[2] : v[0]) + __shfl_xor_sync(0xffffffffu, hi2 ? v[0] : v[2], 2);
        float w1 = (hi2 ? v[3] : v[1]) + __shfl_xor_sync(0xffffffffu, hi2 ? v[1] : v[3], 2);
        const bool hi1 = pp & 1;
        return (hi1 ? w1 : w0) + __shfl_xor_sync(0xffffffffu, hi1 ? w0 : w1, 1);
    } else {
        static_assert(P == 8, "P must be 1, 2, 4 or 8");
        const bool hi4 = pp & 4;
        float w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            w[i] = (hi4 ? v[i + 4] : v[i]) + __shfl_xor_sync(0xffffffffu, hi4 ? v[i] : v[i + 4], 4);
        const bool hi2 = pp & 2;
        const float x0 = (hi2 ? w[2] : w[0]) + __shfl_xor_sync(0xffffffffu, hi2 ? w[0] : w[2], 2);
        const float x1 = (hi2 ? w[3] : w[1]) + __shfl_xor_sync(0xffffffffu, hi2 ? w[1] : w[3], 2);
        const bool hi1 = pp & 1;
        return (hi1 ? x1 : x0) + __shfl_xor_sync(0xffffffffu, hi1 ? x0 : x1, 1);
    }
}

template <int NMAX, int P, int WARPS, int T_, typename Tin, typename Tout, int MODE, bool TMA,
          bool ZOH = false, int WS = 0, int CPL = 1>
__global__ void __launch_bounds__(WARPS * 32 + 32 * (WS == 0 ? 0 : (WS == 1 ? 1 : S6_WSP)))
scan_kernel(const KParams p, const __grid_constant__ TMaps tm) {
    // (modes without a CTA-wide barrier in the chunk loop: the producers do not join one)
    static_assert(!WS || (TMA && (MODE == kFull || MODE == kCheckpoint || MODE == kFullCkpt)),
                  "producer warps: TMA scans and checkpoint passes only");
    static_assert(!(WS && ZOH) || WS == 2, "exact ZOH with producers: form 2 only");
    constexpr int NPROD = WS == 0 ? 0 : (WS == 1 ? 1 : S6_WSP);  // producer warps
    static_assert(CPL == 1 || (MODE == kFull && !ZOH && !WS), "two channels per lane: plain scan");
    constexpr bool kOut = MODE == kFull || MODE == kFullCkpt || MODE == kFullAgg ||
                          MODE == kCorr;                              // writes y
    constexpr bool kCk = MODE == kCheckpoint || MODE == kFullCkpt;    // writes checkpoints
    constexpr bool kCorrM = MODE == kCorr;                            // input-free correction
    constexpr bool kSum = MODE == kAggregate || MODE == kFullAgg;     // segment summaries
    // time-paired exponent arguments (the FMA-pipe exponential and the exact ZOH weight
    // keep the state-paired form)
    constexpr bool kTPX = (MODE == kCorr) || (S6_TPX && !ZOH && S6_POLY == 0);
    static_assert(CPL == 1 || kTPX, "two channels per lane use the time-paired form");
    using Lo = Layout<NMAX, P, WARPS, T_, Tin, Tout, CPL, WS == 2 ? 2 : 1>;
    using V4 = vec4<Tin>;
    using VT = typename V4::type;
    constexpr int T = Lo::T, NS = Lo::NS, G = Lo::G, CW = Lo::CW, CH = Lo::CH, RS = Lo::RS;
    extern __shared__ __align__(128) unsigned char smem[];
    float* sDel = reinterpret_cast<float*>(smem + Lo::off_del);
    float* sDu = reinterpret_cast<float*>(smem + Lo::off_du);
    float* sY = reinterpret_cast<float*>(smem + Lo::off_y);
    float* sBias = reinterpret_cast<float*>(smem + Lo::off_par);
    float* sDsk = sBias + CH;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + Lo::off_bar);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t b = blockIdx.y;
    const int64_t d0 = (int64_t)blockIdx.x * CH;
    const int seg = (int)blockIdx.z + (kCorrM ? p.seg_first : 0);
    const int64_t t_begin = (int64_t)seg * p.seg_len;
    const int64_t t_end = min(p.L, t_begin + p.seg_len);
    const int64_t nchunks = t_end > t_begin ? (t_end - t_begin + T - 1) / T : 0;
    const bool has_z = kOut && p.z != nullptr;
    const bool out_tma = TMA && kOut && !kCorrM && p.y_tma;

    for (int c = tid; c < CH; c += Lo::THREADS) {
        const int64_t d = d0 + c;
        const bool ok = d < p.dim;
        sBias[c] = (ok && p.delta_bias) ? p.delta_bias[d] : 0.f;
        sDsk[c] = (ok && p.D) ? p.D[d] : 0.f;
    }
    if (TMA && tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        if (WS) {
            mbar_init(&bar[2], NPROD);
            mbar_init(&bar[3], NPROD);
            mbar_init(&bar[4], WARPS);
            mbar_init(&bar[5], WARPS);
        }
        fence_barrier_init();
    }

    // This lane's channels (CPL of them, G apart) and states (NS of each).
    const int pp = lane % P;
    int cwk[CPL];
    int64_t dchk[CPL];
#pragma unroll
    for (int k = 0; k < CPL; ++k) {
        cwk[k] = warp * CW + k * G + lane / P;
        dchk[k] = d0 + cwk[k];
    }
    const int cw = cwk[0];
    const int64_t dch = dchk[0];
    f2 a2p[CPL][NS / 2], hp[CPL][NS / 2];
    f2 a2d[kTPX ? CPL : 1][kTPX ? NS : 1];  // (a_n, a_n): one state's factor for two steps
    f2 inv_ap[ZOH ? NS / 2 : 1];  // 1 / A per state, for the exact ZOH input weight
#pragma unroll
    for (int k = 0; k < CPL; ++k) {
#pragma unroll
        for (int j = 0; j < NS; j += 2) {
            float a[2], h[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int nn = pp * NS + j + q;
                const bool ok = dchk[k] < p.dim && nn < p.N;
                a[q] = ok ? p.A[dchk[k] * p.N + nn] * kLog2e : 0.f;  // padded states: Abar = 1, b = 0
                // initial state: the segment's start (split sequences) or the caller's h0
                h[q] = ((kOut || MODE == kCheckpoint) && MODE != kFullAgg && p.seg_h != nullptr && ok)
                           ? p.seg_h[(((int64_t)seg * p.batch + b) * p.dim + dchk[k]) * p.N + nn]
                           : 0.f;
            }
            a2p[k][j / 2] = pack2(a[0], a[1]);
            hp[k][j / 2] = pack2(h[0], h[1]);
            if constexpr (kTPX) {
                a2d[k][j] = pack2(a[0], a[0]);
                a2d[k][j + 1] = pack2(a[1], a[1]);
            }
            if constexpr (ZOH) {
                // 1 / A (infinite for A = 0; the weight then takes its series branch)
                const float ia0 = kLog2e / a[0], ia1 = kLog2e / a[1];
                inv_ap[j / 2] = pack2(ia0, ia1);
            }
        }
    }
    // checkpoint modes: this lane's states of group 0 and the distance between groups
    float* ck_lane = nullptr;
    int64_t ck_gstride = 0;
    if constexpr (MODE == kCheckpoint || MODE == kFullCkpt) {
        const int64_t blocks = (p.L + kCkptSteps - 1) / kCkptSteps;
        ck_lane = p.ckpt + ckpt_index(b, dch < p.dim ? dch : 0, 0, p.dim, blocks, p.N, p.ck_tiled) + pp * NS;
        ck_gstride = (p.ck_tiled ? kCkptTile : 1) * (int64_t)p.N;
    }
    float dsum = 0.f;
    // Correction pass: the state it carries decays monotonically when every A of the lane
    // is <= 0 and Delta >= 0 (softplus); then it may stop once every state is below
    // 2^-24 of the largest it started from.
    bool decay_ok = kCorrM && p.softplus != 0;
    float decay_thr = 0.f;
    if constexpr (kCorrM) {
#pragma unroll
        for (int k = 0; k < CPL; ++k)
#pragma unroll
            for (int j = 0; j < NS / 2; ++j) {
                float a0, a1, h0v, h1v;
                unpack2(a2p[k][j], a0, a1);
                unpack2(hp[k][j], h0v, h1v);
                decay_ok = decay_ok && a0 <= 0.f && a1 <= 0.f;
                decay_thr = fmaxf(decay_thr, fmaxf(fabsf(h0v), fabsf(h1v)));
            }
        decay_thr *= 5.9604645e-8f;  // 2^-24
    }
    __syncthreads();

    // Stage chunk k of this CTA's segment into stage buffer k & 1.
    auto stage_ptr = [&](int64_t k) -> Tin* {
        return reinterpret_cast<Tin*>(smem + (k & 1) * Lo::stage_bytes);
    };
    auto issue_chunk = [&](int64_t k) {  // TMA: called by one thread
        unsigned char* st = smem + (k & 1) * Lo::stage_bytes;
        const int tt = (int)(t_begin + k * T);
        // the correction has no input: neither u nor B is needed; the passes without
        // output (checkpoints, segment summaries) need no C
        const uint32_t bytes = kCorrM ? (uint32_t)((has_z ? 2 : 1) * Lo::rows_bytes + Lo::coef_bytes)
                                      : (uint32_t)((has_z ? 3 : 2) * Lo::rows_bytes +
                                                   (kOut ? 2 : 1) * Lo::coef_bytes);
        uint64_t* bk = &bar[k & 1];
        mbar_arrive_expect_tx(bk, bytes);
        if (!kCorrM) tma_load_3d(st, &tm.u, tt, (int)d0, (int)b, bk);
        tma_load_3d(st + Lo::off_dr, &tm.dr, tt, (int)d0, (int)b, bk);
        if (has_z) tma_load_3d(st + Lo::off_z, &tm.z, tt, (int)d0, (int)b, bk);
        if (!kCorrM) tma_load_3d(st + Lo::off_B, &tm.B, tt, 0, (int)b, bk);
        if (kOut) tma_load_3d(st + Lo::off_C, &tm.C, tt, 0, (int)b, bk);
    };
    auto load_chunk_elementwise = [&](int64_t k) {  // rows not 16-byte multiples
        unsigned char* st = smem + (k & 1) * Lo::stage_bytes;
        const int64_t t0 = t_begin + k * T;
        const Tin* gsrc[5] = {static_cast<const Tin*>(p.u), static_cast<const Tin*>(p.delta),
                              static_cast<const Tin*>(p.z), static_cast<const Tin*>(p.B),
                              static_cast<const Tin*>(p.C)};
        const size_t off[5] = {0, Lo::off_dr, Lo::off_z, Lo::off_B, Lo::off_C};
        const int nx = has_z ? 3 : 2;
        for (int i = tid; i < (nx * CH + 2 * NMAX) * T; i += Lo::THREADS) {
            const int r = i / T, j = i % T;
            const int64_t t = t0 + j;
            int which, row;
            int64_t grow;
            bool ok;
            if (r < nx * CH) {
                which = r / CH, row = r % CH;
                ok = d0 + row < p.dim && t < p.L;
                grow = b * p.dim + d0 + row;
            } else {
                which = 3 + (r - nx * CH) / NMAX, row = (r - nx * CH) % NMAX;
                ok = row < p.N && t < p.L;
                grow = b * p.N + row;
            }
            reinterpret_cast<Tin*>(st + off[which])[row * T + j] =
                ok ? gsrc[which][grow * p.L + t] : Tin(0.f);
        }
    };

    // B, C of chunk k into its coefficient buffer (work items first, first + stride, ...).
    auto convert_chunk = [&](int64_t k, int first, int stride) {
        const unsigned char* stb = reinterpret_cast<const unsigned char*>(stage_ptr(k));
        const Tin* rB = reinterpret_cast<const Tin*>(stb + Lo::off_B);
        const Tin* rC = reinterpret_cast<const Tin*>(stb + Lo::off_C);
        float* sBt = reinterpret_cast<float*>(smem + Lo::off_coef + (k & 1) * Lo::coef_bytes_all);
        float* sCt = sBt + T * NMAX;
        // B, C of the chunk, time-major: every lane then reads the coefficients of its four
        // states for step t with one 16-byte load (bf16: B[4] and C[4] as pairs; fp32: a
        // 16-byte vector from each of two tiles, transposed through 4x4 register blocks).
        if constexpr (Lo::kBC == 1 || (Lo::kBC == 2 && kOut)) {
            // bf16 pairs.  Format 1: per (step, 4-state group) [B0|B1][B2|B3][C0|C1][C2|C3];
            // format 2: the C half only, [C0|C1][C2|C3] per (step, group), after the B tile.
            // Work item: (4-state group, step pair, B or C) -> two 8-byte half-groups.
            constexpr int kWhich = Lo::kBC == 1 ? 2 : 1;
            for (int i = first; i < (NMAX / 4) * (T / 2) * kWhich; i += stride) {
                const int which = kWhich == 2 ? (i & 1) : 1;
                const int i2 = kWhich == 2 ? (i >> 1) : i;
                const int n4 = i2 % (NMAX / 4), t2 = i2 / (NMAX / 4);
                const Tin* src = (which ? rC : rB) + (4 * n4) * T + 2 * t2;
                uint32_t w[4];
#pragma unroll
                for (int r = 0; r < 4; ++r) w[r] = *reinterpret_cast<const uint32_t*>(src + r * T);
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    // step 2*t2+q sits in half q of each row's word; pair rows (0,1), (2,3)
                    const unsigned sel = q ? 0x7632u : 0x5410u;
                    uint2 g;
                    g.x = __byte_perm(w[0], w[1], sel);
                    g.y = __byte_perm(w[2], w[3], sel);
                    const int grp = (2 * t2 + q) * (NMAX / 4) + n4;
                    if (Lo::kBC == 1)
                        reinterpret_cast<uint2*>(sBt)[grp * 2 + which] = g;
                    else
                        reinterpret_cast<uint2*>(sCt)[grp] = g;
                }
            }
        }
        if constexpr (Lo::kBC == 0 || Lo::kBC == 2) {
            // fp32 tiles [T][NMAX], transposed through 4x4 register blocks (C only for the
            // passes with output)
            constexpr int kTiles = Lo::kBC == 0 && kOut ? 2 : 1;
            for (int i = first; i < (NMAX / 4) * (T / 4) * kTiles; i += stride) {
                const int which = kTiles == 2 ? (i & 1) : 0;
                const int i2 = kTiles == 2 ? (i >> 1) : i;
                const int n4 = i2 % (NMAX / 4), t4 = i2 / (NMAX / 4);
                const Tin* src = which ? rC : rB;
                float* dst = which ? sCt : sBt;
                float v[4][4];
#pragma unroll
                for (int r = 0; r < 4; ++r)
                    V4::to_f(*reinterpret_cast<const VT*>(src + (4 * n4 + r) * T + 4 * t4), v[r]);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<float4*>(dst + (4 * t4 + q) * NMAX + 4 * n4) =
                        make_float4(v[0][q], v[1][q], v[2][q], v[3][q]);
            }
        }
    };

    // Phase A on chunk k: work items i0, i0 + istride, ... below nitems, item i being channel
    // cfirst + i / (T/4) at steps 4 (i % (T/4)) .. +3: Delta = softplus(delta + bias) and
    // Delta u (u itself for the exact ZOH weight) into dl, du.  Steps past the end of the
    // segment get Delta = 0 (Abar = 1, no input): the state passes.
    auto phase_a = [&](int64_t k, int cfirst, int nitems, int i0, int istride, float* dl, float* du) {
        const unsigned char* stb = smem + (k & 1) * Lo::stage_bytes;
        const Tin* rU = reinterpret_cast<const Tin*>(stb);
        const Tin* rDr = reinterpret_cast<const Tin*>(stb + Lo::off_dr);
        const int valid = (int)min((int64_t)T, t_end - (t_begin + k * T));
        for (int i = i0; i < nitems; i += istride) {
            const int c = cfirst + i / (T / 4), tb = 4 * (i % (T / 4));
            float x[4], uu[4] = {0.f, 0.f, 0.f, 0.f};
            V4::to_f(*reinterpret_cast<const VT*>(rDr + c * T + tb), x);
            if (!kCorrM) V4::to_f(*reinterpret_cast<const VT*>(rU + c * T + tb), uu);
            const float bias = sBias[c];
            float dt[4], xb[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) xb[q] = x[q] + bias;
            if (p.softplus) {
                softplus4(xb, dt);
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q) dt[q] = xb[q];
            }
            if (valid < T) {
#pragma unroll
                for (int q = 0; q < 4; ++q) dt[q] = tb + q < valid ? dt[q] : 0.f;
            }
            *reinterpret_cast<float4*>(dl + c * RS + tb) = make_float4(dt[0], dt[1], dt[2], dt[3]);
            if constexpr (kCorrM) {
                // no input term
            } else if constexpr (ZOH) {  // the exact ZOH weight needs u itself
                *reinterpret_cast<float4*>(du + c * RS + tb) = make_float4(uu[0], uu[1], uu[2], uu[3]);
            } else {
                const float q0 = dt[0] * uu[0], q1 = dt[1] * uu[1], q2 = dt[2] * uu[2],
                            q3 = dt[3] * uu[3];
                *reinterpret_cast<float4*>(du + c * RS + tb) = make_float4(q0, q1, q2, q3);
            }
        }
        __syncwarp();
    };

    // Producer warp (variant WS): stages every chunk with TMA and converts its
    // coefficients; the compute warps wait only for a chunk to be ready and release its
    // stage when done, so they never wait for one another.
    if constexpr (WS) {
        if (warp >= WARPS) {
            const int pw = warp - WARPS;  // producer warp index
            bool pok = true;
            int64_t issued = -1, landed = -1;
            for (int64_t k = 0; k < nchunks; ++k) {
                const int s = (int)(k & 1);
                if (k >= 2) {  // the compute warps are done with chunk k - 2 in this stage
                    pok = __all_sync(0xffffffffu, mbar_wait_bounded(
                        &bar[4 + s], (uint32_t)(((k >> 1) & 1) ^ 1), kWaitLimitCycles));
                    if (!pok) break;
                }
                if (pw == 0 && lane == 0) {
                    fence_proxy_async();  // the stage was last read through the generic proxy
                    issue_chunk(k);
                }
                issued = k;
                pok = __all_sync(0xffffffffu, mbar_wait_bounded(&bar[s], (uint32_t)((k >> 1) & 1),
                                                                kWaitLimitCycles));
                if (!pok) break;
                landed = k;
                convert_chunk(k, pw * 32 + lane, 32 * NPROD);
                if constexpr (WS == 2)
                    phase_a(k, 0, CH * (T / 4), pw * 32 + lane, 32 * NPROD, sDel + s * Lo::dq_stride,
                            sDu + s * Lo::dq_stride);
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar[2 + s]);
            }
            if (!pok) {
                if (lane == 0) atomicOr(&g_device_error, 1u);
                if (pw == 0 && lane == 0 && issued > landed)  // let the copy in flight land first
                    mbar_wait_bounded(&bar[issued & 1], (uint32_t)((issued >> 1) & 1),
                                      kWaitLimitCycles);
            }
            return;
        }
    }

    if constexpr (TMA && !WS) {
        if (tid == 0 && nchunks > 0) issue_chunk(0);
    }
    bool aborted = false;
    bool drained = false;      // the correction stopped early (its remainder is negligible)
    int64_t abort_chunk = -1;  // the chunk whose copy may still be in flight when stopping
    for (int64_t k = 0; k < nchunks; ++k) {
        bool ok = true;
        if constexpr (WS) {
            ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bar[2 + (k & 1)], (uint32_t)((k >> 1) & 1),
                                                           kWaitLimitCycles));
            if (!ok) {
                if (lane == 0) atomicOr(&g_device_error, 1u);
                aborted = true;
                break;
            }
        } else if constexpr (TMA) {
            ok = mbar_wait_bounded(&bar[k & 1], (uint32_t)((k >> 1) & 1), kWaitLimitCycles);
        } else {
            load_chunk_elementwise(k);
            __syncthreads();
        }

        const Tin* st = stage_ptr(k);
        const unsigned char* stb = reinterpret_cast<const unsigned char*>(st);
        const Tin* rU = st;
        const Tin* rDr = reinterpret_cast<const Tin*>(stb + Lo::off_dr);
        const Tin* rZ = reinterpret_cast<const Tin*>(stb + Lo::off_z);
        const int64_t t0 = t_begin + k * T;
        const int valid = (int)min((int64_t)T, t_end - t0);
        float* sBt = reinterpret_cast<float*>(smem + Lo::off_coef + (k & 1) * Lo::coef_bytes_all);
        float* sCt = sBt + T * NMAX;  // formats 0 and 2: what follows the fp32 B tile

        if constexpr (!WS) {
            convert_chunk(k, tid, Lo::THREADS);
            // The one CTA-wide barrier of a chunk: coefficients visible to every warp, and
            // every warp done with chunk k-1, so its stage can take chunk k+1.
            if (__syncthreads_or(!ok)) {  // every thread agrees to stop if any wait gave up
                if (tid == 0) atomicOr(&g_device_error, 1u);
                aborted = true;
                abort_chunk = k;  // chunk k was issued; chunk k + 1 was not
                break;
            }
            if constexpr (TMA) {
                if (tid == 0 && k + 1 < nchunks) {
                    fence_proxy_async();  // stage (k+1)&1 was last read through the generic proxy
                    issue_chunk(k + 1);
                }
            }
        }

        // Phase A for this warp's channels (with S6_WS=2 the producer warps do it).
        float* sDelK = sDel + (WS == 2 ? (k & 1) * Lo::dq_stride : 0);
        float* sDuK = sDu + (WS == 2 ? (k & 1) * Lo::dq_stride : 0);
        if constexpr (WS != 2) phase_a(k, warp * CW, CW * (T / 4), lane, 32, sDelK, sDuK);

        // checkpoint modes: the state entering every 4-step group of the sequence, at
        // ckpt_index(b, d, group) -- what the backward's reverse sweep starts each group
        // from, so it recomputes no other state
        auto write_ckpt = [&](int t) {
            if (dch >= p.dim || t0 + t >= p.L) return;
            float* ck = ck_lane + ((t0 + t) / kCkptSteps) * ck_gstride;
            if (NS % 4 == 0 && p.N == NMAX && (reinterpret_cast<uintptr_t>(ck) & 15) == 0) {
#pragma unroll
                for (int j = 0; j < NS / 2; j += 2) {
                    float h0, h1, h2, h3;
                    unpack2(hp[0][j], h0, h1);
                    unpack2(hp[0][j + 1], h2, h3);
                    *reinterpret_cast<float4*>(ck + 2 * j) = make_float4(h0, h1, h2, h3);
                }
                return;
            }
#pragma unroll
            for (int j = 0; j < NS / 2; ++j) {
                float h0, h1;
                unpack2(hp[0][j], h0, h1);
                if (pp * NS + 2 * j < p.N) ck[2 * j] = h0;
                if (pp * NS + 2 * j + 1 < p.N) ck[2 * j + 1] = h1;
            }
        };

        // Phase B: the recurrence, four steps per iteration, states in packed pairs.
        f2 ee_next[4][NS / 2];  // the lookahead's Abar of the next group (S6_PIPE)
        float yp8[CPL][8];      // P = 8: partial outputs of two groups for one transpose-reduce
#pragma unroll
        for (int t = 0; t < T; t += 4) {
            if (kCk) write_ckpt(t);
            float4 d4[CPL], q4[CPL];
#pragma unroll
            for (int k = 0; k < CPL; ++k) {
                d4[k] = *reinterpret_cast<const float4*>(sDelK + cwk[k] * RS + t);
                if (!kCorrM) q4[k] = *reinterpret_cast<const float4*>(sDuK + cwk[k] * RS + t);
            }
            float yp[CPL][4];
            // this lane's B and C of step t + kk, as fp32 pairs (states 2j, 2j + 1)
            auto coefs = [&](int kk, f2 (&bq)[NS / 2], f2 (&cq)[NS / 2]) {
                if constexpr (NS == 2) {  // one state pair per lane: half of a 4-state group
                    const int q = pp >> 1, hw = pp & 1;
                    if constexpr (Lo::kBC == 1) {
                        const uint32_t* g = reinterpret_cast<const uint32_t*>(sBt) +
                                            ((t + kk) * (NMAX / 4) + q) * 4;
                        bq[0] = bf16pair(g[hw]);
                        cq[0] = bf16pair(g[2 + hw]);
                    } else {
                        bq[0] = f2{*reinterpret_cast<const unsigned long long*>(sBt + (t + kk) * NMAX + 2 * pp)};
                        if constexpr (Lo::kBC == 2)
                            cq[0] = bf16pair(reinterpret_cast<const uint32_t*>(sCt)[((t + kk) * (NMAX / 4) + q) * 2 + hw]);
                        else
                            cq[0] = f2{*reinterpret_cast<const unsigned long long*>(sCt + (t + kk) * NMAX + 2 * pp)};
                    }
                    return;
                }
#pragma unroll
                for (int j = 0; j < NS / 4; ++j) {
                    if constexpr (Lo::kBC == 1) {
                        const uint4 g = reinterpret_cast<const uint4*>(sBt)[(t + kk) * (NMAX / 4) +
                                                                            pp * (NS / 4) + j];
                        bq[2 * j] = bf16pair(g.x), bq[2 * j + 1] = bf16pair(g.y);
                        cq[2 * j] = bf16pair(g.z), cq[2 * j + 1] = bf16pair(g.w);
                    } else if constexpr (Lo::kBC == 2) {
                        const ulonglong2 bb = reinterpret_cast<const ulonglong2*>(
                            sBt + (t + kk) * NMAX + pp * NS)[j];
                        const uint2 g = reinterpret_cast<const uint2*>(sCt)[(t + kk) * (NMAX / 4) +
                                                                          pp * (NS / 4) + j];
                        bq[2 * j] = f2{bb.x}, bq[2 * j + 1] = f2{bb.y};
                        cq[2 * j] = bf16pair(g.x), cq[2 * j + 1] = bf16pair(g.y);
                    } else {
                        const ulonglong2 bb = reinterpret_cast<const ulonglong2*>(
                            sBt + (t + kk) * NMAX + pp * NS)[j];
                        const ulonglong2 cc = reinterpret_cast<const ulonglong2*>(
                            sCt + (t + kk) * NMAX + pp * NS)[j];
                        bq[2 * j] = f2{bb.x}, bq[2 * j + 1] = f2{bb.y};
                        cq[2 * j] = f2{cc.x}, cq[2 * j + 1] = f2{cc.y};
                    }
                }
            };
            if constexpr (kTPX) {
                // Abar of the four steps first (their SFU latency overlaps): per state, the
                // arguments of steps (t, t+1) and (t+2, t+3) as two packed products.
                float ee[CPL][4][NS];
#pragma unroll
                for (int k = 0; k < CPL; ++k)
#pragma unroll
                    for (int j = 0; j < NS; ++j) {
                        float x0, x1, x2, x3;
                        unpack2(mul2(pack2(d4[k].x, d4[k].y), a2d[k][j]), x0, x1);
                        unpack2(mul2(pack2(d4[k].z, d4[k].w), a2d[k][j]), x2, x3);
                        ee[k][0][j] = ex2(x0);
                        ee[k][1][j] = ex2(x1);
                        ee[k][2][j] = ex2(x2);
                        ee[k][3][j] = ex2(x3);
                    }
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    f2 bq[NS / 2], cq[NS / 2];
                    coefs(kk, bq, cq);
#pragma unroll
                    for (int k = 0; k < CPL; ++k) {
                        f2 acc = pack2(0.f, 0.f);
#pragma unroll
                        for (int j = 0; j < NS / 2; ++j) {
                            const f2 e = pack2(ee[k][kk][2 * j], ee[k][kk][2 * j + 1]);
                            if constexpr (kCorrM) {
                                hp[k][j] = mul2(e, hp[k][j]);  // no input: h = Abar h
                            } else {
                                const float qa[4] = {q4[k].x, q4[k].y, q4[k].z, q4[k].w};
                                const f2 qq = pack2(qa[kk], qa[kk]);
                                hp[k][j] = fma2(e, hp[k][j], mul2(qq, bq[j]));
                            }
                            acc = fma2(cq[j], hp[k][j], acc);
                        }
                        float lo, hi;
                        unpack2(acc, lo, hi);
                        yp[k][kk] = lo + hi;
                    }
                }
            } else {
                const float4 dv = d4[0], qv = q4[0];
                const f2 dd4[4] = {pack2(dv.x, dv.x), pack2(dv.y, dv.y), pack2(dv.z, dv.z),
                                   pack2(dv.w, dv.w)};
                const f2 qq4[4] = {pack2(qv.x, qv.x), pack2(qv.y, qv.y), pack2(qv.z, qv.z),
                                   pack2(qv.w, qv.w)};
                constexpr bool kPipe = S6_PIPE && S6_PREEXP && !ZOH && S6_POLY == 0;
                // all Abar factors of the four steps first, so their SFU latency overlaps
                // (with the lookahead, they were formed during the previous group)
                f2 ee[4][NS / 2];
                if constexpr (kPipe) {
                    if (t == 0) {
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
#pragma unroll
                            for (int j = 0; j < NS / 2; ++j)
                                ee_next[kk][j] = ex2x2(mul2(dd4[kk], a2p[0][j]));
                    }
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
                        for (int j = 0; j < NS / 2; ++j) ee[kk][j] = ee_next[kk][j];
                } else if constexpr (S6_PREEXP && !ZOH && S6_POLY == 0) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
                        for (int j = 0; j < NS / 2; ++j) ee[kk][j] = ex2x2(mul2(dd4[kk], a2p[0][j]));
                }
                // the next group's step sizes, for the lookahead
                f2 ddn[4];
                if constexpr (kPipe) {
                    if (t + 4 < T) {
                        const float4 dn = *reinterpret_cast<const float4*>(sDelK + cwk[0] * RS + t + 4);
                        ddn[0] = pack2(dn.x, dn.x), ddn[1] = pack2(dn.y, dn.y);
                        ddn[2] = pack2(dn.z, dn.z), ddn[3] = pack2(dn.w, dn.w);
                    }
                }
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    if constexpr (kPipe) {
                        if (t + 4 < T) {
#pragma unroll
                            for (int j = 0; j < NS / 2; ++j)
                                ee_next[kk][j] = ex2x2(mul2(ddn[kk], a2p[0][j]));
                        }
                    }
                    const f2 dd = dd4[kk];
                    // ZOH: qq4 holds (u, u); Delta u is formed here
                    const f2 uu = qq4[kk];
                    const f2 qq = ZOH ? mul2(dd, uu) : qq4[kk];
                    f2 bq[NS / 2], cq[NS / 2];
                    coefs(kk, bq, cq);
                    f2 acc = pack2(0.f, 0.f);
#pragma unroll
                    for (int j = 0; j < NS / 2; ++j) {
                        if constexpr (ZOH) {
                            const f2 x0 = mul2(dd, a2p[0][j]);
                            const f2 e0 = ex2x2(x0);
                            const f2 m0 = zoh_weight_u2(x0, e0, inv_ap[j], uu, qq);
                            hp[0][j] = fma2(e0, hp[0][j], mul2(m0, bq[j]));
                        } else if constexpr (S6_PREEXP && S6_POLY == 0) {
                            hp[0][j] = fma2(ee[kk][j], hp[0][j], mul2(qq, bq[j]));
                        } else {
                            const bool on_fma = (j & 1) && (S6_POLY == 2 || (S6_POLY == 1 && (kk & 1)));
                            const f2 e0 = on_fma ? exp2_fma2(mul2(dd, a2p[0][j]))
                                                 : ex2x2(mul2(dd, a2p[0][j]));
                            hp[0][j] = fma2(e0, hp[0][j], mul2(qq, bq[j]));
                        }
                        acc = fma2(cq[j], hp[0][j], acc);
                    }
                    float lo, hi;
                    unpack2(acc, lo, hi);
                    yp[0][kk] = lo + hi;
                }
            }
            if constexpr (kSum) dsum += (d4[0].x + d4[0].y) + (d4[0].z + d4[0].w);
            if constexpr (kOut) {
#pragma unroll
                for (int k = 0; k < CPL; ++k) {
                    if constexpr (P == 1) {
                        *reinterpret_cast<float4*>(sY + cwk[k] * RS + t) =
                            make_float4(yp[k][0], yp[k][1], yp[k][2], yp[k][3]);
                    } else if constexpr (P == 8) {
                        // eight steps per transpose-reduce: this group's and the previous one's
#pragma unroll
                        for (int q = 0; q < 4; ++q) yp8[k][(t & 4) + q] = yp[k][q];
                        if (t & 4) sY[cwk[k] * RS + (t - 4) + pp] = transpose_reduce<P>(yp8[k], pp);
                    } else {
#pragma unroll
                        for (int g = 0; g < 4; g += P)
                            sY[cwk[k] * RS + t + g + pp] = transpose_reduce<P>(yp[k] + g, pp);
                    }
                }
            }
        }

        if (kOut) {
            // Phase C: skip term, gate; four steps per lane into this warp's rows of the
            // output tile, which its lane 0 then stores with TMA (or straight to global
            // memory when rows cannot be described to TMA).  The warp's previous store
            // has long finished reading the tile; lane 0 confirms before it is rewritten.
            if (out_tma && lane == 0) tma_store_wait_read<0>();
            __syncwarp();
            Tout* sOut = reinterpret_cast<Tout*>(smem + Lo::off_out);
            Tout* gy = static_cast<Tout*>(p.y);
            for (int i = lane; i < CW * (T / 4); i += 32) {
                const int c = warp * CW + i / (T / 4), tb = 4 * (i % (T / 4));
                const float4 y4 = *reinterpret_cast<const float4*>(sY + c * RS + tb);
                float uu[4] = {0.f, 0.f, 0.f, 0.f}, zz[4];
                if (!kCorrM) V4::to_f(*reinterpret_cast<const VT*>(rU + c * T + tb), uu);
                if (has_z) V4::to_f(*reinterpret_cast<const VT*>(rZ + c * T + tb), zz);
                const float yv[4] = {y4.x, y4.y, y4.z, y4.w};
                const float dsk = sDsk[c];
                float o[4], sz[4];
                if (has_z) {
                    if constexpr (S6_SILU4) {
                        silu4(zz, sz);
                    } else {
#pragma unroll
                        for (int q = 0; q < 4; ++q) sz[q] = silu(zz[q]);
                    }
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    o[q] = kCorrM ? yv[q] : fmaf(dsk, uu[q], yv[q]);  // D u is in y already
                    if (has_z) o[q] *= sz[q];
                }
                if (out_tma) {
                    store4(sOut + c * T + tb, o);
                } else {
                    const int64_t d = d0 + c;
                    if (d >= p.dim || tb >= valid) continue;
                    Tout* dst = gy + (b * p.dim + d) * p.L + t0 + tb;
                    if constexpr (kCorrM) {  // the correction adds to the first pass's output
                        if (p.y_vec && tb + 4 <= valid) {
                            float yo[4];
                            vec4<Tout>::to_f(*reinterpret_cast<const typename vec4<Tout>::type*>(dst), yo);
#pragma unroll
                            for (int q = 0; q < 4; ++q) o[q] += yo[q];
                        } else {
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                if (tb + q < valid) o[q] += io<Tout>::to_f(dst[q]);
                        }
                    }
                    if (p.y_vec && tb + 4 <= valid) {
                        store4(dst, o);
                    } else {
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            if (tb + q < valid) dst[q] = io<Tout>::from_f(o[q]);
                    }
                }
            }
            if (out_tma) {
                fence_proxy_async();  // this lane's tile writes, before the async-proxy read
                __syncwarp();
                if (lane == 0 && d0 + warp * CW < p.dim) {  // rows past dim are clipped
                    tma_store_3d(&tm.y, sOut + warp * CW * T, (int)t0, (int)(d0 + warp * CW), (int)b);
                    tma_store_commit();
                }
            }
        }
        if constexpr (WS) {  // this warp is done with the chunk's stage and coefficients
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[4 + (k & 1)]);
        }
        if constexpr (kCorrM) {
            // The carried start state only decays (Abar in (0, 1] when A <= 0 and Delta >= 0):
            // once every state of every channel of the CTA is below 2^-24 of where it
            // started, the rest of the correction is below fp32 resolution and the CTA stops.
            bool small = decay_ok;
#pragma unroll
            for (int kc = 0; kc < CPL; ++kc)
#pragma unroll
                for (int j = 0; j < NS / 2; ++j) {
                    float h0v, h1v;
                    unpack2(hp[kc][j], h0v, h1v);
                    small = small && fabsf(h0v) <= decay_thr && fabsf(h1v) <= decay_thr;
                }
            if (__syncthreads_and(small)) {
                if (TMA && k + 1 < nchunks) abort_chunk = k + 1;  // issued, still in flight
                drained = true;
                break;
            }
        }
    }

    if constexpr (TMA && !WS) {
        if (tid == 0) {
            // let the copy still in flight (the chunk the loop stopped at) land before the
            // CTA exits; earlier chunks completed their phases already
            if ((aborted || drained) && abort_chunk >= 0)
                mbar_wait_bounded(&bar[abort_chunk & 1], (uint32_t)((abort_chunk >> 1) & 1),
                                  kWaitLimitCycles);
        }
    }
    if (out_tma && lane == 0) tma_store_wait_all();
    if (aborted) return;

#pragma unroll
    for (int k = 0; k < CPL; ++k) {
        if (dchk[k] >= p.dim) continue;
        float h[NS];
#pragma unroll
        for (int j = 0; j < NS / 2; ++j) unpack2(hp[k][j], h[2 * j], h[2 * j + 1]);
        if constexpr (MODE == kFull || MODE == kFullCkpt) {
            if (p.last_state && seg == (int)gridDim.z - 1) {
#pragma unroll
                for (int n = 0; n < NS; ++n) {
                    const int nn = pp * NS + n;
                    if (nn < p.N) p.last_state[(b * p.dim + dchk[k]) * p.N + nn] = h[n];
                }
            }
        } else if constexpr (kSum) {
            const int64_t row = ((int64_t)seg * p.batch + b) * p.dim + dch;
#pragma unroll
            for (int n = 0; n < NS; ++n) {
                const int nn = pp * NS + n;
                if (nn < p.N) p.seg_h[row * p.N + nn] = h[n];
            }
            if (pp == 0) p.seg_sum[row] = dsum;
        }
    }
}

// Failure-detection probe: one bounded wait on an mbarrier that nothing ever completes.
// It gives up after limit_cycles SM clocks and records that in the device error word, as
// any bounded wait of the scan does -- so the host's detection path can be exercised
// without a fault.
__global__ void wait_timeout_probe_kernel(long long limit_cycles) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
        if (!mbar_wait_bounded(&bar, 0, limit_cycles)) atomicOr(&g_device_error, 1u);
    }
}

// Fold the segments left to right.  Thread per (batch, channel, state):
// on entry seg_h[s] holds segment s's end state from h = 0 (s < nseg - 1) and
// seg_sum[s] its summed step; on exit seg_h[s] holds segment s's true start state
// (segment 0 starts from h0, or from zero when h0 is null).
__global__ void carry_kernel(float* seg_h, const float* seg_sum, const float* A, int64_t batch,
                             int64_t dim, int N, int nseg, const float* h0) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t lanes = batch * dim * N;
    if (i >= lanes) return;
    const int n = (int)(i % N);
    const int64_t bd = i / N;
    const int64_t d = bd % dim;
    const float a2 = A[d * N + n] * kLog2e;
    float H = h0 ? h0[bd * N + n] : 0.f;
    for (int s = 0; s < nseg - 1; ++s) {
        const int64_t row = (int64_t)s * batch * dim + bd;
        const float hend = seg_h[row * N + n];
        seg_h[row * N + n] = H;
        H = fmaf(ex2(a2 * seg_sum[row]), H, hend);  // (prod Abar, h_end) (+) (., H)
    }
    seg_h[((int64_t)(nseg - 1) * batch * dim + bd) * N + n] = H;
}

// The one-pass split's fold.  Thread per (batch, channel, state): on entry seg_h[s]
// holds the end state of segment s scanned from h = 0 and seg_sum[s] its summed step,
// for every segment; on exit seg_h[s] holds segment s's true start state (segment 0
// from h0, or zero), and last_state (when not null) the state after the whole sequence.
__global__ void carry_all_kernel(float* seg_h, const float* seg_sum, const float* A, int64_t batch,
                                 int64_t dim, int N, int nseg, const float* h0, float* last_state) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t lanes = batch * dim * N;
    if (i >= lanes) return;
    const int n = (int)(i % N);
    const int64_t bd = i / N;
    const int64_t d = bd % dim;
    const float a2 = A[d * N + n] * kLog2e;
    float H = h0 ? h0[bd * N + n] : 0.f;
    for (int s = 0; s < nseg; ++s) {
        const int64_t row = (int64_t)s * batch * dim + bd;
        const float hend = seg_h[row * N + n];
        seg_h[row * N + n] = H;
        H = fmaf(ex2(a2 * seg_sum[row]), H, hend);  // (prod Abar, h_end) (+) (., H)
    }
    if (last_state) last_state[bd * N + n] = H;
}

// Inclusive fold of `count` segment summaries (h_end from zero, summed step) applied to h0:
// h_out = the state after all of them, dsum_out = their total step.  Thread per
// (batch, channel, state); the pair (exp(A * dsum), h_end) is the associative combine's
// element, so folding consecutive summaries is applying them in order.
__global__ void fold_kernel(const float* hend, const float* dsum, const float* A, const float* h0,
                            int64_t count, int64_t batch, int64_t dim, int N, float* h_out,
                            float* dsum_out) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t lanes = batch * dim * N;
    if (i >= lanes) return;
    const int n = (int)(i % N);
    const int64_t bd = i / N;
    const int64_t d = bd % dim;
    const float a2 = A[d * N + n] * kLog2e;
    float H = h0 ? h0[bd * N + n] : 0.f, S = 0.f;
    for (int64_t s = 0; s < count; ++s) {
        const int64_t row = s * batch * dim + bd;
        H = fmaf(ex2(a2 * dsum[row]), H, hend[row * N + n]);
        S += dsum[row];
    }
    h_out[bd * N + n] = H;
    if (dsum_out && n == 0) dsum_out[bd] = S;
}

// ---- host side ---------------------------------------------------------------------------

using EncodeFn = PFN_cuTensorMapEncodeTiled_v12000;

EncodeFn tensor_map_encoder() {
    static EncodeFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeFn>(ptr);
    });
    return fn;
}

// Describe a row-major (outer, mid, inner) tensor with a (box_inner, box_mid, 1) box.
template <typename T>
bool encode_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t mid, uint64_t outer,
               uint32_t box_inner, uint32_t box_mid) {
    EncodeFn enc = tensor_map_encoder();
    if (!enc) return false;
    const CUtensorMapDataType dt = sizeof(T) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                  : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    cuuint64_t dims[3] = {inner, mid, outer};
    cuuint64_t strides[2] = {inner * sizeof(T), inner * mid * sizeof(T)};
    cuuint32_t box[3] = {box_inner, box_mid, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor maps of one launch: boxes of T steps x the tile's channels for u, delta (and z
// when gated), of T steps x NMAX states for B and C, and of T steps x one warp's channels
// for y when the output rows can be stored by TMA.
template <typename Lo, int NMAX, typename Tin, typename Tout>
bool make_maps(const ScanArgs& a, bool want_z, bool want_y, TMaps* tm) {
    memset(tm, 0, sizeof(*tm));
    bool ok = encode_3d<Tin>(&tm->u, a.u, a.L, a.dim, a.batch, Lo::T, Lo::CH) &&
              encode_3d<Tin>(&tm->dr, a.delta, a.L, a.dim, a.batch, Lo::T, Lo::CH) &&
              encode_3d<Tin>(&tm->B, a.B, a.L, a.N, a.batch, Lo::T, NMAX) &&
              encode_3d<Tin>(&tm->C, a.C, a.L, a.N, a.batch, Lo::T, NMAX);
    if (ok && want_z && a.z) ok = encode_3d<Tin>(&tm->z, a.z, a.L, a.dim, a.batch, Lo::T, Lo::CH);
    if (ok && want_y) ok = encode_3d<Tout>(&tm->y, a.y, a.L, a.dim, a.batch, Lo::T, Lo::CW);
    return ok;
}

// Multiprocessors of the current device (148 on a B200 if the query fails).
int64_t sm_count() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
        return 148;
    return sms;
}

// Rows that TMA can describe: a 16-byte multiple of elements, coordinates in int32.
template <typename T>
bool tma_rows(const ScanArgs& a) {
    const bool fits = a.L < (1LL << 31) && a.dim < (1LL << 31) && a.batch < (1LL << 31);
    return fits && a.L > 0 && (a.L * (int64_t)sizeof(T)) % 16 == 0;
}

// The producer form pays off for a grid of one wave at 2.5 to 3 CTAs per SM (two producer
// warps per CTA then fit beside the compute warps); elsewhere the plain form is faster.
template <typename Lo>
bool producer_plan(const ScanArgs& a, int64_t nz) {
    const int64_t ctas = (a.dim + Lo::CH - 1) / Lo::CH * a.batch * nz;
    const int64_t sms = sm_count();
    return 2 * ctas >= 5 * sms && ctas <= 3 * sms;
}

// One launch of the scan kernel over (channel tiles, batch, segments); `nz` segments
// (the grid's z extent).  TMA launches build their tensor maps from the kernel's layout.
template <int NMAX, int P, int WARPS, int T, typename Tin, typename Tout, int MODE, bool TMA,
          bool ZOH = false, int WS = 0, int CPL = 1>
cudaError_t launch_one(const ScanArgs& a, KParams kp, int64_t nz, cudaStream_t s) {
    using Lo = Layout<NMAX, P, WARPS, T, Tin, Tout, CPL, WS == 2 ? 2 : 1>;
    constexpr int kProd = WS == 0 ? 0 : (WS == 1 ? 1 : S6_WSP);
    constexpr bool kOut = MODE == kFull || MODE == kFullCkpt || MODE == kFullAgg || MODE == kCorr;
    TMaps tm;
    memset(&tm, 0, sizeof(tm));
    kp.y_tma = 0;
    if constexpr (TMA) {
        const bool out16 = kOut && tma_rows<Tout>(a);
        if (!make_maps<Lo, NMAX, Tin, Tout>(a, kOut, out16, &tm)) return cudaErrorInvalidValue;
        kp.y_tma = out16 ? 1 : 0;
    }
    auto kern = scan_kernel<NMAX, P, WARPS, T, Tin, Tout, MODE, TMA, ZOH, WS, CPL>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Lo::bytes);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)((a.dim + Lo::CH - 1) / Lo::CH), (unsigned)a.batch, (unsigned)nz);
    kern<<<grid, Lo::THREADS + 32 * kProd, Lo::bytes, s>>>(kp, tm);
    return cudaGetLastError();
}

// Instantiation per state width for the split passes, checkpoints and the exact ZOH scan:
// N = 16 uses the tuned tile; narrower states keep four states per lane.
template <int NMAX>
struct Tile {
    static constexpr int P = NMAX == 16 ? S6_P16 : NMAX / 4;
    static constexpr int WARPS = NMAX == 16 ? S6_WARPS16 : (NMAX == 8 ? 2 : 1);
    static constexpr int T = NMAX == 16 ? S6_CHUNK : 64;
};

// The plain forward (one pass, no checkpoints, Delta * B weight).
template <int NMAX>
struct TileFwd {
    static constexpr int P = Tile<NMAX>::P;
    static constexpr int CPL = NMAX == 16 ? S6_CPL16 : 1;
    static constexpr int WARPS = NMAX == 16 ? S6_WARPS16F : Tile<NMAX>::WARPS;
    static constexpr int T = Tile<NMAX>::T;
};

template <int NMAX, typename Tin, typename Tout, bool TMA, bool ZOH>
cudaError_t launch_typed(const ScanArgs& a, const KParams& kp, cudaStream_t s) {
    using TL = Tile<NMAX>;
    using TF = TileFwd<NMAX>;
    if (a.nseg > 1 && !a.ckpt) {
        // One pass over every segment from h = 0 (y, end states, summed steps), the fold,
        // then the input-free correction of every segment that starts from a nonzero state
        // (segment 0 only when the caller gave h0), for as long as that state matters.
        cudaError_t e = launch_one<NMAX, TL::P, TL::WARPS, TL::T, Tin, Tout, kFullAgg, TMA, ZOH>(
            a, kp, a.nseg, s);
        if (e != cudaSuccess) return e;
        const int64_t lanes = a.batch * a.dim * a.N;
        carry_all_kernel<<<(unsigned)((lanes + 255) / 256), 256, 0, s>>>(
            a.seg_h, a.seg_sum, a.A, a.batch, a.dim, (int)a.N, (int)a.nseg, a.h0, a.last_state);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        KParams kc = kp;
        kc.seg_first = a.h0 ? 0 : 1;
        return launch_one<NMAX, TL::P, TL::WARPS, TL::T, Tin, Tout, kCorr, TMA, ZOH>(
            a, kc, a.nseg - kc.seg_first, s);
    }
    if (a.nseg > 1) {  // a training forward: exact starts first, so the checkpoints are true
        cudaError_t e = launch_one<NMAX, TL::P, TL::WARPS, TL::T, Tin, Tout, kAggregate, TMA, ZOH>(
            a, kp, a.nseg - 1, s);
        if (e != cudaSuccess) return e;
        const int64_t lanes = a.batch * a.dim * a.N;
        carry_kernel<<<(unsigned)((lanes + 255) / 256), 256, 0, s>>>(
            a.seg_h, a.seg_sum, a.A, a.batch, a.dim, (int)a.N, (int)a.nseg, a.h0);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if constexpr (ZOH) {
        if (a.ckpt)  // the training forward of the exact-ZOH scan: barrier form
            return launch_one<NMAX, TL::P, TL::WARPS, TL::T, Tin, Tout, kFullCkpt, TMA, true>(
                a, kp, a.nseg, s);
    }
    if constexpr (!ZOH) {
        if (a.ckpt) {
            if constexpr (TMA && S6_WS_CKPT) {
                if (producer_plan<Layout<NMAX, TL::P, TL::WARPS, TL::T, Tin, Tout>>(a, a.nseg))
                    return launch_one<NMAX, TL::P, TL::WARPS, TL::T, Tin, Tout, kFullCkpt, TMA,
                                      false, 2>(a, kp, a.nseg, s);
            }
            return launch_one<NMAX, TL::P, TL::WARPS, TL::T, Tin, Tout, kFullCkpt, TMA, false>(
                a, kp, a.nseg, s);
        }
        // the split's rescan keeps the tile its segment plan was made for
        if (a.nseg == 1) {
#ifdef S6_WS
            return launch_one<NMAX, TF::P, TF::WARPS, TF::T, Tin, Tout, kFull, TMA, false,
                              TMA ? S6_WS : 0, TF::CPL>(a, kp, 1, s);
#else
            if constexpr (TMA && TF::CPL == 1) {
                if (producer_plan<Layout<NMAX, TF::P, TF::WARPS, TF::T, Tin, Tout, 1>>(a, 1))
                    return launch_one<NMAX, TF::P, TF::WARPS, TF::T, Tin, Tout, kFull, TMA, false,
                                      2>(a, kp, 1, s);
            }
            return launch_one<NMAX, TF::P, TF::WARPS, TF::T, Tin, Tout, kFull, TMA, false, 0,
                              TF::CPL>(a, kp, 1, s);
#endif
        }
    }
#ifdef S6_WS
    constexpr int kWsSplit = (TMA && !ZOH) ? S6_WS : 0;
#else
    constexpr int kWsSplit = 0;
#endif
#if S6_ZOH_WS
    // the exact-ZOH forward in one pass: the same plan as the Delta*B forward
    if constexpr (ZOH && TMA) {
        if (a.nseg == 1 && producer_plan<Layout<NMAX, TL::P, TL::WARPS, TL::T, Tin, Tout, 1>>(a, 1))
            return launch_one<NMAX, TL::P, TL::WARPS, TL::T, Tin, Tout, kFull, TMA, ZOH, 2>(a, kp, 1, s);
    }
#endif
    return launch_one<NMAX, TL::P, TL::WARPS, TL::T, Tin, Tout, kFull, TMA, ZOH, kWsSplit>(
        a, kp, a.nseg, s);
}

template <int NMAX, typename Tin, typename Tout, bool ZOH>
cudaError_t launch_io(const ScanArgs& a, const KParams& kp, cudaStream_t s) {
    return tma_rows<Tin>(a) ? launch_typed<NMAX, Tin, Tout, true, ZOH>(a, kp, s)
                            : launch_typed<NMAX, Tin, Tout, false, ZOH>(a, kp, s);
}

template <int NMAX, typename Tin, bool ZOH>
cudaError_t launch_ckpt_io(const ScanArgs& a, const KParams& kp, cudaStream_t s) {
    using TL = Tile<NMAX>;
    if (a.nseg > 1) {
        // a split sequence: every segment's true start first (the summaries of all but the
        // last segment from zero, then the fold), so each segment records true states
        const bool tr = tma_rows<Tin>(a);
        cudaError_t e =
            tr ? launch_one<NMAX, TL::P, TL::WARPS, TL::T, Tin, Tin, kAggregate, true, ZOH>(a, kp, a.nseg - 1, s)
               : launch_one<NMAX, TL::P, TL::WARPS, TL::T, Tin, Tin, kAggregate, false, ZOH>(a, kp, a.nseg - 1, s);
        if (e != cudaSuccess) return e;
        const int64_t lanes = a.batch * a.dim * a.N;
        carry_kernel<<<(unsigned)((lanes + 255) / 256), 256, 0, s>>>(
            a.seg_h, a.seg_sum, a.A, a.batch, a.dim, (int)a.N, (int)a.nseg, nullptr);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        return tr ? launch_one<NMAX, TL::P, TL::WARPS, TL::T, Tin, Tin, kCheckpoint, true, ZOH>(a, kp, a.nseg, s)
                  : launch_one<NMAX, TL::P, TL::WARPS, TL::T, Tin, Tin, kCheckpoint, false, ZOH>(a, kp, a.nseg, s);
    }
#if S6_WS_CKPT
    if (!ZOH && tma_rows<Tin>(a) &&
        producer_plan<Layout<NMAX, TL::P, TL::WARPS, TL::T, Tin, Tin>>(a, 1))
        return launch_one<NMAX, TL::P, TL::WARPS, TL::T, Tin, Tin, kCheckpoint, true, false, 2>(
            a, kp, 1, s);
#endif
    return tma_rows<Tin>(a)
               ? launch_one<NMAX, TL::P, TL::WARPS, TL::T, Tin, Tin, kCheckpoint, true, ZOH>(a, kp, 1, s)
               : launch_one<NMAX, TL::P, TL::WARPS, TL::T, Tin, Tin, kCheckpoint, false, ZOH>(a, kp, 1, s);
}

template <int NMAX, bool ZOH>
cudaError_t launch_ckpt_n(const ScanArgs& a, const KParams& kp, cudaStream_t s) {
    return a.in_dtype == DType::BF16 ? launch_ckpt_io<NMAX, __nv_bfloat16, ZOH>(a, kp, s)
                                     : launch_ckpt_io<NMAX, float, ZOH>(a, kp, s);
}

template <bool ZOH>
cudaError_t launch_ckpt_z(const ScanArgs& a, const KParams& kp, cudaStream_t s) {
    if (a.N <= 4) return launch_ckpt_n<4, ZOH>(a, kp, s);
    if (a.N <= 8) return launch_ckpt_n<8, ZOH>(a, kp, s);
    return launch_ckpt_n<16, ZOH>(a, kp, s);
}

// Segment summaries: kAggregate over `nseg` segments (all of them) into seg_h / seg_sum.
template <int NMAX, typename Tin, bool ZOH>
cudaError_t launch_summary_io(const ScanArgs& a, const KParams& kp, cudaStream_t s) {
    using TL = Tile<NMAX>;
    return tma_rows<Tin>(a)
               ? launch_one<NMAX, TL::P, TL::WARPS, TL::T, Tin, Tin, kAggregate, true, ZOH>(a, kp, a.nseg, s)
               : launch_one<NMAX, TL::P, TL::WARPS, TL::T, Tin, Tin, kAggregate, false, ZOH>(a, kp, a.nseg, s);
}

template <int NMAX, bool ZOH>
cudaError_t launch_summary_n(const ScanArgs& a, const KParams& kp, cudaStream_t s) {
    return a.in_dtype == DType::BF16 ? launch_summary_io<NMAX, __nv_bfloat16, ZOH>(a, kp, s)
                                     : launch_summary_io<NMAX, float, ZOH>(a, kp, s);
}

template <bool ZOH>
cudaError_t launch_summary_z(const ScanArgs& a, const KParams& kp, cudaStream_t s) {
    if (a.N <= 4) return launch_summary_n<4, ZOH>(a, kp, s);
    if (a.N <= 8) return launch_summary_n<8, ZOH>(a, kp, s);
    return launch_summary_n<16, ZOH>(a, kp, s);
}

template <int NMAX, bool ZOH>
cudaError_t launch_nmax_z(const ScanArgs& a, const KParams& kp, cudaStream_t s) {
    const bool ib = a.in_dtype == DType::BF16, ob = a.out_dtype == DType::BF16;
    if (ib && ob) return launch_io<NMAX, __nv_bfloat16, __nv_bfloat16, ZOH>(a, kp, s);
    if (ib && !ob) return launch_io<NMAX, __nv_bfloat16, float, ZOH>(a, kp, s);
    if (!ib && ob) return launch_io<NMAX, float, __nv_bfloat16, ZOH>(a, kp, s);
    return launch_io<NMAX, float, float, ZOH>(a, kp, s);
}

template <int NMAX>
cudaError_t launch_nmax(const ScanArgs& a, const KParams& kp, cudaStream_t s) {
    return a.zoh ? launch_nmax_z<NMAX, true>(a, kp, s) : launch_nmax_z<NMAX, false>(a, kp, s);
}

}  // namespace

int scan_chunk_steps(int64_t N) {
    if (N <= 4) return Tile<4>::T;
    if (N <= 8) return Tile<8>::T;
    return Tile<16>::T;
}

int checkpoint_steps(int64_t) { return kCkptSteps; }

cudaError_t launch_scan_checkpoints(const ScanArgs& a, float* ckpt, cudaStream_t stream) {
    KParams kp;
    memset(&kp, 0, sizeof(kp));
    kp.u = a.u;
    kp.delta = a.delta;
    kp.A = a.A;
    kp.B = a.B;
    kp.C = a.C;
    kp.delta_bias = a.delta_bias;
    kp.ckpt = ckpt;
    kp.ck_tiled = ckpt_tiled(a.L, a.N) ? 1 : 0;
    kp.batch = a.batch;
    kp.dim = a.dim;
    kp.L = a.L;
    kp.seg_len = a.L;
    kp.N = (int)a.N;
    kp.nseg = 1;
    kp.softplus = a.softplus ? 1 : 0;
    if (a.nseg > 1) {  // segments of a split sequence, each from its true start
        kp.seg_len = a.seg_len;
        kp.nseg = (int)a.nseg;
        kp.seg_h = a.seg_h;
        kp.seg_sum = a.seg_sum;
    }
    return a.zoh ? launch_ckpt_z<true>(a, kp, stream) : launch_ckpt_z<false>(a, kp, stream);
}

cudaError_t launch_fold(const float* hend, const float* dsum, const float* A, const float* h0,
                        int64_t count, int64_t batch, int64_t dim, int64_t N, float* h_out,
                        float* dsum_out, cudaStream_t stream) {
    const int64_t lanes = batch * dim * N;
    fold_kernel<<<(unsigned)((lanes + 255) / 256), 256, 0, stream>>>(
        hend, dsum, A, h0, count, batch, dim, (int)N, h_out, dsum_out);
    return cudaGetLastError();
}

cudaError_t launch_scan_summary(const ScanArgs& a, float* h_end, float* dsum, cudaStream_t stream) {
    KParams kp;
    memset(&kp, 0, sizeof(kp));
    kp.u = a.u;
    kp.delta = a.delta;
    kp.A = a.A;
    kp.B = a.B;
    kp.C = a.C;
    kp.delta_bias = a.delta_bias;
    kp.batch = a.batch;
    kp.dim = a.dim;
    kp.L = a.L;
    kp.seg_len = a.nseg > 1 ? a.seg_len : (a.L > 0 ? a.L : 1);
    kp.N = (int)a.N;
    kp.nseg = (int)a.nseg;
    kp.softplus = a.softplus ? 1 : 0;
    // one segment: the aggregate pass writes the outputs directly
    kp.seg_h = a.nseg > 1 ? a.seg_h : h_end;
    kp.seg_sum = a.nseg > 1 ? a.seg_sum : dsum;
    cudaError_t e = a.zoh ? launch_summary_z<true>(a, kp, stream) : launch_summary_z<false>(a, kp, stream);
    if (e != cudaSuccess || a.nseg <= 1) return e;
    return launch_fold(a.seg_h, a.seg_sum, a.A, nullptr, a.nseg, a.batch, a.dim, a.N, h_end, dsum,
                       stream);
}

cudaError_t launch_wait_timeout_probe(long long limit_cycles, cudaStream_t stream) {
    wait_timeout_probe_kernel<<<1, 32, 0, stream>>>(limit_cycles);
    return cudaGetLastError();
}

cudaError_t read_device_error(unsigned* out, bool clear, cudaStream_t stream) {
    unsigned v = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_device_error, sizeof(v), 0,
                                              cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e == cudaSuccess && clear && v) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbolAsync(g_device_error, &zero, sizeof(zero), 0,
                                    cudaMemcpyHostToDevice, stream);
        if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    }
    *out = v;
    return e;
}

namespace {

// CTAs of the N-state tile (input and output of type Tio) resident at once on the current
// device: its SM count times the CTAs an SM holds by the tile's shared memory (228 KB per
// SM, 1 KB reserved per CTA) and threads.  One wave.
template <int NMAX, typename Tio>
int64_t wave_ctas() {
    using TL = Tile<NMAX>;
    using Lo = Layout<NMAX, TL::P, TL::WARPS, TL::T, Tio, Tio>;
    constexpr int64_t by_smem = 233472 / ((int64_t)Lo::bytes + 1024);
    constexpr int64_t by_threads = 2048 / Lo::THREADS;
    constexpr int64_t r = by_smem < by_threads ? by_smem : by_threads;
    return sm_count() * (r < 32 ? r : 32);
}

template <int NMAX>
constexpr int64_t tile_channels() {
    using TL = Tile<NMAX>;
    return Layout<NMAX, TL::P, TL::WARPS, TL::T, __nv_bfloat16, __nv_bfloat16>::CH;
}

}  // namespace

namespace {

// Segment length for n segments of L steps: a multiple of kChunk; returns the count that
// length gives.
int64_t segment_len(int64_t L, int64_t n, int64_t* len_out) {
    int64_t len = (L + n - 1) / n;
    len = (len + kChunk - 1) / kChunk * kChunk;
    if (len == 0) len = kChunk;
    *len_out = len;
    return std::max<int64_t>(1, (L + len - 1) / len);
}

}  // namespace

int64_t split_segments_bound(int64_t batch, int64_t dim, int64_t L) {
    // Split only when the channels alone cannot fill the GPU (fewer than 4096, so under
    // about a warp per SM sub-partition) and L is long; at most enough segments for
    // 32768 channel-segments and none shorter than 4096 steps.
    const int64_t channels = batch * dim;
    const int64_t kMinSeg = 4096;
    int64_t n = 1;
    if (channels < 4096 && L >= 4 * kMinSeg) {
        const int64_t want = (32768 + channels - 1) / channels;
        n = std::max<int64_t>(1, std::min<int64_t>(want, L / kMinSeg));
    }
    int64_t len;
    return segment_len(L, n, &len);
}

void plan_segments(int64_t batch, int64_t dim, int64_t dstate, int64_t L, int64_t* nseg,
                   int64_t* seg_len, bool fp32_in) {
    // Each CTA of a split sweeps a whole segment, so a second, partial wave of CTAs costs a
    // whole segment's time again, while the split's extra pass costs about the same for
    // any number of segments: take no more segments than one wave of CTAs holds (and
    // never more than the bound the workspace is sized for).
    int64_t n = split_segments_bound(batch, dim, L);
    if (n > 1) {
        const int64_t ch = dstate <= 4 ? tile_channels<4>() : dstate <= 8 ? tile_channels<8>()
                                                                           : tile_channels<16>();
        int64_t wave;
        if (fp32_in)
            wave = dstate <= 4 ? wave_ctas<4, float>() : dstate <= 8 ? wave_ctas<8, float>()
                                                                     : wave_ctas<16, float>();
        else
            wave = dstate <= 4 ? wave_ctas<4, __nv_bfloat16>()
                   : dstate <= 8 ? wave_ctas<8, __nv_bfloat16>() : wave_ctas<16, __nv_bfloat16>();
        const int64_t per_seg = (dim + ch - 1) / ch * batch;
        n = std::max<int64_t>(1, std::min<int64_t>(n, wave / per_seg));
    }
    *nseg = segment_len(L, n, seg_len);
}

cudaError_t launch_scan(const ScanArgs& a, cudaStream_t stream) {
    KParams kp;
    kp.u = a.u;
    kp.delta = a.delta;
    kp.z = a.z;
    kp.A = a.A;
    kp.B = a.B;
    kp.C = a.C;
    kp.D = a.D;
    kp.delta_bias = a.delta_bias;
    kp.y = a.y;
    kp.last_state = a.last_state;
    // with one segment the kernel reads its initial state through seg_h (read only)
    kp.seg_h = a.nseg > 1 ? a.seg_h : const_cast<float*>(a.h0);
    kp.ckpt = a.ckpt;
    kp.ck_tiled = ckpt_tiled(a.L, a.N) ? 1 : 0;
    kp.seg_sum = a.seg_sum;
    kp.batch = a.batch;
    kp.dim = a.dim;
    kp.L = a.L;
    kp.seg_len = a.seg_len;
    kp.N = (int)a.N;
    kp.nseg = (int)a.nseg;
    kp.softplus = a.softplus ? 1 : 0;
    kp.y_vec = a.L % 4 == 0 ? 1 : 0;
    kp.y_tma = 0;
    kp.seg_first = 0;
    if (a.N <= 4) return launch_nmax<4>(a, kp, stream);
    if (a.N <= 8) return launch_nmax<8>(a, kp, stream);
    return launch_nmax<16>(a, kp, stream);
}

}  // namespace s6
