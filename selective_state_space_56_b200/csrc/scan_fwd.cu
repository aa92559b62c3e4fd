// scan_fwd.cu -- fused selective-scan (S6) forward for sm_100a.
//
// One CTA owns 32 channels of one batch row (and, for a split sequence, one
// segment of L) and walks L in chunks of kChunk steps:
//
//   stage     u, delta, z rows and the batch's B, C rows of the chunk are copied
//             global -> shared with 16-byte async copies (double-buffered, the next
//             chunk streams in while this one computes);
//   phase A   per (channel, t): Delta = softplus(delta + bias), Delta*u  (one warp
//             per 32/P channels; lanes walk t, so every access is conflict-free);
//   phase B   the recurrence.  P lanes share a channel, each holding NS = N/P states
//             in registers: Abar = 2^(Delta * A log2 e) on the SFU,
//             h = Abar h + (Delta u) B, partial y = sum C h.  The P partial sums of
//             each t are combined by a transpose-reduce over lanes (P - 1 shuffles
//             per P steps), leaving one lane with the complete C.h for one t;
//   phase C   y = (C.h + D u) * silu(z), rounded to the output type and stored.
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
#include <algorithm>

#include "s6_device.cuh"
#include "s6_launch.h"

namespace s6 {
namespace {

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
    int64_t batch, dim, L, seg_len;
    int N;
    int nseg;
    int softplus;
    int aligned;
};

enum Mode : int { kFull = 0, kAggregate = 1 };

// Shared-memory carve-up for one instantiation.
template <int NMAX, int P, typename Tin>
struct Layout {
    static constexpr int T = kChunk;
    static constexpr int NS = NMAX / P;        // states per lane
    static constexpr int CW = 32 / P;          // channels per warp
    static constexpr int WARPS = P;            // 32 channels per CTA
    static constexpr int CH = WARPS * CW;
    static constexpr int THREADS = WARPS * 32;
    static constexpr int RS = T + 4;           // fp32 row stride: rows land 16 B apart in banks
    static constexpr int PADB = 16 / (int)sizeof(Tin);
    static constexpr int RB = T + PADB;        // raw B/C row stride (elements)
    static constexpr size_t stage_elems = (size_t)3 * CH * T + (size_t)2 * NMAX * RB;
    static constexpr size_t stage_bytes = stage_elems * sizeof(Tin);
    static constexpr size_t off_bt = 2 * stage_bytes;            // float [T][NMAX]
    static constexpr size_t off_ct = off_bt + (size_t)T * NMAX * 4;
    static constexpr size_t off_del = off_ct + (size_t)T * NMAX * 4;  // float [CH][RS]
    static constexpr size_t off_du = off_del + (size_t)CH * RS * 4;
    static constexpr size_t off_y = off_du + (size_t)CH * RS * 4;
    static constexpr size_t off_par = off_y + (size_t)CH * RS * 4;   // bias[CH], D[CH]
    static constexpr size_t bytes = off_par + (size_t)2 * CH * 4;
    static_assert(NS % 4 == 0, "states per lane must be a multiple of 4");
    static_assert(stage_bytes % 16 == 0, "stages must stay 16-byte aligned");
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
    } else {
        static_assert(P == 4, "P must be 1, 2 or 4");
        const bool hi2 = pp & 2;
        float w0 = (hi2 ? v[2] : v[0]) + __shfl_xor_sync(0xffffffffu, hi2 ? v[0] : v[2], 2);
        float w1 = (hi2 ? v[3] : v[1]) + __shfl_xor_sync(0xffffffffu, hi2 ? v[1] : v[3], 2);
        const bool hi1 = pp & 1;
        return (hi1 ? w1 : w0) + __shfl_xor_sync(0xffffffffu, hi1 ? w0 : w1, 1);
    }
}

template <int NMAX, int P, typename Tin, typename Tout, int MODE>
__global__ void __launch_bounds__(Layout<NMAX, P, Tin>::THREADS)
scan_kernel(const KParams p) {
    using Lo = Layout<NMAX, P, Tin>;
    constexpr int T = Lo::T, NS = Lo::NS, CW = Lo::CW, CH = Lo::CH, RS = Lo::RS, RB = Lo::RB;
    extern __shared__ __align__(16) unsigned char smem[];
    Tin* stage0 = reinterpret_cast<Tin*>(smem);
    Tin* stage1 = reinterpret_cast<Tin*>(smem + Lo::stage_bytes);
    float* sBt = reinterpret_cast<float*>(smem + Lo::off_bt);
    float* sCt = reinterpret_cast<float*>(smem + Lo::off_ct);
    float* sDel = reinterpret_cast<float*>(smem + Lo::off_del);
    float* sDu = reinterpret_cast<float*>(smem + Lo::off_du);
    float* sY = reinterpret_cast<float*>(smem + Lo::off_y);
    float* sBias = reinterpret_cast<float*>(smem + Lo::off_par);
    float* sDsk = sBias + CH;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t b = blockIdx.y;
    const int64_t d0 = (int64_t)blockIdx.x * CH;
    const int seg = blockIdx.z;
    const int64_t t_begin = (int64_t)seg * p.seg_len;
    const int64_t t_end = min(p.L, t_begin + p.seg_len);
    const int64_t nchunks = t_end > t_begin ? (t_end - t_begin + T - 1) / T : 0;
    const bool has_z = (MODE == kFull) && p.z != nullptr;

    for (int c = tid; c < CH; c += Lo::THREADS) {
        const int64_t d = d0 + c;
        const bool ok = d < p.dim;
        sBias[c] = (ok && p.delta_bias) ? p.delta_bias[d] : 0.f;
        sDsk[c] = (ok && p.D) ? p.D[d] : 0.f;
    }

    // This lane's channel and states.
    const int pp = lane % P;
    const int cw = warp * CW + lane / P;
    const int64_t dch = d0 + cw;
    const bool ch_ok = dch < p.dim;
    float a2[NS], h[NS];
#pragma unroll
    for (int n = 0; n < NS; ++n) {
        const int nn = pp * NS + n;
        const bool ok = ch_ok && nn < p.N;
        a2[n] = ok ? p.A[dch * p.N + nn] * kLog2e : 0.f;  // padded states: Abar = 1, b = 0
        h[n] = 0.f;
        if (MODE == kFull && p.nseg > 1 && ok)
            h[n] = p.seg_h[(((int64_t)seg * p.batch + b) * p.dim + dch) * p.N + nn];
    }
    float dsum = 0.f;

    const Tin* gu = static_cast<const Tin*>(p.u);
    const Tin* gdr = static_cast<const Tin*>(p.delta);
    const Tin* gz = static_cast<const Tin*>(p.z);
    const Tin* gB = static_cast<const Tin*>(p.B);
    const Tin* gC = static_cast<const Tin*>(p.C);
    const int nrows_x = has_z ? 3 * CH : 2 * CH;

    // Stage chunk k of this CTA's segment into `st`; rows past dim / N and steps
    // past L are zero-filled.
    auto load_chunk = [&](int64_t k, Tin* st) {
        const int64_t t0 = t_begin + k * T;
        if (p.aligned) {
            constexpr int EPP = 16 / (int)sizeof(Tin);
            constexpr int PPR = T / EPP;
            const int total = (nrows_x + 2 * NMAX) * PPR;
            for (int i = tid; i < total; i += Lo::THREADS) {
                const int r = i / PPR, j = i % PPR;
                const int64_t tt = t0 + j * EPP;
                const Tin* src;
                Tin* dst;
                bool ok;
                if (r < nrows_x) {
                    const int which = r / CH, c = r % CH;
                    const int64_t d = d0 + c;
                    ok = d < p.dim && tt < p.L;
                    const Tin* base = which == 0 ? gu : (which == 1 ? gdr : gz);
                    src = base + ((b * p.dim + (ok ? d : 0)) * p.L + (ok ? tt : 0));
                    dst = st + (size_t)which * CH * T + c * T + j * EPP;
                } else {
                    const int r2 = r - nrows_x, which = r2 / NMAX, n = r2 % NMAX;
                    ok = n < p.N && tt < p.L;
                    const Tin* base = which == 0 ? gB : gC;
                    src = base + ((b * p.N + (ok ? n : 0)) * p.L + (ok ? tt : 0));
                    dst = st + (size_t)3 * CH * T + (size_t)which * NMAX * RB + n * RB + j * EPP;
                }
                cp_async16(dst, src, ok ? 16 : 0);
            }
        } else {
            const int total = (nrows_x + 2 * NMAX) * T;
            for (int i = tid; i < total; i += Lo::THREADS) {
                const int r = i / T, j = i % T;
                const int64_t tt = t0 + j;
                if (r < nrows_x) {
                    const int which = r / CH, c = r % CH;
                    const int64_t d = d0 + c;
                    const Tin* base = which == 0 ? gu : (which == 1 ? gdr : gz);
                    Tin v = Tin(0.f);
                    if (d < p.dim && tt < p.L) v = base[(b * p.dim + d) * p.L + tt];
                    st[(size_t)which * CH * T + c * T + j] = v;
                } else {
                    const int r2 = r - nrows_x, which = r2 / NMAX, n = r2 % NMAX;
                    const Tin* base = which == 0 ? gB : gC;
                    Tin v = Tin(0.f);
                    if (n < p.N && tt < p.L) v = base[(b * p.N + n) * p.L + tt];
                    st[(size_t)3 * CH * T + (size_t)which * NMAX * RB + n * RB + j] = v;
                }
            }
        }
    };

    if (nchunks > 0) load_chunk(0, stage0);
    cp_async_commit();
    for (int64_t k = 0; k < nchunks; ++k) {
        if (k + 1 < nchunks) load_chunk(k + 1, ((k + 1) & 1) ? stage1 : stage0);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();

        const Tin* st = (k & 1) ? stage1 : stage0;
        const Tin* rU = st;
        const Tin* rDr = st + CH * T;
        const Tin* rZ = st + 2 * CH * T;
        const Tin* rB = st + 3 * CH * T;
        const Tin* rC = rB + NMAX * RB;
        const int64_t t0 = t_begin + k * T;
        const int valid = (int)min((int64_t)T, t_end - t0);

        // B, C of the chunk to fp32, time-major: every lane then reads its states'
        // coefficients for step t as one 16-byte vector.
        for (int i = tid; i < NMAX * T; i += Lo::THREADS) {
            const int t = i / NMAX, n = i % NMAX;
            sBt[i] = io<Tin>::to_f(rB[n * RB + t]);
            sCt[i] = io<Tin>::to_f(rC[n * RB + t]);
        }
        __syncthreads();

        // Phase A: step sizes of this warp's channels.  Steps past the end of the
        // segment get Delta = 0 (Abar = 1, no input): the state passes through.
        for (int i = lane; i < CW * T; i += 32) {
            const int c = warp * CW + i / T, t = i % T;
            const float x = io<Tin>::to_f(rDr[c * T + t]) + sBias[c];
            float dt = p.softplus ? softplus(x) : x;
            dt = t < valid ? dt : 0.f;
            sDel[c * RS + t] = dt;
            sDu[c * RS + t] = dt * io<Tin>::to_f(rU[c * T + t]);
        }
        __syncwarp();

        // Phase B: the recurrence, four steps per iteration.
        for (int t = 0; t < T; t += 4) {
            const float4 d4 = *reinterpret_cast<const float4*>(sDel + cw * RS + t);
            const float4 q4 = *reinterpret_cast<const float4*>(sDu + cw * RS + t);
            const float dv[4] = {d4.x, d4.y, d4.z, d4.w};
            const float qv[4] = {q4.x, q4.y, q4.z, q4.w};
            float yp[4];
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const float* bt = sBt + (t + kk) * NMAX + pp * NS;
                const float* ct = sCt + (t + kk) * NMAX + pp * NS;
                float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
                for (int n = 0; n < NS; n += 4) {
                    const float4 bb = *reinterpret_cast<const float4*>(bt + n);
                    const float4 cc = *reinterpret_cast<const float4*>(ct + n);
                    const float bv[4] = {bb.x, bb.y, bb.z, bb.w};
                    const float cv[4] = {cc.x, cc.y, cc.z, cc.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float abar = ex2(dv[kk] * a2[n + j]);
                        h[n + j] = fmaf(abar, h[n + j], qv[kk] * bv[j]);
                        if (j & 1)
                            acc1 = fmaf(cv[j], h[n + j], acc1);
                        else
                            acc0 = fmaf(cv[j], h[n + j], acc0);
                    }
                }
                yp[kk] = acc0 + acc1;
            }
            if (MODE == kAggregate) {
                dsum += (dv[0] + dv[1]) + (dv[2] + dv[3]);
            } else if constexpr (P == 1) {
                *reinterpret_cast<float4*>(sY + cw * RS + t) = make_float4(yp[0], yp[1], yp[2], yp[3]);
            } else {
#pragma unroll
                for (int g = 0; g < 4; g += P) sY[cw * RS + t + g + pp] = transpose_reduce<P>(yp + g, pp);
            }
        }

        if (MODE == kFull) {
            __syncwarp();
            // Phase C: skip term, gate, store (lanes walk t: coalesced rows).
            Tout* gy = static_cast<Tout*>(p.y);
            for (int i = lane; i < CW * T; i += 32) {
                const int c = warp * CW + i / T, t = i % T;
                const int64_t d = d0 + c;
                if (t < valid && d < p.dim) {
                    float yv = sY[c * RS + t] + sDsk[c] * io<Tin>::to_f(rU[c * T + t]);
                    if (has_z) yv *= silu(io<Tin>::to_f(rZ[c * T + t]));
                    gy[(b * p.dim + d) * p.L + t0 + t] = io<Tout>::from_f(yv);
                }
            }
        }
        __syncthreads();
    }

    if (MODE == kFull) {
        if (p.last_state && seg == (int)gridDim.z - 1 && ch_ok) {
#pragma unroll
            for (int n = 0; n < NS; ++n) {
                const int nn = pp * NS + n;
                if (nn < p.N) p.last_state[(b * p.dim + dch) * p.N + nn] = h[n];
            }
        }
    } else if (ch_ok) {
        const int64_t row = ((int64_t)seg * p.batch + b) * p.dim + dch;
#pragma unroll
        for (int n = 0; n < NS; ++n) {
            const int nn = pp * NS + n;
            if (nn < p.N) p.seg_h[row * p.N + nn] = h[n];
        }
        if (pp == 0) p.seg_sum[row] = dsum;
    }
}

// Fold the segments left to right.  Thread per (batch, channel, state):
// on entry seg_h[s] holds segment s's end state from h = 0 (s < nseg - 1) and
// seg_sum[s] its summed step; on exit seg_h[s] holds segment s's true start state.
__global__ void carry_kernel(float* seg_h, const float* seg_sum, const float* A, int64_t batch,
                             int64_t dim, int N, int nseg) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t lanes = batch * dim * N;
    if (i >= lanes) return;
    const int n = (int)(i % N);
    const int64_t bd = i / N;
    const int64_t d = bd % dim;
    const float a2 = A[d * N + n] * kLog2e;
    float H = 0.f;
    for (int s = 0; s < nseg - 1; ++s) {
        const int64_t row = (int64_t)s * batch * dim + bd;
        const float hend = seg_h[row * N + n];
        seg_h[row * N + n] = H;
        H = fmaf(ex2(a2 * seg_sum[row]), H, hend);  // (prod Abar, h_end) (+) (., H)
    }
    seg_h[((int64_t)(nseg - 1) * batch * dim + bd) * N + n] = H;
}

template <int NMAX, int P, typename Tin, typename Tout, int MODE>
cudaError_t launch_one(const KParams& kp, dim3 grid, cudaStream_t s) {
    using Lo = Layout<NMAX, P, Tin>;
    auto kern = scan_kernel<NMAX, P, Tin, Tout, MODE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Lo::bytes);
    if (e != cudaSuccess) return e;
    kern<<<grid, Lo::THREADS, Lo::bytes, s>>>(kp);
    return cudaGetLastError();
}

template <int NMAX, typename Tin, typename Tout>
cudaError_t launch_typed(const ScanArgs& a, KParams kp, cudaStream_t s) {
    constexpr int P = NMAX / 4;
    using Lo = Layout<NMAX, P, Tin>;
    const unsigned gx = (unsigned)((a.dim + Lo::CH - 1) / Lo::CH);
    if (a.nseg > 1) {
        cudaError_t e = launch_one<NMAX, P, Tin, Tout, kAggregate>(
            kp, dim3(gx, (unsigned)a.batch, (unsigned)(a.nseg - 1)), s);
        if (e != cudaSuccess) return e;
        const int64_t lanes = a.batch * a.dim * a.N;
        carry_kernel<<<(unsigned)((lanes + 255) / 256), 256, 0, s>>>(
            a.seg_h, a.seg_sum, a.A, a.batch, a.dim, (int)a.N, (int)a.nseg);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return launch_one<NMAX, P, Tin, Tout, kFull>(kp, dim3(gx, (unsigned)a.batch, (unsigned)a.nseg),
                                                 s);
}

template <int NMAX>
cudaError_t launch_nmax(const ScanArgs& a, const KParams& kp, cudaStream_t s) {
    const bool ib = a.in_dtype == DType::BF16, ob = a.out_dtype == DType::BF16;
    if (ib && ob) return launch_typed<NMAX, __nv_bfloat16, __nv_bfloat16>(a, kp, s);
    if (ib && !ob) return launch_typed<NMAX, __nv_bfloat16, float>(a, kp, s);
    if (!ib && ob) return launch_typed<NMAX, float, __nv_bfloat16>(a, kp, s);
    return launch_typed<NMAX, float, float>(a, kp, s);
}

}  // namespace

void plan_segments(int64_t batch, int64_t dim, int64_t L, int64_t* nseg, int64_t* seg_len) {
    // Split only when the channels alone cannot fill the GPU (fewer than 4096 lanes
    // of 32 channels... i.e. under ~1 warp per SM sub-partition) and L is long:
    // a split costs a second pass over all but the last segment.
    const int64_t channels = batch * dim;
    const int64_t kMinSeg = 4096;
    int64_t n = 1;
    if (channels < 4096 && L >= 4 * kMinSeg) {
        const int64_t want = (32768 + channels - 1) / channels;
        n = std::max<int64_t>(1, std::min<int64_t>(want, L / kMinSeg));
    }
    int64_t len = (L + n - 1) / n;
    len = (len + kChunk - 1) / kChunk * kChunk;
    if (len == 0) len = kChunk;
    n = std::max<int64_t>(1, (L + len - 1) / len);
    *nseg = n;
    *seg_len = len;
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
    kp.seg_h = a.seg_h;
    kp.seg_sum = a.seg_sum;
    kp.batch = a.batch;
    kp.dim = a.dim;
    kp.L = a.L;
    kp.seg_len = a.seg_len;
    kp.N = (int)a.N;
    kp.nseg = (int)a.nseg;
    kp.softplus = a.softplus ? 1 : 0;
    const int64_t esize = a.in_dtype == DType::BF16 ? 2 : 4;
    kp.aligned = (a.L * esize) % 16 == 0 ? 1 : 0;  // base pointers are checked by the ABI
    if (a.N <= 4) return launch_nmax<4>(a, kp, stream);
    if (a.N <= 8) return launch_nmax<8>(a, kp, stream);
    return launch_nmax<16>(a, kp, stream);
}

}  // namespace s6
