// scan_bwd.cu -- backward of the selective scan (S6) with recomputation, sm_100a.
//
// Mamba ("Hardware-aware state expansion"): the intermediate states are not stored for
// the backward pass; they are recomputed on chip.  Here the forward kernel first records
// only the state entering every chunk (checkpoints, one N-vector per 32 steps per
// channel).  This kernel then walks the chunks of a channel tile in reverse:
//
//   stage     u, delta, z, dy rows and the batch's B, C for the chunk -> shared memory;
//   phase A   per (channel, t): Delta, softplus'(x), Delta*u, silu(z), silu'(z);
//   forward   the chunk's states h_t recomputed from the checkpoint into shared memory
//             (4 states per lane, 4 lanes per channel), and the pre-gate output
//             yt_t = C.h + D u (lane transpose-reduce) for dz;
//   reverse   the adjoint state g (registers) swept from the chunk's last step to its
//             first: g += dyt C;  dC += dyt h;  dB += g Delta u;  dq = g.B;
//             dDelta = dq u + sum g h_{t-1} Abar A;  dA += g h_{t-1} Abar Delta;
//             g *= Abar.  dq and the state part of dDelta are summed over a channel's
//             lanes every four steps (transpose-reduce); dB and dC, shared by all
//             channels of a batch, are summed over the warp's channels per step
//             (8-lane transpose-reduce), over the CTA in shared memory, and added to
//             global memory with one atomic per (t, n) and CTA;
//   store     du, dDelta_raw (= dDelta * softplus'(x)), dz; dA, dD, dbias by atomics.
//
// Gradients flowing through softplus use softplus'(x) = sigmoid(x); through the gate
// silu'(z) = sigmoid(z) (1 + z (1 - sigmoid(z))).
#include <cstring>

#include "s6_device.cuh"
#include "s6_launch.h"

namespace s6 {
namespace {

struct BParams {
    const void* u;
    const void* delta;
    const void* z;
    const void* dy;
    const float* A;
    const void* B;
    const void* C;
    const float* D;
    const float* delta_bias;
    const float* ckpt;
    void* du;
    void* ddelta;
    void* dz;
    float* dA;
    float* dD;
    float* dbias;
    float* dB;
    float* dC;
    int64_t batch, dim, L;
    int N;
    int softplus;
    int chunks;
};

constexpr int kBW = 2;           // warps per CTA
constexpr int kBP = 4;           // lanes per channel
constexpr int kBG = 32 / kBP;    // channels per warp
constexpr int kBCH = kBW * kBG;  // channels per CTA

constexpr size_t a16(size_t x) { return (x + 15) / 16 * 16; }

template <int T, typename Tin>
struct BLayout {
    static constexpr int RS = T + 4;
    static constexpr size_t raw = a16((size_t)kBCH * T * sizeof(Tin));  // one [CH][T] row set
    static constexpr size_t off_u = 0;
    static constexpr size_t off_dr = off_u + raw;
    static constexpr size_t off_z = off_dr + raw;
    static constexpr size_t off_dy = off_z + raw;
    static constexpr size_t off_B = off_dy + raw;                 // fp32 [T][16]
    static constexpr size_t off_C = off_B + (size_t)T * 16 * 4;
    static constexpr size_t f = (size_t)kBCH * RS * 4;           // one fp32 [CH][RS]
    static constexpr size_t off_del = off_C + (size_t)T * 16 * 4;
    static constexpr size_t off_q = off_del + f;
    static constexpr size_t off_sg = off_q + f;                  // softplus'(x)
    static constexpr size_t off_gz = off_sg + f;                 // silu(z), then dy*silu(z)
    static constexpr size_t off_ds = off_gz + f;                 // silu'(z)
    static constexpr size_t off_yt = off_ds + f;                 // pre-gate output
    static constexpr size_t off_odu = off_yt + f;                // Tin [CH][T] outputs
    static constexpr size_t off_odd = off_odu + raw;
    static constexpr size_t off_odz = off_odd + raw;
    static constexpr size_t off_h = a16(off_odz + raw);          // fp32 [T][CH][16]
    static constexpr size_t off_acc = off_h + (size_t)T * kBCH * 16 * 4;  // fp32 [T][32]
    static constexpr size_t bytes = off_acc + (size_t)T * 32 * 4;
};

__device__ __forceinline__ float sigmoidf_fast(float x) { return rcp(1.f + ex2(-x * kLog2e)); }

// Sum of v[0..7] over the 8 lanes that share lane % 4 (lane bits 2..4): afterwards the
// lane with channel index cl = lane / 4 holds the total of entry cl.
__device__ __forceinline__ float transpose_reduce8(const float (&v)[8], int lane) {
    const bool b1 = lane & 16, b2 = lane & 8, b3 = lane & 4;
    float w[4], x[2];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        w[i] = (b1 ? v[i + 4] : v[i]) + __shfl_xor_sync(0xffffffffu, b1 ? v[i] : v[i + 4], 16);
#pragma unroll
    for (int i = 0; i < 2; ++i)
        x[i] = (b2 ? w[i + 2] : w[i]) + __shfl_xor_sync(0xffffffffu, b2 ? w[i] : w[i + 2], 8);
    return (b3 ? x[1] : x[0]) + __shfl_xor_sync(0xffffffffu, b3 ? x[0] : x[1], 4);
}

// Four partial sums (entries 0..3) over the 4 lanes of a channel: lane pp gets entry pp.
__device__ __forceinline__ float transpose_reduce4(const float (&v)[4], int pp) {
    const bool hi2 = pp & 2;
    const float w0 = (hi2 ? v[2] : v[0]) + __shfl_xor_sync(0xffffffffu, hi2 ? v[0] : v[2], 2);
    const float w1 = (hi2 ? v[3] : v[1]) + __shfl_xor_sync(0xffffffffu, hi2 ? v[1] : v[3], 2);
    const bool hi1 = pp & 1;
    return (hi1 ? w1 : w0) + __shfl_xor_sync(0xffffffffu, hi1 ? w0 : w1, 1);
}

template <int T, typename Tin>
__global__ void __launch_bounds__(kBW * 32) scan_bwd_kernel(const BParams p) {
    using Lo = BLayout<T, Tin>;
    constexpr int RS = Lo::RS;
    extern __shared__ __align__(16) unsigned char smem[];
    Tin* rU = reinterpret_cast<Tin*>(smem + Lo::off_u);
    Tin* rDr = reinterpret_cast<Tin*>(smem + Lo::off_dr);
    Tin* rZ = reinterpret_cast<Tin*>(smem + Lo::off_z);
    Tin* rDy = reinterpret_cast<Tin*>(smem + Lo::off_dy);
    float* sB = reinterpret_cast<float*>(smem + Lo::off_B);
    float* sC = reinterpret_cast<float*>(smem + Lo::off_C);
    float* sDel = reinterpret_cast<float*>(smem + Lo::off_del);
    float* sQ = reinterpret_cast<float*>(smem + Lo::off_q);
    float* sSg = reinterpret_cast<float*>(smem + Lo::off_sg);
    float* sGz = reinterpret_cast<float*>(smem + Lo::off_gz);
    float* sDs = reinterpret_cast<float*>(smem + Lo::off_ds);
    float* sYt = reinterpret_cast<float*>(smem + Lo::off_yt);
    Tin* oDu = reinterpret_cast<Tin*>(smem + Lo::off_odu);
    Tin* oDd = reinterpret_cast<Tin*>(smem + Lo::off_odd);
    Tin* oDz = reinterpret_cast<Tin*>(smem + Lo::off_odz);
    float* sH = reinterpret_cast<float*>(smem + Lo::off_h);
    float* sAcc = reinterpret_cast<float*>(smem + Lo::off_acc);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int pp = lane & 3, cl = lane >> 2;
    const int cw = warp * kBG + cl;
    const int64_t b = blockIdx.y, d0 = (int64_t)blockIdx.x * kBCH, dch = d0 + cw;
    const bool chok = dch < p.dim;
    const bool has_z = p.z != nullptr;

    float a2[4], an[4], g[4], dAacc[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int n = pp * 4 + j;
        an[j] = (chok && n < p.N) ? p.A[dch * p.N + n] : 0.f;  // padded states stay zero
        a2[j] = an[j] * kLog2e;
        g[j] = 0.f;
        dAacc[j] = 0.f;
    }
    const float Dd = (chok && p.D) ? p.D[dch] : 0.f;
    float dDacc = 0.f, dbacc = 0.f;

    for (int k = p.chunks - 1; k >= 0; --k) {
        const int64_t t0 = (int64_t)k * T;
        const int valid = (int)min((int64_t)T, p.L - t0);
        __syncthreads();  // the previous (later) chunk is done with shared memory

        // stage: rows past dim and steps past L are zero
        for (int i = tid; i < 4 * kBCH * T; i += kBW * 32) {
            const int which = i / (kBCH * T), r = (i / T) % kBCH, t = i % T;
            const int64_t d = d0 + r;
            const Tin* src = static_cast<const Tin*>(which == 0 ? p.u : which == 1 ? p.delta
                                                     : which == 2 ? p.z : p.dy);
            Tin* dst = which == 0 ? rU : which == 1 ? rDr : which == 2 ? rZ : rDy;
            Tin v = Tin(0.f);
            if (d < p.dim && t < valid && src) v = src[(b * p.dim + d) * p.L + t0 + t];
            dst[r * T + t] = v;
        }
        for (int i = tid; i < 2 * 16 * T; i += kBW * 32) {
            const int which = i / (16 * T), n = (i / T) % 16, t = i % T;
            const Tin* src = static_cast<const Tin*>(which ? p.C : p.B);
            float v = 0.f;
            if (n < p.N && t < valid) v = io<Tin>::to_f(src[(b * p.N + n) * p.L + t0 + t]);
            (which ? sC : sB)[t * 16 + n] = v;
        }
        for (int i = tid; i < T * 32; i += kBW * 32) sAcc[i] = 0.f;
        __syncthreads();

        // phase A: per (channel, t) of this warp
        for (int i = lane; i < kBG * T; i += 32) {
            const int c = warp * kBG + i / T, t = i % T;
            const int64_t d = d0 + c;
            const float bias = (d < p.dim && p.delta_bias) ? p.delta_bias[d] : 0.f;
            const float x = io<Tin>::to_f(rDr[c * T + t]) + bias;
            float dt = p.softplus ? softplus(x) : x;
            dt = t < valid ? dt : 0.f;
            const float zz = io<Tin>::to_f(rZ[c * T + t]);
            const float sz = sigmoidf_fast(zz);
            sDel[c * RS + t] = dt;
            sQ[c * RS + t] = dt * io<Tin>::to_f(rU[c * T + t]);
            sSg[c * RS + t] = p.softplus ? sigmoidf_fast(x) : 1.f;
            sGz[c * RS + t] = has_z ? zz * sz : 1.f;
            sDs[c * RS + t] = has_z ? sz * (1.f + zz * (1.f - sz)) : 0.f;
        }
        __syncwarp();

        // forward: the chunk's states from its checkpoint
        float hck[4], h[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = pp * 4 + j;
            hck[j] = (chok && n < p.N) ? p.ckpt[((b * p.dim + dch) * p.chunks + k) * p.N + n] : 0.f;
            h[j] = hck[j];
        }
        for (int t = 0; t < T; t += 4) {
            float yp[4];
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                const float dt = sDel[cw * RS + t + s], q = sQ[cw * RS + t + s];
                const float4 bb = *reinterpret_cast<const float4*>(sB + (t + s) * 16 + pp * 4);
                const float4 cc = *reinterpret_cast<const float4*>(sC + (t + s) * 16 + pp * 4);
                const float bv[4] = {bb.x, bb.y, bb.z, bb.w}, cv[4] = {cc.x, cc.y, cc.z, cc.w};
                float acc = 0.f;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    h[j] = fmaf(ex2(dt * a2[j]), h[j], q * bv[j]);
                    acc = fmaf(cv[j], h[j], acc);
                }
                *reinterpret_cast<float4*>(sH + ((t + s) * kBCH + cw) * 16 + pp * 4) =
                    make_float4(h[0], h[1], h[2], h[3]);
                yp[s] = acc;
            }
            sYt[cw * RS + t + pp] = transpose_reduce4(yp, pp) +
                                    Dd * io<Tin>::to_f(rU[cw * T + t + pp]);
        }
        __syncwarp();

        // dz and dy * silu(z) per (channel, t)
        for (int i = lane; i < kBG * T; i += 32) {
            const int c = warp * kBG + i / T, t = i % T;
            const float dyv = io<Tin>::to_f(rDy[c * T + t]);
            oDz[c * T + t] = io<Tin>::from_f(dyv * sYt[c * RS + t] * sDs[c * RS + t]);
            sGz[c * RS + t] = dyv * sGz[c * RS + t];
        }
        __syncwarp();

        // reverse sweep, four steps per group (last group first)
        for (int tg = T - 4; tg >= 0; tg -= 4) {
            float dqv[4], ddv[4];
#pragma unroll
            for (int s = 3; s >= 0; --s) {
                const int t = tg + s;
                const float dyt = sGz[cw * RS + t], dt = sDel[cw * RS + t], q = sQ[cw * RS + t];
                const float4 bb = *reinterpret_cast<const float4*>(sB + t * 16 + pp * 4);
                const float4 cc = *reinterpret_cast<const float4*>(sC + t * 16 + pp * 4);
                const float4 hc = *reinterpret_cast<const float4*>(sH + (t * kBCH + cw) * 16 + pp * 4);
                float hpv[4];
                if (t > 0) {
                    const float4 hpr =
                        *reinterpret_cast<const float4*>(sH + ((t - 1) * kBCH + cw) * 16 + pp * 4);
                    hpv[0] = hpr.x, hpv[1] = hpr.y, hpv[2] = hpr.z, hpv[3] = hpr.w;
                } else {
                    hpv[0] = hck[0], hpv[1] = hck[1], hpv[2] = hck[2], hpv[3] = hck[3];
                }
                const float bv[4] = {bb.x, bb.y, bb.z, bb.w}, cv[4] = {cc.x, cc.y, cc.z, cc.w};
                const float hv[4] = {hc.x, hc.y, hc.z, hc.w};
                float part[8], dq = 0.f, dd = 0.f;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    g[j] = fmaf(dyt, cv[j], g[j]);
                    part[4 + j] = dyt * hv[j];  // dC
                    part[j] = g[j] * q;         // dB
                    dq = fmaf(g[j], bv[j], dq);
                    const float abar = ex2(dt * a2[j]);
                    const float gh = g[j] * hpv[j] * abar;
                    dd = fmaf(gh, an[j], dd);
                    dAacc[j] = fmaf(gh, dt, dAacc[j]);
                    g[j] *= abar;
                }
                dqv[s] = dq;
                ddv[s] = dd;
                // dB / dC of step t summed over the warp's 8 channels, then over the CTA
                const float r = transpose_reduce8(part, lane);
                const int slot = (cl < 4 ? 0 : 16) + pp * 4 + (cl & 3);
                atomicAdd(&sAcc[t * 32 + slot], r);
            }
            // lane pp completes step tg + pp of its channel
            const float dq = transpose_reduce4(dqv, pp), dd = transpose_reduce4(ddv, pp);
            const int t = tg + pp;
            const float uu = io<Tin>::to_f(rU[cw * T + t]);
            const float dyt = sGz[cw * RS + t], dt = sDel[cw * RS + t];
            const float ddelta = (dd + dq * uu) * sSg[cw * RS + t];
            oDu[cw * T + t] = io<Tin>::from_f(fmaf(dyt, Dd, dq * dt));
            oDd[cw * T + t] = io<Tin>::from_f(ddelta);
            if (t < valid) {
                dbacc += ddelta;
                dDacc = fmaf(dyt, uu, dDacc);
            }
        }
        __syncthreads();

        // store du, ddelta, dz rows and add the CTA's dB / dC of the chunk
        for (int i = tid; i < kBCH * T; i += kBW * 32) {
            const int r = i / T, t = i % T;
            const int64_t d = d0 + r;
            if (d >= p.dim || t >= valid) continue;
            const int64_t off = (b * p.dim + d) * p.L + t0 + t;
            static_cast<Tin*>(p.du)[off] = oDu[r * T + t];
            static_cast<Tin*>(p.ddelta)[off] = oDd[r * T + t];
            if (p.dz) static_cast<Tin*>(p.dz)[off] = oDz[r * T + t];
        }
        for (int i = tid; i < T * 32; i += kBW * 32) {
            const int t = i / 32, slot = i % 32, n = slot & 15;
            if (t >= valid || n >= p.N) continue;
            float* dst = slot < 16 ? p.dB : p.dC;
            atomicAdd(dst + (b * p.N + n) * p.L + t0 + t, sAcc[i]);
        }
    }

    if (chok) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (pp * 4 + j < p.N) atomicAdd(p.dA + dch * p.N + pp * 4 + j, dAacc[j]);
    }
    // dD and dbias: sum the 4 lanes of the channel
    dDacc += __shfl_xor_sync(0xffffffffu, dDacc, 1);
    dDacc += __shfl_xor_sync(0xffffffffu, dDacc, 2);
    dbacc += __shfl_xor_sync(0xffffffffu, dbacc, 1);
    dbacc += __shfl_xor_sync(0xffffffffu, dbacc, 2);
    if (chok && pp == 0) {
        if (p.dD) atomicAdd(p.dD + dch, dDacc);
        if (p.dbias) atomicAdd(p.dbias + dch, dbacc);
    }
}

template <int T, typename Tin>
cudaError_t launch_bwd_typed(const BParams& bp, int64_t batch, int64_t dim, cudaStream_t s) {
    using Lo = BLayout<T, Tin>;
    auto kern = scan_bwd_kernel<T, Tin>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Lo::bytes);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)((dim + kBCH - 1) / kBCH), (unsigned)batch, 1);
    kern<<<grid, kBW * 32, Lo::bytes, s>>>(bp);
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_bwd_io(const BParams& bp, int T, int64_t batch, int64_t dim, cudaStream_t s) {
    if (T == 32) return launch_bwd_typed<32, Tin>(bp, batch, dim, s);
    if (T == 64) return launch_bwd_typed<64, Tin>(bp, batch, dim, s);
    return cudaErrorInvalidConfiguration;
}

}  // namespace

cudaError_t launch_scan_backward(const ScanArgs& a, const BackwardArgs& g, float* ckpt,
                                 cudaStream_t stream) {
    // the backward walks the chunks the forward checkpointed
    const int T = scan_chunk_steps(a.N);
    const int64_t chunks = (a.L + T - 1) / T;
    cudaError_t e;
    // outputs accumulated with atomics start at zero
    const size_t bnl = (size_t)a.batch * a.N * a.L * sizeof(float);
    if ((e = cudaMemsetAsync(g.dB, 0, bnl, stream)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(g.dC, 0, bnl, stream)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(g.dA, 0, (size_t)a.dim * a.N * sizeof(float), stream)) != cudaSuccess)
        return e;
    if (g.dD && (e = cudaMemsetAsync(g.dD, 0, (size_t)a.dim * sizeof(float), stream)) != cudaSuccess)
        return e;
    if (g.ddelta_bias &&
        (e = cudaMemsetAsync(g.ddelta_bias, 0, (size_t)a.dim * sizeof(float), stream)) != cudaSuccess)
        return e;
    if (a.L == 0) return cudaSuccess;
    if ((e = launch_scan_checkpoints(a, ckpt, stream)) != cudaSuccess) return e;
    BParams bp;
    memset(&bp, 0, sizeof(bp));
    bp.u = a.u;
    bp.delta = a.delta;
    bp.z = a.z;
    bp.dy = g.dy;
    bp.A = a.A;
    bp.B = a.B;
    bp.C = a.C;
    bp.D = a.D;
    bp.delta_bias = a.delta_bias;
    bp.ckpt = ckpt;
    bp.du = g.du;
    bp.ddelta = g.ddelta;
    bp.dz = g.dz;
    bp.dA = g.dA;
    bp.dD = g.dD;
    bp.dbias = g.ddelta_bias;
    bp.dB = g.dB;
    bp.dC = g.dC;
    bp.batch = a.batch;
    bp.dim = a.dim;
    bp.L = a.L;
    bp.N = (int)a.N;
    bp.softplus = a.softplus ? 1 : 0;
    bp.chunks = (int)chunks;
    if (a.in_dtype == DType::BF16) return launch_bwd_io<__nv_bfloat16>(bp, T, a.batch, a.dim, stream);
    return launch_bwd_io<float>(bp, T, a.batch, a.dim, stream);
}

}  // namespace s6
