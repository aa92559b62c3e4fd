// state_update.cu -- single-token selective_state_update for sm_100a.
//
// Decode keeps only the (batch, dim, N) fp32 state per layer and advances it by one
// token (Mamba FAQ on generation: a fixed-size state, constant cost per token).
// The step is a pure stream over the state: each element is read once and
// written once in place, so the kernel is laid out for HBM: G = NMAX / 4 adjacent
// threads share one (batch, channel) lane and each moves 16 contiguous bytes of
// state, so a warp touches 512 consecutive bytes per access.  The per-lane
// readout sum_n C_n h_n is finished with log2(G) xor-shuffles.  A compile-time
// variant uses the exact zero-order-hold input weight (e^{Delta A} - 1) / A.
#include <algorithm>

#include "s6_device.cuh"
#include "s6_launch.h"

namespace s6 {
namespace {

struct UParams {
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
    int64_t batch, dim, lanes;
    int N;
    int softplus;
    int vec;  // N % 4 == 0: 16-byte state / A accesses
};

template <int NMAX, typename Tio, bool ZOH>
__global__ void __launch_bounds__(256) state_update_kernel(const UParams p) {
    constexpr int G = NMAX / 4;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t lane_id = gid / G;
    const int j = (int)(gid % G);
    const bool active = lane_id < p.lanes;
    const int64_t li = active ? lane_id : 0;
    const int64_t bb = li / p.dim, d = li % p.dim;

    const float uu = io<Tio>::load(static_cast<const Tio*>(p.u) + li);
    const float x = io<Tio>::load(static_cast<const Tio*>(p.delta) + li) +
                    (p.delta_bias ? p.delta_bias[d] : 0.f);
    const float dt = p.softplus ? softplus(x) : x;
    const float du = dt * uu;

    float st[4], a[4], bv[4], cv[4];
    const int n0 = 4 * j;
    float* sp = p.state + li * p.N + n0;
    const float* ap = p.A + d * p.N + n0;
    const Tio* bp = static_cast<const Tio*>(p.B) + bb * p.N + n0;
    const Tio* cp = static_cast<const Tio*>(p.C) + bb * p.N + n0;
    const bool jok = n0 < p.N;  // with N % 4 == 0, all four states exist or none
    if (p.vec) {
        const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 s4 = (active && jok) ? *reinterpret_cast<const float4*>(sp) : z4;
        const float4 a4 = jok ? *reinterpret_cast<const float4*>(ap) : z4;
        st[0] = s4.x, st[1] = s4.y, st[2] = s4.z, st[3] = s4.w;
        a[0] = a4.x, a[1] = a4.y, a[2] = a4.z, a[3] = a4.w;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            bv[k] = jok ? io<Tio>::load(bp + k) : 0.f;
            cv[k] = jok ? io<Tio>::load(cp + k) : 0.f;
        }
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const bool ok = active && n0 + k < p.N;
            st[k] = ok ? sp[k] : 0.f;
            a[k] = ok ? ap[k] : 0.f;
            bv[k] = ok ? io<Tio>::load(bp + k) : 0.f;
            cv[k] = ok ? io<Tio>::load(cp + k) : 0.f;
        }
    }
    float acc = 0.f;
    if constexpr (ZOH) {
        // exact zero-order hold: Bbar = (e^{Delta A} - 1) / A * B, states in pairs; 1 / A
        // from rcp.approx (within 1 ulp; infinite for A = 0, where the series branch applies)
        const f2 uu2 = pack2(uu, uu), qq2 = pack2(du, du);
#pragma unroll
        for (int k = 0; k < 4; k += 2) {
            const f2 x = pack2(dt * (a[k] * kLog2e), dt * (a[k + 1] * kLog2e));
            const f2 e = ex2x2(x);
            const f2 m = zoh_weight_u2(x, e, pack2(rcp(a[k]), rcp(a[k + 1])), uu2, qq2);
            float e0, e1, m0, m1;
            unpack2(e, e0, e1);
            unpack2(m, m0, m1);
            st[k] = fmaf(e0, st[k], m0 * bv[k]);
            st[k + 1] = fmaf(e1, st[k + 1], m1 * bv[k + 1]);
            acc = fmaf(cv[k], st[k], acc);
            acc = fmaf(cv[k + 1], st[k + 1], acc);
        }
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float abar = ex2(dt * (a[k] * kLog2e));
            st[k] = fmaf(abar, st[k], du * bv[k]);
            acc = fmaf(cv[k], st[k], acc);
        }
    }
    if (active && jok) {
        if (p.vec) {
            *reinterpret_cast<float4*>(sp) = make_float4(st[0], st[1], st[2], st[3]);
        } else {
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if (n0 + k < p.N) sp[k] = st[k];
        }
    }
#pragma unroll
    for (int m = G / 2; m >= 1; m /= 2) acc += __shfl_xor_sync(0xffffffffu, acc, m);
    if (active && j == 0) {
        float yv = acc + (p.D ? p.D[d] : 0.f) * uu;
        if (p.z) yv *= silu(io<Tio>::load(static_cast<const Tio*>(p.z) + li));
        static_cast<Tio*>(p.y)[li] = io<Tio>::from_f(yv);
    }
}

// N = 16 fast path.  Two threads per (batch, channel) lane, each owning eight states:
// thread h holds states 4h..4h+3 and 8+4h..8+4h+3, so for every 16-byte access the two
// threads of a lane cover one whole 32-byte sector and a warp moves 16 contiguous lanes
// (1 KiB of state) per instruction pair.  The default (persistent) kernel keeps one wave of
// CTAs resident; each thread walks its lanes a grid stride apart with the next lane's loads
// issued before the current lane's arithmetic, and one thread per CTA bulk-prefetches into
// L2 the state block the CTA reaches two strides later.  The other form serves kItems lanes
// per thread and issues every load of all of them before any arithmetic.  Math runs on
// packed fp32 pairs.
#ifndef S6_DEC_ITEMS
#define S6_DEC_ITEMS 2
#endif
// Nonzero: the persistent variant with up to that many CTAs per SM (fewer when the
// instantiation's registers allow fewer); 0: one lane pair per S6_DEC_ITEMS, one wave after
// another.  Measured on the decode workload (256 x 5120 x 16, bf16, L2 flushed before the
// token): 35.6 us with two items per thread, 35.0 us persistent without prefetch, 33.5 us
// persistent with the prefetch two rounds ahead.
#ifndef S6_DEC_PERSIST
#define S6_DEC_PERSIST 3
#endif
// Persistent variant: one thread per CTA prefetches into L2 the state (and u, delta, z)
// of the lanes this CTA takes S6_DEC_PREFETCH grid strides ahead (0 = no prefetch), so
// the HBM reads of later rounds are in flight while this round computes.
#ifndef S6_DEC_PREFETCH
#define S6_DEC_PREFETCH 2
#endif
// Persistent variant: pick a grid whose lane stride is a multiple of dim, so each thread
// keeps one channel and loads its A, D and delta bias (and 1 / A for exact ZOH) once.
// Measured on the decode workload (L2 flushed): 32.8 -> 30.7 us per token (440 CTAs
// instead of 444; bit-identical state and y); the exact-ZOH token 40.9 -> 39.1 us.
#ifndef S6_DEC_FIXED
#define S6_DEC_FIXED 1
#endif

// Bulk prefetch of `bytes` (a multiple of 16, from a 16-byte aligned address) into L2.
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
constexpr int kItems = S6_DEC_ITEMS;

template <typename Tio>
struct Lane16 {
    float4 s0, s1, a0, a1;
    typename vec4<Tio>::type b0, b1, c0, c1;
    float u, x, z, dsk;
};

// Every load of lane li's half h (state, A, B, C, u, delta, z, D) into w; with kFixed the
// channel's A, D and delta bias are the thread's own, loaded once (w.a0, w.a1, w.dsk are
// left as they are and `bias` is added to delta).
template <typename Tio, bool kFixed = false>
__device__ __forceinline__ void load_lane16(const UParams& p, uint32_t li, bool act, int h,
                                            Lane16<Tio>& w, float bias = 0.f) {
    using VT = typename vec4<Tio>::type;
    const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
    const uint32_t dim = (uint32_t)p.dim;
    const uint32_t bb = li / dim, d = li - bb * dim;
    const float* sp = p.state + (size_t)li * 16;
    const float* ap = p.A + (size_t)d * 16;
    const Tio* bp = static_cast<const Tio*>(p.B) + (size_t)bb * 16;
    const Tio* cp = static_cast<const Tio*>(p.C) + (size_t)bb * 16;
    w.s0 = act ? *reinterpret_cast<const float4*>(sp + 4 * h) : z4;
    w.s1 = act ? *reinterpret_cast<const float4*>(sp + 8 + 4 * h) : z4;
    if (!kFixed) {
        w.a0 = __ldg(reinterpret_cast<const float4*>(ap + 4 * h));
        w.a1 = __ldg(reinterpret_cast<const float4*>(ap + 8 + 4 * h));
    }
    w.b0 = *reinterpret_cast<const VT*>(bp + 4 * h);
    w.b1 = *reinterpret_cast<const VT*>(bp + 8 + 4 * h);
    w.c0 = *reinterpret_cast<const VT*>(cp + 4 * h);
    w.c1 = *reinterpret_cast<const VT*>(cp + 8 + 4 * h);
    w.u = io<Tio>::load(static_cast<const Tio*>(p.u) + li);
    w.x = io<Tio>::load(static_cast<const Tio*>(p.delta) + li) +
          (kFixed ? bias : (p.delta_bias ? p.delta_bias[d] : 0.f));
    w.z = p.z ? io<Tio>::load(static_cast<const Tio*>(p.z) + li) : 0.f;
    if (!kFixed) w.dsk = p.D ? p.D[d] : 0.f;
}

template <typename Tio, bool ZOH, bool kInv>
__device__ __forceinline__ void step_lane16(const UParams& p, uint32_t li, bool act, int h,
                                            const Lane16<Tio>& w, const float* inv);

// Persistent variant: a grid of a few CTAs per SM; each thread walks its half of lanes
// one grid stride apart, loading the next lane's data before computing the current one.
// Every thread of a warp runs the same number of rounds (the readout's shuffle needs the
// whole warp); threads past the last lane compute on placeholder data and store nothing.
template <typename Tio, bool ZOH, bool kFixed = false>
__global__ void __launch_bounds__(256) state_update16p_kernel(const UParams p) {
    const uint32_t pairs = (uint32_t)(gridDim.x * blockDim.x) / 2;
    const uint32_t gid = blockIdx.x * blockDim.x + threadIdx.x;
    const int h = gid & 1;
    const uint32_t lanes = (uint32_t)p.lanes;
    uint32_t li = gid >> 1;
    bool act = li < lanes;
    Lane16<Tio> cur, nxt;
    // kFixed: the grid stride is a multiple of dim, so every lane this thread takes is of
    // one channel: its A (and 1 / A), D and delta bias are loaded once
    float bias = 0.f, inv[8];
    if constexpr (kFixed) {
        const uint32_t d = li % (uint32_t)p.dim;
        const float* ap = p.A + (size_t)d * 16;
        cur.a0 = __ldg(reinterpret_cast<const float4*>(ap + 4 * h));
        cur.a1 = __ldg(reinterpret_cast<const float4*>(ap + 8 + 4 * h));
        cur.dsk = p.D ? p.D[d] : 0.f;
        bias = p.delta_bias ? p.delta_bias[d] : 0.f;
        nxt.a0 = cur.a0, nxt.a1 = cur.a1, nxt.dsk = cur.dsk;
        const float av[8] = {cur.a0.x, cur.a0.y, cur.a0.z, cur.a0.w,
                             cur.a1.x, cur.a1.y, cur.a1.z, cur.a1.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) inv[j] = ZOH ? rcp(av[j]) : 0.f;
    }
    load_lane16<Tio, kFixed>(p, act ? li : 0, act, h, cur, bias);
#if S6_DEC_PREFETCH
    // this CTA's lanes in a round: blockDim.x / 2 consecutive ones
    const uint32_t cta_lanes = blockDim.x / 2;
    const uint32_t cta_first = blockIdx.x * cta_lanes;
    auto prefetch_round = [&](uint32_t round) {
        const uint64_t first = (uint64_t)cta_first + (uint64_t)round * pairs;
        if (threadIdx.x != 0 || first >= lanes) return;
        const uint32_t n = (uint32_t)min((uint64_t)cta_lanes, (uint64_t)lanes - first);
        prefetch_l2(p.state + first * 16, n * 64u);
        const size_t esz = sizeof(Tio);
        // u, delta, z of these lanes: the whole 16-byte chunks inside [first, first + n)
        // rounded outwards, but never past the last whole chunk of the buffers
        const uint64_t end = (uint64_t)lanes * esz / 16 * 16;
        const uint64_t b0 = first * esz / 16 * 16;
        const uint64_t b1 = min(((first + n) * esz + 15) / 16 * 16, end);
        if (b1 <= b0) return;
        prefetch_l2(static_cast<const char*>(p.u) + b0, (uint32_t)(b1 - b0));
        prefetch_l2(static_cast<const char*>(p.delta) + b0, (uint32_t)(b1 - b0));
        if (p.z) prefetch_l2(static_cast<const char*>(p.z) + b0, (uint32_t)(b1 - b0));
    };
#pragma unroll
    for (uint32_t r = 1; r <= S6_DEC_PREFETCH; ++r) prefetch_round(r);
    uint32_t round = 0;
#endif
    while (__any_sync(0xffffffffu, act)) {
#if S6_DEC_PREFETCH
        prefetch_round(++round + S6_DEC_PREFETCH);
#endif
        const uint32_t nl = li + pairs;
        const bool nact = nl < lanes;
        load_lane16<Tio, kFixed>(p, nact ? nl : 0, nact, h, nxt, bias);
        step_lane16<Tio, ZOH, kFixed>(p, act ? li : 0, act, h, cur, inv);
        cur = nxt;
        li = nl;
        act = nact;
    }
}

template <typename Tio, bool ZOH>
__global__ void __launch_bounds__(256) state_update16_kernel(const UParams p) {
    const uint32_t pairs = (uint32_t)(gridDim.x * blockDim.x) / 2;  // lanes per item sweep
    const uint32_t gid = blockIdx.x * blockDim.x + threadIdx.x;
    const int h = gid & 1;
    Lane16<Tio> v[kItems];
    uint32_t lid[kItems];
    bool act[kItems];
#pragma unroll
    for (int it = 0; it < kItems; ++it) {
        const uint32_t lane_id = (gid >> 1) + it * pairs;
        act[it] = lane_id < (uint32_t)p.lanes;
        lid[it] = act[it] ? lane_id : 0;
        load_lane16<Tio>(p, lid[it], act[it], h, v[it]);
    }
#pragma unroll
    for (int it = 0; it < kItems; ++it) step_lane16<Tio, ZOH, false>(p, lid[it], act[it], h, v[it], nullptr);
}

// The token for one lane half: Delta, Abar, the state update, the readout, y.
template <typename Tio, bool ZOH, bool kInv = false>
__device__ __forceinline__ void step_lane16(const UParams& p, uint32_t li, bool act, int h,
                                            const Lane16<Tio>& w, const float* inv = nullptr) {
    {
        float bv[8], cv[8], t[4];
        vec4<Tio>::to_f(w.b0, t);
        bv[0] = t[0], bv[1] = t[1], bv[2] = t[2], bv[3] = t[3];
        vec4<Tio>::to_f(w.b1, t);
        bv[4] = t[0], bv[5] = t[1], bv[6] = t[2], bv[7] = t[3];
        vec4<Tio>::to_f(w.c0, t);
        cv[0] = t[0], cv[1] = t[1], cv[2] = t[2], cv[3] = t[3];
        vec4<Tio>::to_f(w.c1, t);
        cv[4] = t[0], cv[5] = t[1], cv[6] = t[2], cv[7] = t[3];
        const float dt = p.softplus ? softplus(w.x) : w.x;
        const f2 dd = pack2(dt * kLog2e, dt * kLog2e);
        const f2 qq = pack2(dt * w.u, dt * w.u);
        const float sv[8] = {w.s0.x, w.s0.y, w.s0.z, w.s0.w, w.s1.x, w.s1.y, w.s1.z, w.s1.w};
        const float av[8] = {w.a0.x, w.a0.y, w.a0.z, w.a0.w, w.a1.x, w.a1.y, w.a1.z, w.a1.w};
        float out[8];
        f2 acc = pack2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
            const f2 x = mul2(dd, pack2(av[j], av[j + 1]));
            const f2 e = ex2x2(x);
            f2 m = qq;
            if constexpr (ZOH)  // exact zero-order hold: Bbar = (e^{Delta A} - 1) / A * B
                m = zoh_weight_u2(x, e, kInv ? pack2(inv[j], inv[j + 1]) : pack2(rcp(av[j]), rcp(av[j + 1])),
                                  pack2(w.u, w.u), qq);
            const f2 hn = fma2(e, pack2(sv[j], sv[j + 1]), mul2(m, pack2(bv[j], bv[j + 1])));
            acc = fma2(pack2(cv[j], cv[j + 1]), hn, acc);
            unpack2(hn, out[j], out[j + 1]);
        }
        if (act) {
            float* wp = p.state + (size_t)li * 16;
            *reinterpret_cast<float4*>(wp + 4 * h) = make_float4(out[0], out[1], out[2], out[3]);
            *reinterpret_cast<float4*>(wp + 8 + 4 * h) = make_float4(out[4], out[5], out[6], out[7]);
        }
        float lo, hi;
        unpack2(acc, lo, hi);
        float yv = lo + hi;
        yv += __shfl_xor_sync(0xffffffffu, yv, 1);
        if (act && h == 0) {
            yv = fmaf(w.dsk, w.u, yv);
            if (p.z) yv *= silu(w.z);
            static_cast<Tio*>(p.y)[li] = io<Tio>::from_f(yv);
        }
    }
}

template <int NMAX, typename Tio, bool ZOH>
cudaError_t launch_u(const UParams& p, cudaStream_t s) {
    constexpr int G = NMAX / 4;
    const int64_t threads = p.lanes * G;
    const unsigned blocks = (unsigned)((threads + 255) / 256);
    state_update_kernel<NMAX, Tio, ZOH><<<blocks, 256, 0, s>>>(p);
    return cudaGetLastError();
}

template <typename Tio, bool ZOH>
cudaError_t launch_u_typed(const UParams& p, cudaStream_t s) {
    if (p.N == 16 && p.lanes < (1LL << 29)) {
#if S6_DEC_PERSIST
        // one wave: up to S6_DEC_PERSIST resident CTAs of 256 threads on every SM
        int dev = 0, sms = 0, occ = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e == cudaSuccess)
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, state_update16p_kernel<Tio, ZOH>,
                                                              256, 0);
        if (e != cudaSuccess) return e;
        const int64_t per_sm = std::max(1, std::min(occ, S6_DEC_PERSIST));
        const int64_t need = (2 * p.lanes + 255) / 256;
        int64_t blocks = std::min<int64_t>(need, (int64_t)sms * per_sm);
#if S6_DEC_FIXED
        // a grid whose lane stride (128 lanes per CTA) is a multiple of dim, if one within
        // a tenth of the full grid exists: every thread then keeps one channel
        for (int64_t bl = blocks; S6_DEC_FIXED && bl * 10 >= blocks * 9 && bl * 128 <= p.lanes; --bl) {
            if ((bl * 128) % p.dim == 0) {
                state_update16p_kernel<Tio, ZOH, true><<<(unsigned)bl, 256, 0, s>>>(p);
                return cudaGetLastError();
            }
        }
#endif
        state_update16p_kernel<Tio, ZOH><<<(unsigned)blocks, 256, 0, s>>>(p);
#else
        const int64_t threads = 2 * ((p.lanes + kItems - 1) / kItems);
        state_update16_kernel<Tio, ZOH><<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(p);
#endif
        return cudaGetLastError();
    }
    if (p.N <= 4) return launch_u<4, Tio, ZOH>(p, s);
    if (p.N <= 8) return launch_u<8, Tio, ZOH>(p, s);
    return launch_u<16, Tio, ZOH>(p, s);
}

}  // namespace

cudaError_t launch_state_update(const StateUpdateArgs& a, cudaStream_t stream) {
    UParams p;
    p.state = a.state;
    p.u = a.u;
    p.delta = a.delta;
    p.z = a.z;
    p.A = a.A;
    p.B = a.B;
    p.C = a.C;
    p.D = a.D;
    p.delta_bias = a.delta_bias;
    p.y = a.y;
    p.batch = a.batch;
    p.dim = a.dim;
    p.lanes = a.batch * a.dim;
    p.N = (int)a.N;
    p.softplus = a.softplus ? 1 : 0;
    p.vec = (a.N % 4 == 0) ? 1 : 0;
    const bool bf = a.io_dtype == DType::BF16;
    if (a.zoh) return bf ? launch_u_typed<__nv_bfloat16, true>(p, stream)
                         : launch_u_typed<float, true>(p, stream);
    return bf ? launch_u_typed<__nv_bfloat16, false>(p, stream) : launch_u_typed<float, false>(p, stream);
}

}  // namespace s6
