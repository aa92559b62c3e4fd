// s6_device.cuh -- small device helpers shared by the sm_100a selective-scan kernels.
//
// The SFU (MUFU) instructions are issued directly through inline PTX so the
// instruction mix is explicit: ex2.approx / lg2.approx / rcp.approx are single
// hardware instructions with documented error bounds (PTX ISA: relative error of
// ex2.approx.f32 about 2^-22, lg2.approx.f32 absolute error about 2^-22, rcp.approx
// within 1 ulp).  No CUDA math-library routine is reproduced here.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace s6 {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float lg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float rcp(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// log1p(e) / e on [0, 1] as a degree-7 polynomial (Remez fit for relative error made
// for this library: 1.9e-7 in exact arithmetic, 3.3e-7 with fp32 Horner steps).
__device__ __forceinline__ float log1p_over_x(float e) {
    float q = fmaf(-8.5392082e-3f, e, 4.4089634e-2f);
    q = fmaf(q, e, -1.0768171e-1f);
    q = fmaf(q, e, 1.7745242e-1f);
    q = fmaf(q, e, -2.4495463e-1f);
    q = fmaf(q, e, 3.3275479e-1f);
    q = fmaf(q, e, -4.9997404e-1f);
    return fmaf(q, e, 9.9999982e-1f);
}

// softplus(x) = log(1 + e^x) = max(x, 0) + log1p(e^-|x|): one SFU exponential and a
// polynomial, no cancellation for either sign of x (e^-|x| lies in (0, 1]).
__device__ __forceinline__ float softplus(float x) {
    const float e = ex2(-fabsf(x) * kLog2e);
    return fmaxf(x, 0.f) + e * log1p_over_x(e);
}

// z * sigmoid(z) = z / (1 + e^-z); e^-z = +inf for very negative z gives z * 0.
__device__ __forceinline__ float silu(float z) { return z * rcp(1.f + ex2(-z * kLog2e)); }

// z * sigmoid(z) for four values with one reciprocal between them (Montgomery's batch
// inversion): d_q = 1 + 2^(-z_q log2 e), r = 1 / (d0 d1 d2 d3), then 1 / d0 = r d1 (d2 d3)
// and so on.  The exponent is capped at 31, so every d_q <= 2^31 + 1 and their product
// stays far from overflow; below z = -21.4 the cap leaves sigmoid(z) at 2^-31 instead of
// e^z, an absolute change under 5e-10 in z * sigmoid(z) / |z|.  The products and the
// reciprocal add about four rounding steps to the single-division form.
__device__ __forceinline__ void silu4(const float (&z)[4], float (&out)[4]) {
    float d[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) d[q] = 1.f + ex2(fminf(-z[q] * kLog2e, 31.f));
    const float p01 = d[0] * d[1], p23 = d[2] * d[3];
    const float r = rcp(p01 * p23);
    const float r01 = r * p23, r23 = r * p01;
    out[0] = z[0] * (r01 * d[1]);
    out[1] = z[1] * (r01 * d[0]);
    out[2] = z[2] * (r23 * d[3]);
    out[3] = z[3] * (r23 * d[2]);
}

template <typename T> struct io;
template <> struct io<float> {
    __device__ __forceinline__ static float load(const float* p) { return *p; }
    __device__ __forceinline__ static float to_f(float v) { return v; }
    __device__ __forceinline__ static float from_f(float v) { return v; }
};
template <> struct io<__nv_bfloat16> {
    __device__ __forceinline__ static float load(const __nv_bfloat16* p) {
        return __bfloat162float(*p);
    }
    __device__ __forceinline__ static float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
    __device__ __forceinline__ static __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};

// 16-byte global -> shared async copy (Ampere+ LDGSTS); src_bytes = 0 zero-fills.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src, int src_bytes) {
    uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem_src),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

}  // namespace s6

namespace s6 {

// Two fp32 lanes in one 64-bit register pair, for the packed sm_100 FP32 instructions
// (add/mul/fma .f32x2: one issue slot for two operations).
struct f2 {
    unsigned long long v;
};

__device__ __forceinline__ f2 pack2(float lo, float hi) {
    f2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r.v) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void unpack2(f2 x, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(x.v));
}
__device__ __forceinline__ f2 fma2(f2 a, f2 b, f2 c) {
    f2 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d.v) : "l"(a.v), "l"(b.v), "l"(c.v));
    return d;
}
__device__ __forceinline__ f2 mul2(f2 a, f2 b) {
    f2 d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d.v) : "l"(a.v), "l"(b.v));
    return d;
}
__device__ __forceinline__ f2 add2(f2 a, f2 b) {
    f2 d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d.v) : "l"(a.v), "l"(b.v));
    return d;
}
__device__ __forceinline__ f2 sub2(f2 a, f2 b) {
    f2 d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d.v) : "l"(a.v), "l"(b.v));
    return d;
}

// 2^x on both halves using only the FMA and integer pipes, so part of the exponentials
// can bypass the SFU.  Cody-Waite style split in base 2: x is clamped to [-126, 127],
// j = rint(x) is obtained by adding and subtracting 1.5 * 2^23 (which also leaves j in
// the low mantissa bits of the sum), f = x - j lies in [-1/2, 1/2], 2^f comes from a
// degree-5 polynomial fitted here by the Remez exchange for minimum relative error on
// [-1/2, 1/2] (max 7.5e-8 in exact arithmetic, 2.1e-7 with fp32 Horner steps, about
// the SFU's ex2.approx bound), and 2^j is added into the exponent field as j << 23.
__device__ __forceinline__ f2 exp2_fma2(f2 x) {
    constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
    float x0, x1;
    unpack2(x, x0, x1);
    x0 = fminf(fmaxf(x0, -126.f), 127.f);
    x1 = fminf(fmaxf(x1, -126.f), 127.f);
    const f2 xc = pack2(x0, x1);
    const f2 t = add2(xc, pack2(kRound, kRound));
    const f2 f = sub2(xc, sub2(t, pack2(kRound, kRound)));
    f2 p = fma2(pack2(1.3276472e-3f, 1.3276472e-3f), f, pack2(9.6755410e-3f, 9.6755410e-3f));
    p = fma2(p, f, pack2(5.5507131e-2f, 5.5507131e-2f));
    p = fma2(p, f, pack2(2.4022120e-1f, 2.4022120e-1f));
    p = fma2(p, f, pack2(6.9314694e-1f, 6.9314694e-1f));
    p = fma2(p, f, pack2(1.0000001f, 1.0000001f));
    float t0, t1, p0, p1;
    unpack2(t, t0, t1);
    unpack2(p, p0, p1);
    return pack2(__uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23)),
                 __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23)));
}

// Exact zero-order-hold input weight for a pair of states (Mamba, "Method": Bbar =
// (Delta A)^-1 (exp(Delta A) - I) Delta B, per diagonal state w = (e^{Delta A} - 1) / A).
// Inputs: x = Delta A log2(e) (so Abar = e = 2^x), e, 1/A, uu = (u, u), qq = (Delta u,
// Delta u).  Returns m = w u, the factor of B in the state update.
//   |Delta A| >= 1/16: m = u (e - 1) / A  (|e - 1| >= 0.0606 there, so an error of a few
//                      1e-7 in e costs under 5e-6 relative);
//   |Delta A| <  1/16: m = Delta u phi(Delta A), phi(y) = expm1(y) / y = sum_k y^k / (k+1)!
//                      truncated after y^3 (the first dropped term, y^4 / 120, is below
//                      1.3e-7 relative), evaluated in x with coefficients ln2^k / (k+1)!;
//                      this avoids the cancellation of e - 1 as Delta A -> 0 (and covers
//                      A = 0, where 1/A is infinite).
__device__ __forceinline__ f2 zoh_weight_u2(f2 x, f2 e, f2 inv_a, f2 uu, f2 qq) {
    f2 p = fma2(pack2(1.3876027e-02f, 1.3876027e-02f), x, pack2(8.0075502e-02f, 8.0075502e-02f));
    p = fma2(p, x, pack2(3.4657359e-01f, 3.4657359e-01f));
    p = fma2(p, x, pack2(1.0f, 1.0f));
    const f2 small = mul2(qq, p);
    const f2 large = mul2(uu, mul2(add2(e, pack2(-1.f, -1.f)), inv_a));
    float x0, x1, s0, s1, l0, l1;
    unpack2(x, x0, x1);
    unpack2(small, s0, s1);
    unpack2(large, l0, l1);
    constexpr float kTau = 0.09016844f;  // |Delta A| = 1/16 in log2 units
    return pack2(fabsf(x0) < kTau ? s0 : l0, fabsf(x1) < kTau ? s1 : l1);
}

// softplus on four values at once, the polynomial on packed pairs.
__device__ __forceinline__ void softplus4(const float (&x)[4], float (&out)[4]) {
    float e[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) e[q] = ex2(-fabsf(x[q]) * kLog2e);
#pragma unroll
    for (int q = 0; q < 4; q += 2) {
        const f2 ee = pack2(e[q], e[q + 1]);
        f2 p = fma2(pack2(-8.5392082e-3f, -8.5392082e-3f), ee, pack2(4.4089634e-2f, 4.4089634e-2f));
        p = fma2(p, ee, pack2(-1.0768171e-1f, -1.0768171e-1f));
        p = fma2(p, ee, pack2(1.7745242e-1f, 1.7745242e-1f));
        p = fma2(p, ee, pack2(-2.4495463e-1f, -2.4495463e-1f));
        p = fma2(p, ee, pack2(3.3275479e-1f, 3.3275479e-1f));
        p = fma2(p, ee, pack2(-4.9997404e-1f, -4.9997404e-1f));
        p = fma2(p, ee, pack2(9.9999982e-1f, 9.9999982e-1f));
        const f2 r = fma2(ee, p, pack2(fmaxf(x[q], 0.f), fmaxf(x[q + 1], 0.f)));
        unpack2(r, out[q], out[q + 1]);
    }
}

// A bf16 pair (element 0 in the low half of the word) widened exactly to an fp32 pair.
__device__ __forceinline__ f2 bf16pair(uint32_t w) {
    return pack2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
// 2^x on both halves (two SFU operations).
__device__ __forceinline__ f2 ex2x2(f2 x) {
    float lo, hi;
    unpack2(x, lo, hi);
    return pack2(ex2(lo), ex2(hi));
}

// Four consecutive input elements of type T as one aligned vector load.
template <typename T> struct vec4;
template <> struct vec4<float> {
    using type = float4;
    __device__ __forceinline__ static void to_f(const type& v, float (&o)[4]) {
        o[0] = v.x, o[1] = v.y, o[2] = v.z, o[3] = v.w;
    }
};
template <> struct vec4<__nv_bfloat16> {
    using type = uint2;  // 4 x bf16
    __device__ __forceinline__ static void to_f(const type& v, float (&o)[4]) {
        o[0] = __uint_as_float(v.x << 16);
        o[1] = __uint_as_float(v.x & 0xffff0000u);
        o[2] = __uint_as_float(v.y << 16);
        o[3] = __uint_as_float(v.y & 0xffff0000u);
    }
};

}  // namespace s6

// ---- Tensor-memory-accelerator (TMA) bulk copies and mbarriers (sm_90+ PTX) ----
namespace s6 {

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

// Make barrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Order this thread's earlier generic-proxy shared-memory accesses before later
// async-proxy (TMA) accesses of the same memory.
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

// Plain arrival (release semantics at CTA scope): the arriving thread's earlier
// shared-memory writes, and those it has synchronised with, become visible to a thread
// whose wait observes the phase completing.
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Bounded wait for phase `parity` of `bar`: gives up after `limit_cycles` SM clocks
// (about a second) and returns false, so a lost transfer cannot hang the GPU.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  long long limit_cycles) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long start = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - start > limit_cycles) return false;
    }
    return true;
}

// 3-D tiled bulk tensor load global -> shared, completing on `bar` (transaction bytes).
// c0 is the innermost coordinate; out-of-range elements are filled with zeros.
__device__ __forceinline__ void tma_load_3d(void* dst, const void* tmap, int c0, int c1, int c2,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(bar))
        : "memory");
}

// 3-D tiled bulk tensor store shared -> global; elements outside the tensor are skipped.
__device__ __forceinline__ void tma_store_3d(const void* tmap, const void* src, int c0, int c1,
                                             int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(tmap)),
        "r"(smem_addr(src)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}
__device__ __forceinline__ void tma_store_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until at most N committed store groups still read shared memory.
template <int N>
__device__ __forceinline__ void tma_store_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until every committed store group has completed.
__device__ __forceinline__ void tma_store_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

}  // namespace s6
