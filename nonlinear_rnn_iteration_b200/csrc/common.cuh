// common.cuh -- device helpers shared by the forward and backward kernels:
// vectorised row loads/stores, the global timer for bounded waits, and the
// activation functions.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace pararnn {

// ---- workspace header (first 256 bytes of every workspace) -------------
// word 0: status bits, word 1: tile ticket counter.  The rest is padding.
constexpr unsigned kStatusNonFinite = 1u;
constexpr unsigned kStatusTimeout = 2u;
constexpr size_t kHeaderBytes = 256;

// ---- element loads -------------------------------------------------------

template <typename T>
struct PxTraits;

template <>
struct PxTraits<float> {
    static __device__ __forceinline__ float cvt(float x) { return x; }
};
template <>
struct PxTraits<__nv_bfloat16> {
    static __device__ __forceinline__ float cvt(__nv_bfloat16 x) { return __bfloat162float(x); }
};

// Load V consecutive values starting at p (p is V-element aligned when V > 1).
// Streaming data: read once, so the load asks L1 not to keep the line.
template <int V>
__device__ __forceinline__ void load_row(const float* p, float (&out)[V]) {
    if constexpr (V == 4) {
        float4 v;
        asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
                     : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                     : "l"(p));
        out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
    } else if constexpr (V == 2) {
        float2 v;
        asm volatile("ld.global.nc.L1::no_allocate.v2.f32 {%0,%1}, [%2];" : "=f"(v.x), "=f"(v.y) : "l"(p));
        out[0] = v.x; out[1] = v.y;
    } else {
#pragma unroll
        for (int i = 0; i < V; ++i) out[i] = __ldg(p + i);
    }
}

template <int V>
__device__ __forceinline__ void load_row(const __nv_bfloat16* p, float (&out)[V]) {
    if constexpr (V == 4) {
        uint2 v;
        asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
        out[0] = __uint_as_float(v.x << 16);
        out[1] = __uint_as_float(v.x & 0xffff0000u);
        out[2] = __uint_as_float(v.y << 16);
        out[3] = __uint_as_float(v.y & 0xffff0000u);
    } else if constexpr (V == 2) {
        unsigned v;
        asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
        out[0] = __uint_as_float(v << 16);
        out[1] = __uint_as_float(v & 0xffff0000u);
    } else {
#pragma unroll
        for (int i = 0; i < V; ++i) out[i] = __bfloat162float(p[i]);
    }
}

// Shared-memory row reads of V consecutive values (one vector access per lane).
template <int V>
__device__ __forceinline__ void lds_row(const float* p, float (&out)[V]) {
    if constexpr (V == 4) {
        const float4 v = *reinterpret_cast<const float4*>(p);
        out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
    } else if constexpr (V == 2) {
        const float2 v = *reinterpret_cast<const float2*>(p);
        out[0] = v.x; out[1] = v.y;
    } else {
#pragma unroll
        for (int i = 0; i < V; ++i) out[i] = p[i];
    }
}

template <int V>
__device__ __forceinline__ void lds_row(const __nv_bfloat16* p, float (&out)[V]) {
    if constexpr (V == 4) {
        const uint2 v = *reinterpret_cast<const uint2*>(p);
        out[0] = __uint_as_float(v.x << 16);
        out[1] = __uint_as_float(v.x & 0xffff0000u);
        out[2] = __uint_as_float(v.y << 16);
        out[3] = __uint_as_float(v.y & 0xffff0000u);
    } else if constexpr (V == 2) {
        const unsigned v = *reinterpret_cast<const unsigned*>(p);
        out[0] = __uint_as_float(v << 16);
        out[1] = __uint_as_float(v & 0xffff0000u);
    } else {
#pragma unroll
        for (int i = 0; i < V; ++i) out[i] = __bfloat162float(p[i]);
    }
}

template <int V>
__device__ __forceinline__ void store_row(float* p, const float (&v)[V]) {
    if constexpr (V == 4) {
        *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    } else if constexpr (V == 2) {
        *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
    } else {
#pragma unroll
        for (int i = 0; i < V; ++i) p[i] = v[i];
    }
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Block-wide barrier usable from warp-uniform divergent code paths (the
// compute warps and the scan warp arrive at it from different code); it
// orders shared- and global-memory accesses like __syncthreads.
__device__ __forceinline__ void block_sync() { asm volatile("bar.sync 0;" ::: "memory"); }

// ---- numerics --------------------------------------------------------------

// e^x = 2^(x log2 e) with the PTX approximate base-2 exponential, and the
// PTX approximate reciprocal (both flush subnormal results to zero; the
// state and gates here never need them).  e^x overflowing to +inf and
// 1/inf = 0 give the saturated limits below exactly.
__device__ __forceinline__ float exp2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
constexpr float kLog2e = 1.4426950408889634f;

// sigma(x) = 1 / (1 + e^{-x})
__device__ __forceinline__ float sigmoid_f(float x) { return rcp_approx(1.0f + exp2_approx(x * -kLog2e)); }

// tanh from its definition, tanh x = 1 - 2 / (e^{2x} + 1), with the odd
// Taylor series x - x^3/3 + 2x^5/15 below |x| = 1/16, where the subtraction
// would cancel (the first omitted term, 17x^7/315, is below 4e-9 of tanh
// there, far under float32 rounding).  e^{2x} overflowing to +inf gives
// exactly 1, underflowing to 0 exactly -1.
__device__ __forceinline__ float tanh_f(float x) {
    const float big = __fmaf_rn(-2.0f, rcp_approx(exp2_approx(x * (2.0f * kLog2e)) + 1.0f), 1.0f);
    const float x2 = x * x;
    const float poly = x * __fmaf_rn(x2, __fmaf_rn(x2, 2.0f / 15.0f, -1.0f / 3.0f), 1.0f);
    return fabsf(x) < 0.0625f ? poly : big;
}

// ---- gates that share one reciprocal ---------------------------------------
// Two gates that do not depend on one another need the reciprocals of two
// denominators 1 + e^u at once.  Simultaneous inversion (P. L. Montgomery,
// "Speeding the Pollard and elliptic curve methods of factorization", Math.
// Comp. 48 (1987)) forms both from one reciprocal of their product,
// 1/a = b (1/(ab)) and 1/b = a (1/(ab)), trading a reciprocal on the
// special-function unit (which also feeds the MIO queue) for two multiplies
// on the FMA pipe.  Each exponent is capped at 2^62 so that the product stays
// below 2^125 and its reciprocal is a normal float: a sigmoid below 2^-62
// (an argument below about -43) is returned as 2^-62, less than 2.2e-19 from
// its exact value, and a tanh whose exponent is capped (an argument above
// about 21.5) still rounds to exactly 1.  The cap is taken with min.NaN, so a
// NaN argument stays NaN.
constexpr float kExpCap = 62.0f;

__device__ __forceinline__ float min_nan(float a, float b) {
    float d;
    asm("min.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
    return d;
}
// 1 + e^{-x}, so sigma(x) = 1 / sig_den(x)
__device__ __forceinline__ float sig_den(float x) { return 1.0f + exp2_approx(min_nan(x * -kLog2e, kExpCap)); }
// 1 + e^{2x}, so tanh(x) = 1 - 2 / tanh_den(x)
__device__ __forceinline__ float tanh_den(float x) {
    return exp2_approx(min_nan(x * (2.0f * kLog2e), kExpCap)) + 1.0f;
}
// tanh(x) from inv = 1 / tanh_den(x), with tanh_f's Taylor branch near 0
__device__ __forceinline__ float tanh_from_inv(float x, float inv) {
    const float big = __fmaf_rn(-2.0f, inv, 1.0f);
    const float x2 = x * x;
    const float poly = x * __fmaf_rn(x2, __fmaf_rn(x2, 2.0f / 15.0f, -1.0f / 3.0f), 1.0f);
    return fabsf(x) < 0.0625f ? poly : big;
}
// 1/a and 1/b from one reciprocal
__device__ __forceinline__ void inv_pair(float a, float b, float& ia, float& ib) {
    const float q = rcp_approx(a * b);
    ia = b * q;
    ib = a * q;
}

// ---- packed pairs: two channels per instruction ----------------------------
// sm_100a's fma / add / sub / mul .rn.f32x2 operate on two floats held in a
// register pair and round each half exactly like the scalar instruction, so a
// computation written on pairs gives the same bits as the same computation on
// each channel alone.  There is no packed negation or min/max: signs are
// folded into constants instead.
struct f2 {
    float x, y;
};

__device__ __forceinline__ f2 splat2(float a) { return f2{a, a}; }

__device__ __forceinline__ f2 fma2(f2 a, f2 b, f2 c) {
    f2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ f2 mul2(f2 a, f2 b) {
    f2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ f2 add2(f2 a, f2 b) {
    f2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ f2 sub2(f2 a, f2 b) {
    f2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ f2 ex2_2(f2 a) { return f2{exp2_approx(a.x), exp2_approx(a.y)}; }
__device__ __forceinline__ f2 rcp_2(f2 a) { return f2{rcp_approx(a.x), rcp_approx(a.y)}; }

// -sigma(x) = 1 / (-1 - e^{-x}): the same rounding as sigmoid_f, negated
// (a reciprocal of a negated value is the exact negation), which saves the
// packed negation the callers would otherwise need
__device__ __forceinline__ f2 neg_sigmoid2(f2 x) {
    return rcp_2(sub2(splat2(-1.0f), ex2_2(mul2(x, splat2(-kLog2e)))));
}
__device__ __forceinline__ f2 sigmoid2(f2 x) {
    return rcp_2(add2(ex2_2(mul2(x, splat2(-kLog2e))), splat2(1.0f)));
}
// tanh_f on a pair, the same operations in the same order
__device__ __forceinline__ f2 tanh2(f2 x) {
    const f2 big = fma2(splat2(-2.0f), rcp_2(add2(ex2_2(mul2(x, splat2(2.0f * kLog2e))), splat2(1.0f))),
                        splat2(1.0f));
    const f2 x2 = mul2(x, x);
    const f2 poly = mul2(x, fma2(x2, fma2(x2, splat2(2.0f / 15.0f), splat2(-1.0f / 3.0f)), splat2(1.0f)));
    return f2{fabsf(x.x) < 0.0625f ? poly.x : big.x, fabsf(x.y) < 0.0625f ? poly.y : big.y};
}

// the shared-reciprocal helpers above on pairs, with the same operations in
// the same order, so that each half gives the scalar helper's bits
__device__ __forceinline__ f2 min_nan2(f2 a, float b) { return f2{min_nan(a.x, b), min_nan(a.y, b)}; }
__device__ __forceinline__ f2 sig_den2(f2 x) {
    return add2(splat2(1.0f), ex2_2(min_nan2(mul2(x, splat2(-kLog2e)), kExpCap)));
}
// -(1 + e^{-x}): sig_den negated exactly (round-to-nearest is symmetric in
// sign, and so are products and reciprocals), for the sign-free algebra of
// the GRU, whose callers want -sigma and have no packed negation
__device__ __forceinline__ f2 neg_sig_den2(f2 x) {
    return sub2(splat2(-1.0f), ex2_2(min_nan2(mul2(x, splat2(-kLog2e)), kExpCap)));
}
__device__ __forceinline__ f2 tanh_den2(f2 x) {
    return add2(ex2_2(min_nan2(mul2(x, splat2(2.0f * kLog2e)), kExpCap)), splat2(1.0f));
}
__device__ __forceinline__ f2 tanh2_from_inv(f2 x, f2 inv) {
    const f2 big = fma2(splat2(-2.0f), inv, splat2(1.0f));
    const f2 x2 = mul2(x, x);
    const f2 poly = mul2(x, fma2(x2, fma2(x2, splat2(2.0f / 15.0f), splat2(-1.0f / 3.0f)), splat2(1.0f)));
    return f2{fabsf(x.x) < 0.0625f ? poly.x : big.x, fabsf(x.y) < 0.0625f ? poly.y : big.y};
}
__device__ __forceinline__ void inv_pair2(f2 a, f2 b, f2& ia, f2& ib) {
    const f2 q = rcp_2(mul2(a, b));
    ia = mul2(b, q);
    ib = mul2(a, q);
}

// max that keeps a NaN (so a non-finite residual is reported, not hidden)
__device__ __forceinline__ float nanmax_f(float a, float b) { return (a != a || a > b) ? a : b; }

// Non-negative floats order like their bit patterns, and a NaN's bits sort
// above +Inf, so an integer atomicMax on the bits is a deterministic max.
__device__ __forceinline__ void atomic_max_nonneg(float* addr, float v) {
    atomicMax(reinterpret_cast<unsigned*>(addr), __float_as_uint(fabsf(v)) & 0x7fffffffu);
}

}  // namespace pararnn
