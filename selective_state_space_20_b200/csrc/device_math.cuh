// device_math.cuh -- small device helpers for the scan kernels: element
// conversion, 16-byte vectors, and the pointwise functions of the layer.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include <type_traits>

namespace mscan {

constexpr float kLog2e = 1.4426950408889634f;

// 2^x on the special-function unit (PTX ex2.approx.ftz.f32).
__device__ __forceinline__ float ex2_mufu(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// softplus(x) = ln(1 + e^x) = max(x, 0) + log1p(w),  w = e^-|x| = 2^(-|x| log2 e).
// log1p(w) = w * P(w), P the degree-8 Chebyshev interpolant of log1p(w) / w on
// [0, 1] (coefficients from fit_log1p_poly.py in this directory; relative error
// of w * P(w) in fp32 <= 2.3e-7).  One MUFU op and ten FMA-pipe ops, no branch.
// Large |x| underflows w to 0 (flush to zero), giving max(x, 0) exactly.
__device__ __forceinline__ float softplus_f(float x) {
    const float w = ex2_mufu(-fabsf(x) * kLog2e);
    float p = 5.126102362e-03f;
    p = fmaf(p, w, -2.907406539e-02f);
    p = fmaf(p, w, 7.751608640e-02f);
    p = fmaf(p, w, -1.360224783e-01f);
    p = fmaf(p, w, 1.907688081e-01f);
    p = fmaf(p, w, -2.483539879e-01f);
    p = fmaf(p, w, 3.331812024e-01f);
    p = fmaf(p, w, -4.999944568e-01f);
    p = fmaf(p, w, 9.999999404e-01f);
    return fmaf(w, p, fmaxf(x, 0.f));
}

// silu(z) = z (1 / (1 + e^-z)); for z < -88 the denominator overflows and
// the product is 0, which is the correctly rounded fp32 limit.  The same
// operations as silu2_f below, value for value, so the scalar and the packed
// forms give identical bits.
__device__ __forceinline__ float silu_f(float z) {
    return z * __fdividef(1.f, ex2_mufu(z * -kLog2e) + 1.f);
}

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

// 2^x for two values on the FMA pipe, leaving the MUFU free for other work.
// Cody-Waite split x = j + f, j = rint(x) (adding and subtracting 1.5 * 2^23
// rounds to the nearest integer), f in [-1/2, 1/2]; 2^f = Q(f) = 1 + f P(f),
// P the degree-4 Chebyshev interpolant of (2^f - 1) / f (coefficients from
// fit_exp2_poly.py in this directory; relative error of Q in fp32 <= 2.6e-7,
// the order of ex2.approx, and Q(0) = 1 exactly, so a decay near 1 carries no
// fixed bias into the many steps a slow state remembers); 2^j is added into
// the exponent field of Q(f) (the low bits of x + 1.5 * 2^23 hold j, so
// (bits << 23) is j << 23).  x is clamped to [-125, 127] so the exponent field
// cannot wrap: below -125 the result is 2^-125 instead of a denormal or 0,
// above 127 it stays finite.
__device__ __forceinline__ float2 ex2_poly2(float2 x) {
    x.x = fminf(fmaxf(x.x, -125.f), 127.f);
    x.y = fminf(fmaxf(x.y, -125.f), 127.f);
    constexpr float kRound = 12582912.f;  // 1.5 * 2^23
    const float2 t = __fadd2_rn(x, f2(kRound, kRound));
    const float2 j = __fadd2_rn(t, f2(-kRound, -kRound));
    const float2 f = __ffma2_rn(j, f2(-1.f, -1.f), x);
    float2 q = __ffma2_rn(f2(1.338130212e-03f, 1.338130212e-03f), f, f2(9.666368365e-03f, 9.666368365e-03f));
    q = __ffma2_rn(q, f, f2(5.550381169e-02f, 5.550381169e-02f));
    q = __ffma2_rn(q, f, f2(2.402234972e-01f, 2.402234972e-01f));
    q = __ffma2_rn(q, f, f2(6.931471825e-01f, 6.931471825e-01f));
    q = __ffma2_rn(q, f, f2(1.f, 1.f));  // Q(f) = 1 + f P(f)
    return f2(__uint_as_float(__float_as_uint(t.x) * 8388608u + __float_as_uint(q.x)),
              __uint_as_float(__float_as_uint(t.y) * 8388608u + __float_as_uint(q.y)));
}

// softplus on two values with the packed fp32 x2 instructions: the same
// operations as softplus_f (same rounding), at half the FMA-pipe issue.
__device__ __forceinline__ float2 softplus2_f(float2 x) {
    const float2 m = __fmul2_rn(f2(fabsf(x.x), fabsf(x.y)), f2(-kLog2e, -kLog2e));
    const float2 w = f2(ex2_mufu(m.x), ex2_mufu(m.y));
    float2 p = f2(5.126102362e-03f, 5.126102362e-03f);
    p = __ffma2_rn(p, w, f2(-2.907406539e-02f, -2.907406539e-02f));
    p = __ffma2_rn(p, w, f2(7.751608640e-02f, 7.751608640e-02f));
    p = __ffma2_rn(p, w, f2(-1.360224783e-01f, -1.360224783e-01f));
    p = __ffma2_rn(p, w, f2(1.907688081e-01f, 1.907688081e-01f));
    p = __ffma2_rn(p, w, f2(-2.483539879e-01f, -2.483539879e-01f));
    p = __ffma2_rn(p, w, f2(3.331812024e-01f, 3.331812024e-01f));
    p = __ffma2_rn(p, w, f2(-4.999944568e-01f, -4.999944568e-01f));
    p = __ffma2_rn(p, w, f2(9.999999404e-01f, 9.999999404e-01f));
    return __ffma2_rn(w, p, f2(fmaxf(x.x, 0.f), fmaxf(x.y, 0.f)));
}

// silu on two values: z * (1 / (1 + e^-z)), the exponent scaling, the
// "1 +" and the final product on the packed instructions.
__device__ __forceinline__ float2 silu2_f(float2 z) {
    const float2 m = __fmul2_rn(z, f2(-kLog2e, -kLog2e));
    const float2 d = __fadd2_rn(f2(ex2_mufu(m.x), ex2_mufu(m.y)), f2(1.f, 1.f));
    return __fmul2_rn(z, f2(__fdividef(1.f, d.x), __fdividef(1.f, d.y)));
}

// ------------------------------------------------------ fp32-tolerance math
// fp32 activations are held to a 1e-4 relative error, bf16 ones to 2e-2.  At
// 1e-4 the decay is the one thing the special-function unit cannot give: a
// state remembers ~1 / (1 - Abar) steps, and a relative error e in Abar that
// keeps its sign over those steps becomes an error of e / (1 - Abar) in h --
// ex2.approx's bias of a few 2^-24 grows to ~1e-4 and beyond over a few
// hundred steps, where a correctly rounded decay stays near 5e-5.  So with
// fp32 activations the kernels advance a state whose decay is near 1 as
// h + ((Abar - 1) h + b), Abar - 1 from expm1_poly below: its error is
// relative to the small change of h per step, not to h, and carries no bias.
// A decay far from 1 (|delta A| > 1, Abar < e^-1) is used as Abar itself from
// the MUFU exponential: such a state forgets within a step or two, so no
// bias can build up, and fma(Abar, h, b) keeps the relative accuracy of a
// tiny Abar h that the difference form would lose.  bf16 activations keep
// the single MUFU op per decay.

// e^x - 1 = x + x^2 P(x) for |x| <= 1, P the degree-6 Chebyshev interpolant of
// (e^x - 1 - x) / x^2 (coefficients from fit_expm1_poly.py in this directory;
// relative error <= 1.6e-7 in fp32 however close x is to 0).
__device__ __forceinline__ float expm1_poly(float x) {
    float p = 2.528843470e-05f;
    p = fmaf(p, x, 2.032904158e-04f);
    p = fmaf(p, x, 1.388644800e-03f);
    p = fmaf(p, x, 8.330886252e-03f);
    p = fmaf(p, x, 4.166669771e-02f);
    p = fmaf(p, x, 1.666669697e-01f);
    p = fmaf(p, x, 5.000000000e-01f);
    return fmaf(x * x, p, x);
}

// softplus with CUDA's full-precision expf and log1pf (errors of an ulp or
// two); the one-MUFU-op softplus_f rounds its exponent x log2 e to fp32 and
// reaches 8.5e-7 relative error for very negative inputs.
__device__ __forceinline__ float softplus_precise(float x) {
    return fmaxf(x, 0.f) + log1pf(expf(-fabsf(x)));
}

// One state's step h <- Abar h + b with Abar = e^x, x = delta * A * kScale.
//   ACC = false (bf16 activations): A is pre-scaled by log2 e and Abar comes
//     from one ex2 on the MUFU; h <- fma(Abar, h, b).
//   ACC = true (fp32 activations): A is used as is; for |x| <= 1
//     h <- h + fma(e^x - 1, h, b), else h <- fma(e^x, h, b).  The kernels keep
//     such a state in fp64 (the double overload): in fp32, the rounding of h
//     at every step, relative to the largest |h| the state reaches, adds up
//     over the ~1 / (1 - Abar) steps it remembers to ~1e-4 of the typical
//     magnitude -- the fp32 bar itself -- for a state that ends near zero.
//     x, e^x - 1 and b stay fp32 (each rounded once per step, without bias).
template <bool ACC>
struct Decay {
    static constexpr float kScale = ACC ? 1.f : kLog2e;
    // the state's type: fp64 for fp32 activations
    using H = typename std::conditional<ACC, double, float>::type;
    __device__ __forceinline__ static bool near_one(float x) { return fabsf(x) <= 1.f; }
    __device__ __forceinline__ static float step(float x, float h, float b) {
        if (ACC) return near_one(x) ? h + fmaf(expm1_poly(x), h, b) : fmaf(__expf(x), h, b);
        return fmaf(ex2_mufu(x), h, b);
    }
    __device__ __forceinline__ static double step(float x, double h, float b) {
        return near_one(x) ? h + fma((double)expm1_poly(x), h, (double)b) : fma((double)__expf(x), h, (double)b);
    }
    __device__ __forceinline__ static float2 step2(float2 x, float2 h, float2 b) {
        if (ACC) return f2(step(x.x, h.x, b.x), step(x.y, h.y, b.y));
        return __ffma2_rn(f2(ex2_mufu(x.x), ex2_mufu(x.y)), h, b);
    }
    // v * Abar (the adjoint's decay in the backward pass)
    __device__ __forceinline__ static float scale(float x, float v) {
        if (ACC) return near_one(x) ? fmaf(expm1_poly(x), v, v) : __expf(x) * v;
        return ex2_mufu(x) * v;
    }
    // Abar itself
    __device__ __forceinline__ static float abar(float x) {
        if (ACC) return near_one(x) ? 1.f + expm1_poly(x) : __expf(x);
        return ex2_mufu(x);
    }
    // softplus of the step's raw value
    __device__ __forceinline__ static float softplus(float x) {
        if (ACC) return softplus_precise(x);
        return softplus_f(x);
    }
    __device__ __forceinline__ static float2 softplus2(float2 x) {
        if (ACC) return f2(softplus_precise(x.x), softplus_precise(x.y));
        return softplus2_f(x);
    }
};

// ---------------------------------------------------------------- elements
template <typename T> struct Elem;

template <> struct Elem<float> {
    static constexpr int kVec = 4;  // elements per 16 bytes
    __device__ __forceinline__ static float load(const float *p) { return __ldg(p); }  // global only
    __device__ __forceinline__ static float to_f(float v) { return v; }
    __device__ __forceinline__ static void store(float *p, float v) { *p = v; }
    __device__ __forceinline__ static void unpack(const uint4 &w, float *f) {
        f[0] = __uint_as_float(w.x); f[1] = __uint_as_float(w.y);
        f[2] = __uint_as_float(w.z); f[3] = __uint_as_float(w.w);
    }
    __device__ __forceinline__ static uint4 pack(const float *f) {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]),
                          __float_as_uint(f[2]), __float_as_uint(f[3]));
    }
};

template <> struct Elem<__nv_bfloat16> {
    static constexpr int kVec = 8;
    __device__ __forceinline__ static float load(const __nv_bfloat16 *p) {  // global only
        unsigned short s = __ldg(reinterpret_cast<const unsigned short *>(p));
        return __uint_as_float(static_cast<uint32_t>(s) << 16);
    }
    __device__ __forceinline__ static float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
    __device__ __forceinline__ static void store(__nv_bfloat16 *p, float v) {
        *p = __float2bfloat16_rn(v);
    }
    // bf16 -> fp32 is exact: the bf16 bits are the high half of the fp32 bits.
    __device__ __forceinline__ static void unpack2(uint32_t w, float &lo, float &hi) {
        lo = __uint_as_float(w << 16);
        hi = __uint_as_float(w & 0xffff0000u);
    }
    __device__ __forceinline__ static void unpack(const uint4 &w, float *f) {
        unpack2(w.x, f[0], f[1]); unpack2(w.y, f[2], f[3]);
        unpack2(w.z, f[4], f[5]); unpack2(w.w, f[6], f[7]);
    }
    __device__ __forceinline__ static uint32_t pack2(float lo, float hi) {
        __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // round to nearest even
        return *reinterpret_cast<uint32_t *>(&v);
    }
    __device__ __forceinline__ static uint4 pack(const float *f) {
        return make_uint4(pack2(f[0], f[1]), pack2(f[2], f[3]),
                          pack2(f[4], f[5]), pack2(f[6], f[7]));
    }
};

__device__ __forceinline__ uint4 ldg16(const void *p) {
    return __ldg(reinterpret_cast<const uint4 *>(p));
}

// Streaming 16-byte load: read once, do not keep in L1.
__device__ __forceinline__ uint4 ldg16_stream(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// Streaming 16-byte store (evict-first in L2: the output is not re-read).
__device__ __forceinline__ void stg16_stream(void *p, const uint4 &v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};"
                 :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

}  // namespace mscan
