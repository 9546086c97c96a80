// mea_math.cuh -- fp32 device arithmetic of the activation family.
//
// Each activation is a struct with the forward value f(x) and the backward
// product dy * f'(x), both recomputed from x alone (the save-input-only
// contract of "Memory efficient Swish", sections "How is the memory efficient
// version Swish implemented?" and "What makes this implementation save GPU
// memory?").  The family is the one costed in "What activations cost, in
// memory and in arithmetic" (problem B07, GIVEN); definitions are standard.
//
// Sigmoid primitive.  Sigmoid(v) = 1 / (1 + E) with E = e^-v = 2^t,
// t = -v log2(e), evaluated with the PTX instructions ex2.approx.ftz.f32 and
// rcp.approx.ftz.f32 (two MUFU operations).  1 - Sigmoid(v) is taken as
// E * s where v > 0 and as 1 - s where v <= 0, so neither branch cancels.
//
// Precision modes (template flag P):
//  - P = false (bf16 storage): t is one fp32 product.  Its rounding moves E
//    by at most |t| 2^-24 ln 2 relative (< 2^-12 for |t| <= 126), far below
//    half a bf16 ulp.
//  - P = true (fp32 storage): t = x * (c_hi + c_lo) is carried as a
//    float-float pair and E is corrected by (1 + t_lo ln 2), which removes
//    the argument-rounding error that would otherwise reach ~1e-5 at
//    |t| ~ 126.  GELU-tanh forms its cubic argument in fp64 for the same
//    reason.
//
// Deep tails.  Where E > 2^126 the sigmoid itself would be subnormal and the
// .ftz instructions would flush it, although x * Sigmoid(alpha x) is still a
// normal number for alpha x down to about -103.  Those elements (flagged by
// the main path through `tail`) are recomputed from 2^(64 - t), which stays
// normal, and the result is scaled by 2^-64 at the end.
#pragma once

#include <stdint.h>

namespace mea {

constexpr float kLn2f = 0.693147180559945309f;
constexpr float kLog2eHi = 1.44269502162933349609375f;      // fp32(log2 e)
constexpr float kLog2eLo = 1.9259629911266174681e-08f;      // log2 e - kLog2eHi
constexpr double kLog2eD = 1.4426950408889634074;
constexpr float kTailT = 124.0f;       // main path used while t <= this (margin below 126)
constexpr float kCorrMax = 192.0f;     // |t| beyond which E is 0 or inf anyway
constexpr float kTwoM64 = 5.42101086242752217e-20f;          // 2^-64
constexpr float kBig = 3.0e38f;

__device__ __forceinline__ float ex2_ftz(float t)
{
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(t));
    return r;
}

// The MUFU hyperbolic tangent (tanh.approx.f32, sm_75 and later; the PTX ISA
// states a maximum relative error of about 2^-11, a quarter of a bf16 ulp or
// less).  Used for bf16 storage only.
__device__ __forceinline__ float tanh_mufu(float x)
{
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp_ftz(float v)
{
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}

// Two fp32 values in one 64-bit register pair, for the packed .f32x2
// arithmetic of sm_100 (one instruction, two IEEE results with the same
// rounding as the scalar instruction).  Used where a kernel is bound by
// instruction issue rather than by memory.
struct F2 {
    unsigned long long v;
};
__device__ __forceinline__ F2 pk(float lo, float hi)
{
    F2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r.v) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void upk(F2 a, float &lo, float &hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(a.v));
}
__device__ __forceinline__ F2 sp2(float c) { return pk(c, c); }
__device__ __forceinline__ F2 fma2(F2 a, F2 b, F2 c)
{
    F2 r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r.v) : "l"(a.v), "l"(b.v), "l"(c.v));
    return r;
}
__device__ __forceinline__ F2 mul2(F2 a, F2 b)
{
    F2 r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r.v) : "l"(a.v), "l"(b.v));
    return r;
}
__device__ __forceinline__ F2 add2(F2 a, F2 b)
{
    F2 r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r.v) : "l"(a.v), "l"(b.v));
    return r;
}

// Multiplicative correction 2^t_lo ~ 1 + t_lo ln 2 for a float-float t.
__device__ __forceinline__ float corr(float t_hi, float t_lo)
{
    float c = fmaf(t_lo, kLn2f, 1.0f);
    return fabsf(t_hi) < kCorrMax ? c : 1.0f;
}

// Low part of x * (c_hi + c_lo) given t_hi = x * c_hi.
__device__ __forceinline__ float prod_lo(float x, float c_hi, float c_lo, float t_hi)
{
    return fmaf(x, c_lo, fmaf(x, c_hi, -t_hi));
}

// Activations that provide pairwise (packed .f32x2) versions of f and df for
// a precision mode specialise this to true.
template <class A, bool P>
struct HasPairs {
    static constexpr bool value = false;
};
// Activations whose plain (not per-channel) backward also has a pairwise df2
// (a superset of HasPairs).
template <class A, bool P>
struct HasPairsBwd {
    static constexpr bool value = HasPairs<A, P>::value;
};

// Per-launch constants, built on the device from the scalar parameter.
struct Coef {
    float p;      // alpha (Swish) or slope (LeakyReLU)
    float c_hi;   // exponent coefficient (fp32 head)
    float c_lo;   // exponent coefficient (tail)
};

// Float-float value of m * log2(e) for an fp32 m.
__device__ __forceinline__ void scaled_log2e(float m, float &hi, float &lo)
{
    hi = m * kLog2eHi;
    lo = fmaf(m, kLog2eLo, fmaf(m, kLog2eHi, -hi));
}

// ------------------------------------------------- near the zero of f'
// Swish' (as a function of v = alpha x), GELU-erf' and GELU-tanh' each vanish
// at one point v0 < 0, where the terms of f' cancel.  The main paths form
// the argument with one fp32 rounding (alpha x, or gamma x + beta in the
// per-channel kernels) and evaluate f' in fp32: an absolute error of about
// 1.5e-7 (times |dy|), which within about 1e-4 of v0 is a large part of f'
// itself.  With bf16 storage every output must stay within one bf16 ulp of
// the exact result, so there the elements with |v - v0| < kRootWin are
// recomputed from d = v - v0 formed in fp64 (root_d), as the Taylor
// polynomial
//   f'(v0 + d) = d (f''(v0) + d f'''(v0) / 2),
// whose next term is below 1e-7 of f' over the window.  Outside the window
// |f'| > 2.1e-4, so the main path's error stays below 1e-3 of f', inside half
// a bf16 ulp.  The constants (v0 in fp64 and its fp32 rounding for the
// window test, f''(v0), f'''(v0) / 2) come from csrc/near_root_constants.py.
// fp32 storage keeps the main path: its rule is relative to the condition
// scale of f', which that error meets.
constexpr float kRootWin = 0.0009765625f;   // 2^-10

// d = m (g x + b) - v0 in fp64: g x is exact there, each FMA rounds once
// (2^-53 relative) and v0 is held to 2^-53, so d carries an absolute error
// below 5e-16 and the recomputed f' is within a bf16 half-ulp of the exact
// value wherever |d| > 2e-13.  Taken only for the few elements inside the
// window.
__device__ __forceinline__ float root_d(float g, float x, float b, float m, double v0)
{
    const double z = fma((double)g, (double)x, (double)b);
    return (float)fma((double)m, z, -v0);
}

// dy f'(v0 + d) from the Taylor polynomial of activation A at its zero.
template <class A>
__device__ __forceinline__ float root_df(float d, float dy)
{
    return dy * (d * fmaf(A::kRootF3h, d, A::kRootF2));
}

// ------------------------------------------------------------------ ReLU
struct ReLU {
    static constexpr bool kHasRoot = false;
    template <bool P>
    static __device__ __forceinline__ bool bwd_flagged(float, const Coef &) { return false; }
    template <bool P>
    static __device__ __forceinline__ bool is_tail_bwd(float x, const Coef &k) { return is_tail(x, k); }
    static __device__ __forceinline__ Coef coef(float) { return Coef{0.f, 0.f, 0.f}; }
    template <bool P>
    static __device__ __forceinline__ float f(float x, const Coef &, bool &)
    {
        return x > 0.f ? x : (x != x ? x : 0.f);
    }
    template <bool P>
    static __device__ __forceinline__ float f_tail(float x, const Coef &) { return x; }
    template <bool P>
    static __device__ __forceinline__ float df(float x, float dy, const Coef &, bool &)
    {
        return dy * (x > 0.f ? 1.f : 0.f);
    }
    template <bool P>
    static __device__ __forceinline__ float df_tail(float, float dy, const Coef &) { return dy; }
    static __device__ __forceinline__ bool is_tail(float, const Coef &) { return false; }
};

// ------------------------------------------------------------- LeakyReLU
struct LeakyReLU {
    static constexpr bool kHasRoot = false;
    template <bool P>
    static __device__ __forceinline__ bool bwd_flagged(float, const Coef &) { return false; }
    template <bool P>
    static __device__ __forceinline__ bool is_tail_bwd(float x, const Coef &k) { return is_tail(x, k); }
    static __device__ __forceinline__ Coef coef(float slope) { return Coef{slope, 0.f, 0.f}; }
    template <bool P>
    static __device__ __forceinline__ float f(float x, const Coef &k, bool &)
    {
        return x > 0.f ? x : k.p * x;
    }
    template <bool P>
    static __device__ __forceinline__ float f_tail(float x, const Coef &) { return x; }
    template <bool P>
    static __device__ __forceinline__ float df(float x, float dy, const Coef &k, bool &)
    {
        return dy * (x > 0.f ? 1.f : k.p);
    }
    template <bool P>
    static __device__ __forceinline__ float df_tail(float, float dy, const Coef &) { return dy; }
    static __device__ __forceinline__ bool is_tail(float, const Coef &) { return false; }
};

// -------------------------------------------------------------- Sigmoid
// t = -x log2 e; s = 1 / (1 + 2^t).
struct Sigmoid {
    static constexpr bool kHasRoot = false;
    // Every element a backward main path flags (df: |t| > kTailT).
    template <bool P>
    static __device__ __forceinline__ bool bwd_flagged(float x, const Coef &k) { return fabsf(x * k.c_hi) > kTailT; }
    template <bool P>
    static __device__ __forceinline__ bool is_tail_bwd(float x, const Coef &k) { return is_tail(x, k); }
    static __device__ __forceinline__ Coef coef(float)
    {
        Coef k;
        k.p = 1.f;
        scaled_log2e(-1.f, k.c_hi, k.c_lo);
        return k;
    }
    template <bool P>
    static __device__ __forceinline__ float expo(float x, const Coef &k, float &t)
    {
        t = x * k.c_hi;
        float E = ex2_ftz(t);
        if (P) E *= corr(t, prod_lo(x, k.c_hi, k.c_lo, t));
        return E;
    }
    // 2^(64 - t): the sigmoid scaled by 2^64 in the tail (t > 126).
    template <bool P>
    static __device__ __forceinline__ float tail_s64(float x, const Coef &k)
    {
        float t = x * k.c_hi;
        float s64 = ex2_ftz(64.f - t);
        if (P) s64 *= corr(t, -prod_lo(x, k.c_hi, k.c_lo, t));
        return s64;
    }
    // Both tails: for x << 0 the sigmoid, for x >> 0 its complement E s,
    // would be subnormal.  The forward only needs the first; taking both is
    // harmless (the forward's tail value for x >> 0 is exactly 1).
    static __device__ __forceinline__ bool is_tail(float x, const Coef &k)
    {
        return fabsf(x * k.c_hi) > kTailT;
    }

    template <bool P>
    static __device__ __forceinline__ float f(float x, const Coef &k, bool &tail)
    {
        float t;
        float E = expo<P>(x, k, t);
        tail |= t > kTailT;
        return rcp_ftz(1.f + E);
    }
    template <bool P>
    static __device__ __forceinline__ float f_tail(float x, const Coef &k)
    {
        return x > 0.f ? 1.f : tail_s64<P>(x, k) * kTwoM64;
    }
    // dx = dy s (1 - s)
    template <bool P>
    static __device__ __forceinline__ float df(float x, float dy, const Coef &k, bool &tail)
    {
        float t;
        float E = expo<P>(x, k, t);
        tail |= fabsf(t) > kTailT;
        float s = rcp_ftz(1.f + E);
        float sm = x > 0.f ? E * s : 1.f - s;
        return dy * (s * sm);
    }
    // |t| > 124: s (1 - s) = 2^-|t| to within 2^-124 relative, formed as
    // 2^(64 - |t|) 2^-64 so that it stays normal until the final scaling.
    template <bool P>
    static __device__ __forceinline__ float df_tail(float x, float dy, const Coef &k)
    {
        float t = x * k.c_hi;
        float e = ex2_ftz(64.f - fabsf(t));
        if (P) {
            const float lo = prod_lo(x, k.c_hi, k.c_lo, t);
            e *= corr(t, t > 0.f ? -lo : lo);
        }
        return (dy * e) * kTwoM64;
    }
};

// ----------------------------------------------------------------- Tanh
// Forward: CUDA's tanhf for fp32 storage, the MUFU tanh for bf16.  Backward: 1 - tanh^2 x = 4 Sigmoid(2|x|)
// Sigmoid(-2|x|) = 4 E s^2 with E = 2^t, t = -2|x| log2 e (t <= 0),
// s = 1/(1+E) = Sigmoid(2|x|) and Sigmoid(-2|x|) = E s.
struct Tanh {
    static constexpr bool kHasRoot = false;
    // Every element a backward main path flags (df: t < -120).
    template <bool P>
    static __device__ __forceinline__ bool bwd_flagged(float x, const Coef &k) { return fabsf(x) * k.c_hi < -120.f; }
    template <bool P>
    static __device__ __forceinline__ bool is_tail_bwd(float x, const Coef &k) { return is_tail(x, k); }
    static __device__ __forceinline__ Coef coef(float)
    {
        Coef k;
        k.p = 1.f;
        scaled_log2e(-2.f, k.c_hi, k.c_lo);
        return k;
    }
    static __device__ __forceinline__ bool is_tail(float x, const Coef &k)
    {
        return fabsf(x) * k.c_hi < -120.f;
    }
    template <bool P>
    static __device__ __forceinline__ float f(float x, const Coef &, bool &)
    {
        if constexpr (P)
            return tanhf(x);
        else
            return tanh_mufu(x);
    }
    template <bool P>
    static __device__ __forceinline__ float f_tail(float x, const Coef &k)
    {
        bool unused = false;
        return f<P>(x, k, unused);
    }
    template <bool P>
    static __device__ __forceinline__ float df(float x, float dy, const Coef &k, bool &tail)
    {
        float a = fabsf(x);
        float t = a * k.c_hi;
        float E = ex2_ftz(t);
        if (P) E *= corr(t, prod_lo(a, k.c_hi, k.c_lo, t));
        tail |= t < -120.f;
        float s = rcp_ftz(1.f + E);
        return dy * (((4.f * E) * s) * s);
    }
    // t < -120: s = 1, 4E s^2 = 2^(t + 2) may be subnormal; use 2^(t + 66) 2^-64.
    template <bool P>
    static __device__ __forceinline__ float df_tail(float x, float dy, const Coef &k)
    {
        float a = fabsf(x);
        float t = a * k.c_hi;
        float e64 = ex2_ftz(t + 66.f);
        if (P) e64 *= corr(t, prod_lo(a, k.c_hi, k.c_lo, t));
        return (dy * e64) * kTwoM64;
    }
};

// ------------------------------------------------------------- GELU-erf
// y = x Phi(x), Phi(x) = erfc(w) / 2 with w = -x / sqrt 2; backward
// Phi(x) + x phi(x), phi(x) = e^(-w^2) / sqrt(2 pi).
//
// fp32 storage (P = true): CUDA's erfcf and expf, with -x / sqrt 2 and x^2
// carried as float-float pairs and the first-order corrections
// d erfc = -(2 / sqrt pi) e^(-w^2) dw and e^(-l/2) ~ 1 - l/2.
//
// bf16 storage (P = false): the Chebyshev-fitted approximation of erfc from
// Press, Teukolsky, Vetterling and Flannery, "Numerical Recipes in C", 2nd
// ed., section 6.2 (fractional error below 1.2e-7 for every argument):
//   erfc(|w|) = t exp(-w^2 + P(t)),  t = 1 / (1 + |w| / 2),
//   P a degree-9 polynomial in t;  erfc(w) = 2 - erfc(|w|) for w < 0.
// It costs one reciprocal and one exponential on the MUFU pipe plus a
// Horner chain, instead of the library's erfcf.  Where the exponential would
// be subnormal (-w^2 + P(t) < -124 ln 2, i.e. x below about -13.1) but
// x Phi(x) is still normal, the element is recomputed with the exponentials
// scaled by 2^64.
//
// The bf16 forward uses the same form with a degree-5 polynomial fitted
// here (csrc/fit_erfc_bf16.py: near-minimax over |w| <= 9.6, error of
// log erfc below 7.7e-6, far inside the bf16 rounding of the result).  The
// backward, whose value cancels near x = -0.75, needs the full accuracy; it
// writes erfc(|w|) = t e^(-w^2) Q(t) with Q(t) = erfcx(|w|) / t fitted as a
// degree-8 polynomial (same script; fractional error 5e-8 in exact
// arithmetic, about 2e-7 evaluated in fp32, as the degree-9 form), so that
// the Gaussian e^(-w^2) of f' is the only exponential.  Its tail test is on
// that exponential's argument (-w^2 log2 e < -124); the deep-tail recompute
// is the scaled form above.
struct GeluErf {
    // Zero of f' (Phi(x) + x phi(x) = 0) for the compensated recompute of the
    // per-channel kernels; the plain kernels see x exactly, and the bf16 x
    // nearest the zero keep |f'| >= 7e-4, so they need none.
    static constexpr bool kHasRoot = true;
    static constexpr double kRootD = -0.75179152469356445746;
    static constexpr float kRootHi = -0.7517915368080139f;      // fp32(kRootD)
    static constexpr float kRootF2 = 0.43149399757385254f;
    static constexpr float kRootF3h = 0.38828498125076294f;
    static __device__ __forceinline__ float root_scale(const Coef &) { return 1.f; }
    static __device__ __forceinline__ bool near_root(float z, const Coef &)
    {
        return fabsf(__fsub_rn(z, kRootHi)) < kRootWin;
    }
    static constexpr float kNegRsqrt2Hi = -0.707106769084930419921875f;
    static constexpr float kNegRsqrt2Lo = -1.2101617104478969362e-08f;
    static constexpr float kTwoRsqrtPi = 1.12837916709551257f;     // 2 / sqrt(pi)
    static constexpr float kRsqrt2Pi = 0.398942280401432678f;      // 1 / sqrt(2 pi)
    static constexpr float kLog2ef = 1.44269504088896340736f;
    // The bf16 forms use t = 1 / (1 + a / 2) (Press et al., "Numerical
    // Recipes in C", 6.2) through h = t / 2 = 1 / (2 + a): each polynomial in
    // t is evaluated in h with coefficient k scaled by 2^k, which leaves every
    // Horner step the t-form's value times a power of two, so the polynomial's
    // value is bitwise the same, and a product with h is half the product
    // with t, exactly.  That half is the 1/2 of Phi = erfc / 2, which then
    // costs no multiply.
    //
    // Backward: erfc(a) = t e^(-a^2) Q(t) with Q(t) = erfcx(a) / t fitted
    // directly (degree 8, coefficients of t^8 .. t^0, each times 2^k below;
    // csrc/fit_erfc_bf16.py), so that the one exponential e^(-a^2) serves
    // both erfc and the Gaussian of f' (q8, q8_2); h e^(-a^2) Q = erfc / 2.
    static __device__ __forceinline__ float q8(float h)
    {
        float q = -0.058932472f * 256.f;
        q = fmaf(q, h, 0.283905655f * 128.f);
        q = fmaf(q, h, -0.485806316f * 64.f);
        q = fmaf(q, h, 0.276463121f * 32.f);
        q = fmaf(q, h, -0.0255132243f * 16.f);
        q = fmaf(q, h, 0.202212647f * 8.f);
        q = fmaf(q, h, 0.243224636f * 4.f);
        q = fmaf(q, h, 0.282358527f * 2.f);
        return fmaf(q, h, 0.282087386f);
    }
    static __device__ __forceinline__ F2 q8_2(F2 h)
    {
        F2 q = sp2(-0.058932472f * 256.f);
        q = fma2(q, h, sp2(0.283905655f * 128.f));
        q = fma2(q, h, sp2(-0.485806316f * 64.f));
        q = fma2(q, h, sp2(0.276463121f * 32.f));
        q = fma2(q, h, sp2(-0.0255132243f * 16.f));
        q = fma2(q, h, sp2(0.202212647f * 8.f));
        q = fma2(q, h, sp2(0.243224636f * 4.f));
        q = fma2(q, h, sp2(0.282358527f * 2.f));
        return fma2(q, h, sp2(0.282087386f));
    }

    static __device__ __forceinline__ Coef coef(float) { return Coef{1.f, 0.f, 0.f}; }

    // Chebyshev approximation pieces for a = |w| (Press et al.'s degree-9
    // erfc): h, and u = (-a^2 + P(t)) log2 e, so that erfc(a) = 2 h 2^u.
    static __device__ __forceinline__ float nr_parts(float a, float &h)
    {
        h = rcp_ftz(a + 2.0f);
        float p = 0.17087277f * 512.f;
        p = fmaf(p, h, -0.82215223f * 256.f);
        p = fmaf(p, h, 1.48851587f * 128.f);
        p = fmaf(p, h, -1.13520398f * 64.f);
        p = fmaf(p, h, 0.27886807f * 32.f);
        p = fmaf(p, h, -0.18628806f * 16.f);
        p = fmaf(p, h, 0.09678418f * 8.f);
        p = fmaf(p, h, 0.37409196f * 4.f);
        p = fmaf(p, h, 1.00002368f * 2.f);
        p = fmaf(p, h, -1.26551223f);
        return fmaf(-a, a, p) * kLog2ef;
    }
    // Degree-5 form of nr_parts for the bf16 forward.
    static __device__ __forceinline__ float nr5_parts(float a, float &h)
    {
        h = rcp_ftz(a + 2.0f);
        float p = 0.228795588f * 32.f;
        p = fmaf(p, h, -0.709205508f * 16.f);
        p = fmaf(p, h, 0.474508315f * 8.f);
        p = fmaf(p, h, 0.254436046f * 4.f);
        p = fmaf(p, h, 1.01801503f * 2.f);
        p = fmaf(p, h, -1.26654184f);
        return fmaf(-a, a, p) * kLog2ef;
    }
    // The bf16 main paths serve x >= kTailX, where every exponential they take
    // (down to 2^-113 for the Gaussian, about 2^-115 for erfc) stays normal
    // and a = |x| / sqrt 2 stays inside the range the fitted polynomials were
    // fitted on (a <= 9.6, x >= -13.6); the elements below are recomputed with
    // the exponentials scaled by 2^64.  One comparison, so that the per-element
    // test of the recompute loops costs next to nothing.
    static constexpr float kTailX = -12.5f;
    static __device__ __forceinline__ bool is_tail(float x, const Coef &) { return x < kTailX; }
    // Every element a backward main path flags (bf16 only: x < kTailX).
    template <bool P>
    static __device__ __forceinline__ bool bwd_flagged(float x, const Coef &k)
    {
        return !P && is_tail(x, k);
    }
    template <bool P>
    static __device__ __forceinline__ bool is_tail_bwd(float x, const Coef &k) { return is_tail(x, k); }

    // returns erfc(-x / sqrt 2) and sets g = e^(-x^2 / 2) (accurate path)
    static __device__ __forceinline__ float erfc_and_gauss_precise(float x, float &g)
    {
        float w = x * kNegRsqrt2Hi;
        float ec = erfcf(w);
        float h = x * x;
        g = expf(-0.5f * h);
        float l = fmaf(x, x, -h);
        l = h < kBig ? l : 0.f;
        g *= fmaf(-0.5f, l, 1.f);
        float wl = fmaf(x, kNegRsqrt2Lo, fmaf(x, kNegRsqrt2Hi, -w));
        return fmaf(-kTwoRsqrtPi * wl, g, ec);
    }
    // Pairwise bf16-mode forward and backward: the same operations in the
    // same order as f / df below (bitwise the same results), with the
    // multiply-add chains on packed pairs and the two MUFU operations scalar.
    static __device__ __forceinline__ void nr5_parts2(F2 x, float &w0, float &w1, F2 &h, F2 &u)
    {
        const F2 w = mul2(x, sp2(kNegRsqrt2Hi));
        upk(w, w0, w1);
        const F2 a = pk(fabsf(w0), fabsf(w1));
        float d0, d1;
        upk(add2(a, sp2(2.0f)), d0, d1);
        h = pk(rcp_ftz(d0), rcp_ftz(d1));
        F2 p = sp2(0.228795588f * 32.f);
        p = fma2(p, h, sp2(-0.709205508f * 16.f));
        p = fma2(p, h, sp2(0.474508315f * 8.f));
        p = fma2(p, h, sp2(0.254436046f * 4.f));
        p = fma2(p, h, sp2(1.01801503f * 2.f));
        p = fma2(p, h, sp2(-1.26654184f));
        u = mul2(fma2(pk(-fabsf(w0), -fabsf(w1)), a, p), sp2(kLog2ef));
    }
    // Phi(x) = erfc(w) / 2 for w = -x / sqrt 2: h 2^u for w >= 0, else 1 - h 2^u.
    static __device__ __forceinline__ F2 half_erfc2(float w0, float w1, F2 h, float u0, float u1)
    {
        float a0, a1;
        upk(mul2(h, pk(ex2_ftz(u0), ex2_ftz(u1))), a0, a1);
        return pk(w0 >= 0.f ? a0 : 1.f - a0, w1 >= 0.f ? a1 : 1.f - a1);
    }
    static __device__ __forceinline__ void f2(float x0, float x1, const Coef &, bool &tail, float &o0, float &o1)
    {
        const F2 x = pk(x0, x1);
        float w0, w1, u0, u1;
        F2 h, u;
        nr5_parts2(x, w0, w1, h, u);
        upk(u, u0, u1);
        tail |= (x0 < kTailX) | (x1 < kTailX);
        upk(mul2(x, half_erfc2(w0, w1, h, u0, u1)), o0, o1);
    }
    static __device__ __forceinline__ void df2(float x0, float x1, float dy0, float dy1, const Coef &, bool &tail,
                                               float &o0, float &o1)
    {
        const F2 x = pk(x0, x1);
        const F2 w = mul2(x, sp2(kNegRsqrt2Hi));
        float w0, w1;
        upk(w, w0, w1);
        const F2 a = pk(fabsf(w0), fabsf(w1));
        float d0, d1;
        upk(add2(a, sp2(2.0f)), d0, d1);
        const F2 h = pk(rcp_ftz(d0), rcp_ftz(d1));
        const F2 q = q8_2(h);
        float v0, v1;
        upk(mul2(mul2(w, w), sp2(-kLog2ef)), v0, v1);
        tail |= (x0 < kTailX) | (x1 < kTailX);
        const F2 g = pk(ex2_ftz(v0), ex2_ftz(v1));
        float a0, a1;
        upk(mul2(mul2(h, q), g), a0, a1);
        const F2 phi = pk(w0 >= 0.f ? a0 : 1.f - a0, w1 >= 0.f ? a1 : 1.f - a1);   // Phi(x)
        const F2 d = fma2(mul2(x, sp2(kRsqrt2Pi)), g, phi);
        upk(mul2(pk(dy0, dy1), d), o0, o1);
    }

    template <bool P>
    static __device__ __forceinline__ float f(float x, const Coef &, bool &tail)
    {
        if constexpr (P) {
            float g;
            float ec = erfc_and_gauss_precise(x, g);
            return (0.5f * x) * ec;
        } else {
            const float w = x * kNegRsqrt2Hi;
            float h;
            const float u = nr5_parts(fabsf(w), h);
            tail |= x < kTailX;
            const float half = h * ex2_ftz(u);                  // erfc(|w|) / 2
            return x * (w >= 0.f ? half : 1.f - half);          // x Phi(x)
        }
    }
    template <bool P>
    static __device__ __forceinline__ float f_tail(float x, const Coef &k)
    {
        if constexpr (P) {
            bool t = false;
            return f<P>(x, k, t);
        } else {
            // x << 0: w > 0, erfc(w) / 2 = h 2^u with u < -124; scale by 2^64
            const float w = x * kNegRsqrt2Hi;
            float h;
            const float u = nr_parts(w, h);
            return ((x * h) * ex2_ftz(u + 64.f)) * kTwoM64;
        }
    }
    template <bool P>
    static __device__ __forceinline__ float df(float x, float dy, const Coef &, bool &tail)
    {
        if constexpr (P) {
            float g;
            float ec = erfc_and_gauss_precise(x, g);
            return dy * fmaf(x * kRsqrt2Pi, g, 0.5f * ec);
        } else {
            const float w = x * kNegRsqrt2Hi;
            const float h = rcp_ftz(fabsf(w) + 2.0f);
            const float q = q8(h);
            const float v = (w * w) * -kLog2ef;
            tail |= x < kTailX;
            const float g = ex2_ftz(v);
            const float half = (h * q) * g;                     // erfc(|w|) / 2
            return dy * fmaf(x * kRsqrt2Pi, g, w >= 0.f ? half : 1.f - half);
        }
    }
    template <bool P>
    static __device__ __forceinline__ float df_tail(float x, float dy, const Coef &k)
    {
        if constexpr (P) {
            bool t = false;
            return df<P>(x, dy, k, t);
        } else {
            const float w = x * kNegRsqrt2Hi;
            float h;
            const float u = nr_parts(w, h);
            const float e64 = ex2_ftz(u + 64.f);                       // erfc(w) / (2 h), scaled
            const float g64 = ex2_ftz(fmaf(-(w * w), kLog2ef, 64.f));  // e^(-w^2), scaled
            return (dy * fmaf(x * kRsqrt2Pi, g64, h * e64)) * kTwoM64;
        }
    }
};

template <>
struct HasPairs<GeluErf, false> {
    static constexpr bool value = true;
};

// ------------------------------------------------------------ GELU-tanh
// y = x Sigmoid(v), v = 2u = x (k1 + k3 x^2), k1 = 2 sqrt(2/pi),
// k3 = 2 sqrt(2/pi) 0.044715 (Hendrycks and Gimpel's constants).
// t = -v log2 e = x (c1 + c3 x^2).  Backward:
// Sigmoid(v) + x v' Sigmoid(v) Sigmoid(-v), v' = k1 + 3 k3 x^2.
struct GeluTanh {
    // Zero of f' (as for GeluErf: used by the per-channel kernels only).
    static constexpr bool kHasRoot = true;
    static constexpr double kRootD = -0.75246142207101625849;
    static constexpr float kRootHi = -0.7524614334106445f;      // fp32(kRootD)
    static constexpr float kRootF2 = 0.4304001033306122f;
    static constexpr float kRootF3h = 0.38751843571662903f;
    static __device__ __forceinline__ float root_scale(const Coef &) { return 1.f; }
    // Tested on the exponent t = z (c1 + c3 z^2) as the bf16 forms compute it
    // (see SwishT): v0 maps to kRootT, 2^-10 in z to kRootWinT, and the packed
    // backward's u = t - kRootT serves both of its guards.
    static constexpr float kRootT = 1.7761809825897217f;
    static constexpr float kRootWinT = 0.0024190107360482216f;
    static constexpr float kTailU = 122.0f;
    static __device__ __forceinline__ bool near_root(float z, const Coef &)
    {
        float tl;
        return fabsf(__fsub_rn(expo_arg<false>(z, tl), kRootT)) < kRootWinT;
    }
    static constexpr double kK1 = 1.5957691216057307;            // 2 sqrt(2/pi)
    static constexpr double kK3 = 1.5957691216057307 * 0.044715;
    static constexpr float kK1f = (float)kK1;
    static constexpr float kK3x3f = (float)(3.0 * kK3);
    static constexpr float kC1f = (float)(-kK1 * kLog2eD);
    static constexpr float kC3f = (float)(-kK3 * kLog2eD);
    static constexpr double kC1d = -kK1 * kLog2eD;
    static constexpr double kC3d = -kK3 * kLog2eD;

    static __device__ __forceinline__ Coef coef(float) { return Coef{1.f, 0.f, 0.f}; }

    template <bool P>
    static __device__ __forceinline__ float expo_arg(float x, float &t_lo)
    {
        if (P) {
            double xd = (double)x;
            double td = xd * fma(kC3d, xd * xd, kC1d);
            float t = (float)td;
            t_lo = (float)(td - (double)t);
            return t;
        }
        t_lo = 0.f;
        return x * fmaf(kC3f, x * x, kC1f);
    }
    static __device__ __forceinline__ bool is_tail(float x, const Coef &)
    {
        float tl;
        return expo_arg<false>(x, tl) > kTailT;
    }
    // The plain bf16 backward's packed form (df2) also flags t < -kHugeT
    // (x beyond about 2e10, where x v' could overflow); df_tail gives those
    // the scalar form.
    static constexpr float kHugeT = 1e30f;
    template <bool P>
    static __device__ __forceinline__ bool is_tail_bwd(float x, const Coef &k)
    {
        if constexpr (P) return is_tail(x, k);
        float tl;
        const float t = expo_arg<false>(x, tl);
        return t > kTailT || t < -kHugeT;
    }
    // Every element a backward main path flags: t > kTailT (scalar form);
    // for bf16, |u| < kRootWinT or |u| > kTailU, u = t - kRootT (the packed
    // form of the per-channel kernels, which contains the scalar one's).
    template <bool P>
    static __device__ __forceinline__ bool bwd_flagged(float x, const Coef &)
    {
        float tl;
        const float t = expo_arg<P>(x, tl);
        if constexpr (P) return t > kTailT;
        const float u = __fsub_rn(t, kRootT);
        return fabsf(u) < kRootWinT || fabsf(u) > kTailU;
    }
    template <bool P>
    static __device__ __forceinline__ float f(float x, const Coef &, bool &tail)
    {
        float tl;
        float t = expo_arg<P>(x, tl);
        float E = ex2_ftz(t);
        if (P) E *= corr(t, tl);
        tail |= t > kTailT;
        return x * rcp_ftz(1.f + E);
    }
    template <bool P>
    static __device__ __forceinline__ float s64_tail(float x)
    {
        float tl;
        float t = expo_arg<P>(x, tl);
        float s64 = ex2_ftz(64.f - t);
        if (P) s64 *= corr(t, -tl);
        return s64;
    }
    template <bool P>
    static __device__ __forceinline__ float f_tail(float x, const Coef &)
    {
        return (x * s64_tail<P>(x)) * kTwoM64;
    }
    // x v', clamped so that it times a zero sigmoid factor stays 0
    static __device__ __forceinline__ float xdv(float x)
    {
        float q = x * fmaf(kK3x3f, x * x, kK1f);
        return fmaxf(fminf(q, kBig), -kBig);
    }
    template <bool P>
    static __device__ __forceinline__ float df(float x, float dy, const Coef &, bool &tail)
    {
        float tl;
        float t = expo_arg<P>(x, tl);
        float E = ex2_ftz(t);
        if (P) E *= corr(t, tl);
        tail |= t > kTailT;
        float s = rcp_ftz(1.f + E);
        float sm = x > 0.f ? E * s : 1.f - s;
        float q = xdv(x);
        return dy * fmaf(q * s, sm, s);
    }
    // v << 0: Sigmoid(-v) = 1, f' = s (1 + x v'); huge positive x (flagged by
    // df2 only): the scalar form, whose x v' is clamped.
    template <bool P>
    static __device__ __forceinline__ float df_tail(float x, float dy, const Coef &k)
    {
        if constexpr (!P) {
            if (x > 0.f) {
                bool unused = false;
                return df<false>(x, dy, k, unused);
            }
        }
        float q = xdv(x);
        return ((dy * s64_tail<P>(x)) * (1.f + q)) * kTwoM64;
    }
    // Two elements, bf16 storage (the plain backward): t as in expo_arg, E =
    // 2^t, s = 1 / (1 + E), and f' = s (1 + x v' E s) with E s = Sigmoid(-v);
    // flags t > kTailT (deep negative x) and t < -kHugeT.
    static __device__ __forceinline__ void df2(float x0, float x1, float dy0, float dy1, const Coef &, bool &tail,
                                               float &o0, float &o1)
    {
        const F2 x = pk(x0, x1);
        const F2 x2 = mul2(x, x);
        float t0, t1;
        upk(mul2(x, fma2(sp2(kC3f), x2, sp2(kC1f))), t0, t1);
        const float e0 = ex2_ftz(t0), e1 = ex2_ftz(t1);
        tail |= (t0 > kTailT) | (t1 > kTailT) | (t0 < -kHugeT) | (t1 < -kHugeT);
        const F2 E = pk(e0, e1);
        float a0, a1;
        upk(add2(sp2(1.f), E), a0, a1);
        const F2 s = pk(rcp_ftz(a0), rcp_ftz(a1));
        const F2 q = mul2(x, fma2(sp2(kK3x3f), x2, sp2(kK1f)));
        const F2 r = fma2(q, mul2(E, s), sp2(1.f));
        upk(mul2(pk(dy0, dy1), mul2(s, r)), o0, o1);
    }
};

template <>
struct HasPairsBwd<GeluTanh, false> {
    static constexpr bool value = true;
};

// ---------------------------------------------------------------- Swish
// y = x Sigmoid(z), z = alpha x; t = x c, c = -alpha log2 e (float-float).
// dx = dy (s + z s Sigmoid(-z)); d alpha term = dy x^2 s Sigmoid(-z).
// RC: whether the bf16 backward recomputes the neighbourhood of the zero of
// f' (see "near the zero of f'").  Swish (RC = true) is the general form.
// With alpha a power of two (or zero) and bf16 x, alpha x is exact and lies
// on the bf16 grid scaled by 2^k, which is the bf16 grid again, so the
// inputs nearest v0 keep |f'| >= 6e-4 and the main path is within one ulp:
// the streaming kernels then use SwishT<false>, without the test.
template <bool RC>
struct SwishT {
    // Zero of Swish_1'(v) = Sigmoid(v) + v Sigmoid(v) Sigmoid(-v), at
    // v0 = -(1 + W(1/e)); x Sigmoid(alpha x) has x-derivative Swish_1'(alpha x),
    // so an element is near it when alpha x is.  With alpha = 1 and bf16 x the
    // nearest inputs keep |f'| >= 6e-4; any other alpha can put alpha x
    // anywhere, hence the compensated recompute (bf16 storage).
    static constexpr bool kHasRoot = RC;
    static constexpr double kRootD = -1.2784645427610737951;
    static constexpr float kRootHi = -1.2784645557403564f;      // fp32(kRootD)
    static constexpr float kRootF2 = 0.2178117036819458f;
    static constexpr float kRootF3h = 0.14664879441261292f;
    // The window is tested on the sigmoid's exponent variable t = x c_hi =
    // -alpha x log2(e) (rounded once, as every main path forms it): v0 maps to
    // kRootT and 2^-10 in v to kRootWinT.  The packed backward then takes one
    // u = t - kRootT for both of its guards: |u| < kRootWinT (near v0) and
    // |u| > kTailU, which contains |t| > kTailT.
    static constexpr float kRootT = 1.8444344997406006f;      // -v0 log2(e)
    static constexpr float kRootWinT = 0.001408881857059896f; // 2^-10 log2(e)
    static constexpr float kTailU = 122.0f;
    static __device__ __forceinline__ float root_scale(const Coef &k) { return k.p; }
    static __device__ __forceinline__ bool near_root(float z, const Coef &k)
    {
        return fabsf(__fsub_rn(__fmul_rn(z, k.c_hi), kRootT)) < kRootWinT;
    }
    // d = alpha x - v0
    static __device__ __forceinline__ float root_dx(float x, const Coef &k) { return root_d(1.f, x, 0.f, k.p, kRootD); }
    static __device__ __forceinline__ Coef coef(float alpha)
    {
        Coef k;
        k.p = alpha;
        scaled_log2e(-alpha, k.c_hi, k.c_lo);
        return k;
    }
    template <bool P>
    static __device__ __forceinline__ float expo(float x, const Coef &k, float &t)
    {
        t = x * k.c_hi;
        float E = ex2_ftz(t);
        if (P) E *= corr(t, prod_lo(x, k.c_hi, k.c_lo, t));
        return E;
    }
    template <bool P>
    static __device__ __forceinline__ float tail_s64(float x, const Coef &k)
    {
        float t = x * k.c_hi;
        float s64 = ex2_ftz(64.f - t);
        if (P) s64 *= corr(t, -prod_lo(x, k.c_hi, k.c_lo, t));
        return s64;
    }
    static __device__ __forceinline__ bool is_tail(float x, const Coef &k) { return x * k.c_hi > kTailT; }
    template <bool P>
    static __device__ __forceinline__ bool is_tail_bwd(float x, const Coef &k)
    {
        if constexpr (!P && RC) return is_tail(x, k) || near_root(x, k);
        return is_tail(x, k);
    }
    // Every element a backward main path flags: t > kTailT (scalar form),
    // |t| > kTailT (the packed bf16 form of the per-channel kernels), and with
    // bf16 storage the neighbourhood of the zero of f'.
    template <bool P>
    static __device__ __forceinline__ bool bwd_flagged(float x, const Coef &k)
    {
        if constexpr (!P && RC) {
            const float u = __fsub_rn(__fmul_rn(x, k.c_hi), kRootT);
            return fabsf(u) < kRootWinT || fabsf(u) > kTailU;
        }
        if constexpr (!P) return fabsf(x * k.c_hi) > kTailT;
        return x * k.c_hi > kTailT;
    }

    template <bool P>
    static __device__ __forceinline__ float f(float x, const Coef &k, bool &tail)
    {
        float t;
        float E = expo<P>(x, k, t);
        tail |= t > kTailT;
        return x * rcp_ftz(1.f + E);
    }
    template <bool P>
    static __device__ __forceinline__ float f_tail(float x, const Coef &k)
    {
        return (x * tail_s64<P>(x, k)) * kTwoM64;
    }
    template <bool P>
    static __device__ __forceinline__ float df(float x, float dy, const Coef &k, bool &tail)
    {
        float t;
        float E = expo<P>(x, k, t);
        tail |= t > kTailT;
        float s = rcp_ftz(1.f + E);
        float z = __fmul_rn(k.p, x);
        if constexpr (!P && RC) tail |= fabsf(__fsub_rn(t, kRootT)) < kRootWinT;
        float sm = z > 0.f ? E * s : 1.f - s;
        z = fminf(z, kBig);
        return dy * fmaf(z * s, sm, s);
    }
    // Elements flagged by df: near the zero of f' (bf16 storage), or the deep
    // negative tail.
    template <bool P>
    static __device__ __forceinline__ float df_tail(float x, float dy, const Coef &k)
    {
        if constexpr (!P && RC) {
            if (near_root(x, k)) return root_df<SwishT>(root_dx(x, k), dy);
        }
        float z = fmaxf(k.p * x, -kBig);
        return ((dy * tail_s64<P>(x, k)) * (1.f + z)) * kTwoM64;
    }
    // Backward plus the d alpha term dy x^2 s (1 - s).
    template <bool P>
    static __device__ __forceinline__ float df_da(float x, float dy, const Coef &k, bool &tail,
                                                  float &term)
    {
        float t;
        float E = expo<P>(x, k, t);
        tail |= t > kTailT;
        float s = rcp_ftz(1.f + E);
        float z = __fmul_rn(k.p, x);
        if constexpr (!P && RC) tail |= fabsf(__fsub_rn(t, kRootT)) < kRootWinT;
        float sm = z > 0.f ? E * s : 1.f - s;
        term = (((x * s) * sm) * x) * dy;
        z = fminf(z, kBig);
        return dy * fmaf(z * s, sm, s);
    }
    // As df_tail; near the zero of f' the d alpha term (a product, which does
    // not cancel) keeps its main-path value.
    template <bool P>
    static __device__ __forceinline__ float df_da_tail(float x, float dy, const Coef &k, float &term)
    {
        if constexpr (!P && RC) {
            if (near_root(x, k)) {
                bool unused = false;
                (void)df_da<P>(x, dy, k, unused, term);
                return root_df<SwishT>(root_dx(x, k), dy);
            }
        }
        float s64 = tail_s64<P>(x, k);
        float z = fmaxf(k.p * x, -kBig);
        term = (((x * s64) * x) * dy) * kTwoM64;
        return ((dy * s64) * (1.f + z)) * kTwoM64;
    }
};
using Swish = SwishT<true>;

}  // namespace mea
