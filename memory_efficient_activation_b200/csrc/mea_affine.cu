// mea_affine.cu -- fused per-channel affine + activation, forward and backward:
//
//   z = gamma_c x + beta_c,  y = f(z)
//   dz = dy f'(z),  dx = gamma_c dz,
//   dgamma_c = sum dz x,  dbeta_c = sum dz        (over all N H W positions)
//
// for every activation of the family (with Swish, alpha = the scalar
// parameter; the affine + Swish entry points use alpha = 1).  The data
// movement and the deterministic reductions are the per-channel kernels of
// mea_channel.cuh; this file supplies the arithmetic (AffineOp) and the
// dispatch over activation and storage dtype.
#include <type_traits>

#include "mea_channel.cuh"

namespace mea {

// Swish'(z) dy for two elements of bf16 storage, in the fewest packed
// .f32x2 operations: with E = 2^t = e^(-alpha z) and s = 1 / (1 + E),
// Sigmoid(-alpha z) = E s (a product, no cancellation on either side), and
//   dz = dy (s (1 + alpha z E s))
// (s times the bracket first: s may be as small as 2^-124, and dy s could
// fall below the normal range where the final result does not).
// Every finite product stays finite while |t| <= kTailT.  One u = t -
// Swish::kRootT gives both flags: |u| > Swish::kTailU (which contains |t| >
// kTailT: deep negative z, and z beyond +86 or +inf, where alpha z E s could
// be inf * 0) and |u| < Swish::kRootWinT (alpha z near the zero of Swish');
// the caller recomputes the flagged elements.  Rounding differs from the
// scalar form by a few fp32 ulps, far inside a bf16 ulp.
__device__ __forceinline__ void swish_df2_bf16(float z0, float z1, float d0, float d1, const Coef &k, bool &tail,
                                               float &o0, float &o1)
{
    const F2 z = pk(z0, z1);
    float t0, t1;
    upk(mul2(z, sp2(k.c_hi)), t0, t1);
    const float e0 = ex2_ftz(t0), e1 = ex2_ftz(t1);
    float u0, u1;
    upk(add2(pk(t0, t1), sp2(-Swish::kRootT)), u0, u1);
    tail |= (fabsf(u0) < Swish::kRootWinT) | (fabsf(u1) < Swish::kRootWinT) | (fabsf(u0) > Swish::kTailU) |
            (fabsf(u1) > Swish::kTailU);
    const F2 E = pk(e0, e1);
    float a0, a1;
    upk(add2(sp2(1.f), E), a0, a1);
    const F2 s = pk(rcp_ftz(a0), rcp_ftz(a1));
    const F2 r = fma2(mul2(sp2(k.p), z), mul2(E, s), sp2(1.f));
    upk(mul2(pk(d0, d1), mul2(s, r)), o0, o1);
}

// Swish (y = z Sigmoid(alpha z)) and the sigmoid for two elements of bf16
// storage: the operations of Swish::f<false> / Sigmoid::f<false> with the
// multiplies and adds as packed .f32x2 pairs, bitwise the scalar results.
__device__ __forceinline__ F2 sigmoid_parts2(F2 z, const Coef &k, bool &tail)
{
    float t0, t1;
    upk(mul2(z, sp2(k.c_hi)), t0, t1);
    const float e0 = ex2_ftz(t0), e1 = ex2_ftz(t1);
    tail |= (t0 > kTailT) | (t1 > kTailT);
    float a0, a1;
    upk(add2(sp2(1.f), pk(e0, e1)), a0, a1);
    return pk(rcp_ftz(a0), rcp_ftz(a1));
}

// GELU-tanh for two elements of bf16 storage: t = z (c1 + c3 z^2) as in
// GeluTanh, E = 2^t, s = 1 / (1 + E) = Sigmoid(v), Sigmoid(-v) = E s, and
//   y = z s,   dz = dy (s (1 + z v' E s)),  v' = k1 + 3 k3 z^2,
// The forward flags t > kTailT (deep negative z) for the tail form; the
// backward uses swish_df2_bf16's two guards on u = t - GeluTanh::kRootT
// (inside them z v' E s is finite and z is away from the zero of f').
template <bool kBothSides>
__device__ __forceinline__ F2 gelu_tanh_parts2(F2 z, F2 &z2, bool &tail, F2 &E)
{
    z2 = mul2(z, z);
    float t0, t1;
    upk(mul2(z, fma2(sp2(GeluTanh::kC3f), z2, sp2(GeluTanh::kC1f))), t0, t1);
    const float e0 = ex2_ftz(t0), e1 = ex2_ftz(t1);
    if constexpr (kBothSides) {
        // backward: the guards of swish_df2_bf16, on GeluTanh's constants
        float u0, u1;
        upk(add2(pk(t0, t1), sp2(-GeluTanh::kRootT)), u0, u1);
        tail |= (fabsf(u0) < GeluTanh::kRootWinT) | (fabsf(u1) < GeluTanh::kRootWinT) |
                (fabsf(u0) > GeluTanh::kTailU) | (fabsf(u1) > GeluTanh::kTailU);
    } else {
        tail |= (t0 > kTailT) | (t1 > kTailT);
    }
    E = pk(e0, e1);
    float a0, a1;
    upk(add2(sp2(1.f), E), a0, a1);
    return pk(rcp_ftz(a0), rcp_ftz(a1));
}
__device__ __forceinline__ void gelu_tanh_f2_bf16(float z0, float z1, bool &tail, float &o0, float &o1)
{
    const F2 z = pk(z0, z1);
    F2 z2, E;
    upk(mul2(z, gelu_tanh_parts2<false>(z, z2, tail, E)), o0, o1);
}
__device__ __forceinline__ void gelu_tanh_df2_bf16(float z0, float z1, float d0, float d1, bool &tail, float &o0,
                                                   float &o1)
{
    const F2 z = pk(z0, z1);
    F2 z2, E;
    const F2 s = gelu_tanh_parts2<true>(z, z2, tail, E);
    const F2 q = mul2(z, fma2(sp2(GeluTanh::kK3x3f), z2, sp2(GeluTanh::kK1f)));
    const F2 r = fma2(q, mul2(E, s), sp2(1.f));
    upk(mul2(pk(d0, d1), mul2(s, r)), o0, o1);
}

template <class A>
struct AffineOp {
    static constexpr int NR = 2;   // dgamma, dbeta
    using K = Coef;
    struct Ch {
        float g, b;
    };
    static __device__ __forceinline__ K kcoef(const ChanArgs &a) { return A::coef(a.scalar); }
    static __device__ __forceinline__ Ch load(const ChanArgs &a, int c) { return Ch{__ldg(a.p0 + c), __ldg(a.p1 + c)}; }
    static __device__ __forceinline__ float z(float x, const Ch &h) { return fmaf(h.g, x, h.b); }

    template <bool P>
    static __device__ __forceinline__ float f(float x, const K &k, const Ch &h, bool &tail)
    {
        return A::template f<P>(z(x, h), k, tail);
    }
    template <bool P>
    static __device__ __forceinline__ float f_tail(float x, const K &k, const Ch &h)
    {
        return A::template f_tail<P>(z(x, h), k);
    }
    static __device__ __forceinline__ bool is_tail(float x, const K &k, const Ch &h) { return A::is_tail(z(x, h), k); }
    // Every element the backward main paths (scalar or packed) may flag: the
    // deep tails, the packed forms' overflow guards and, with bf16 storage,
    // the neighbourhood of the zero of f'.  Only these are recomputed.
    template <bool P>
    static __device__ __forceinline__ bool flag_bwd(float x, const K &k, const Ch &h)
    {
        const float zz = z(x, h);
        if constexpr (!P && A::kHasRoot) return A::template bwd_flagged<P>(zz, k) || A::near_root(zz, k);
        return A::template bwd_flagged<P>(zz, k);
    }
    // o = dz
    template <bool P>
    static __device__ __forceinline__ void bwd(float x, float dy, const K &k, const Ch &h, bool &tail, float &o,
                                               float &)
    {
        const float zz = z(x, h);
        o = A::template df<P>(zz, dy, k, tail);
        if constexpr (!P && A::kHasRoot) tail |= A::near_root(zz, k);
    }
    // A flagged element: near the zero of f' (bf16 storage), d = v - v0 from
    // z = gamma x + beta formed in fp64 and f' from its Taylor polynomial
    // there; in the deep tail the scaled tail form; else (a packed form's
    // overflow guard) the scalar main form.
    template <bool P>
    static __device__ __forceinline__ void bwd_tail(float x, float dy, const K &k, const Ch &h, float &o, float &)
    {
        const float zz = z(x, h);
        if constexpr (!P && A::kHasRoot) {
            if (A::near_root(zz, k)) {
                o = root_df<A>(root_d(h.g, x, h.b, A::root_scale(k), A::kRootD), dy);
                return;
            }
        }
        if (A::is_tail(zz, k)) {
            o = A::template df_tail<P>(zz, dy, k);
            return;
        }
        bool unused = false;
        o = A::template df<P>(zz, dy, k, unused);
    }
    static __device__ __forceinline__ float finish(float x, float o, float, const Ch &h, float (&acc)[NR])
    {
        acc[0] = fmaf(o, x, acc[0]);   // dz x
        acc[1] += o;                   // dz
        return h.g * o;                // dx
    }

    // Two channels at once: the affine, the reduction terms and dx as packed
    // .f32x2 operations (bitwise the scalar results); f' pairwise where the
    // activation provides it, else per element.
    struct Ch2 {
        F2 g, b;
    };
    static __device__ __forceinline__ Ch2 pair(const Ch &a, const Ch &c) { return Ch2{pk(a.g, c.g), pk(a.b, c.b)}; }
    template <bool P>
    static __device__ __forceinline__ F2 f2(F2 x, const K &k, const Ch2 &h, bool &tail)
    {
        float z0, z1, o0, o1;
        upk(fma2(h.g, x, h.b), z0, z1);
        if constexpr (HasPairs<A, P>::value) {
            A::f2(z0, z1, k, tail, o0, o1);
        } else if constexpr (std::is_same<A, GeluTanh>::value && !P) {
            gelu_tanh_f2_bf16(z0, z1, tail, o0, o1);
        } else if constexpr (std::is_same<A, Swish>::value && !P) {
            const F2 z = pk(z0, z1);
            upk(mul2(z, sigmoid_parts2(z, k, tail)), o0, o1);
        } else if constexpr (std::is_same<A, Sigmoid>::value && !P) {
            upk(sigmoid_parts2(pk(z0, z1), k, tail), o0, o1);
        } else {
            o0 = A::template f<P>(z0, k, tail);
            o1 = A::template f<P>(z1, k, tail);
        }
        return pk(o0, o1);
    }
    template <bool P>
    static __device__ __forceinline__ void bwd2(F2 x, F2 dy, const K &k, const Ch2 &h, bool &tail, F2 &o, F2 &)
    {
        float z0, z1, d0, d1, o0, o1;
        const F2 zp = fma2(h.g, x, h.b);
        upk(zp, z0, z1);
        upk(dy, d0, d1);
        if constexpr (!P && std::is_same<A, GeluErf>::value) {
            // the same test as A::near_root, on both elements (the packed
            // Swish and GELU-tanh forms test their own exponent instead)
            float e0, e1;
            upk(add2(zp, sp2(-A::kRootHi)), e0, e1);
            tail |= (fabsf(e0) < kRootWin) | (fabsf(e1) < kRootWin);
        }
        if constexpr (HasPairs<A, P>::value) {
            A::df2(z0, z1, d0, d1, k, tail, o0, o1);
        } else if constexpr (std::is_same<A, Swish>::value && !P) {
            swish_df2_bf16(z0, z1, d0, d1, k, tail, o0, o1);
        } else if constexpr (std::is_same<A, GeluTanh>::value && !P) {
            gelu_tanh_df2_bf16(z0, z1, d0, d1, tail, o0, o1);
        } else {
            o0 = A::template df<P>(z0, d0, k, tail);
            o1 = A::template df<P>(z1, d1, k, tail);
        }
        o = pk(o0, o1);
    }
    static __device__ __forceinline__ F2 finish2(F2 x, F2 o, F2, const Ch2 &h, F2 (&acc)[NR])
    {
        acc[0] = fma2(o, x, acc[0]);
        acc[1] = add2(acc[1], o);
        return mul2(h.g, o);
    }
};

template <typename T, int MODE>
static cudaError_t by_act(const AffineLaunch &a)
{
    const ChanArgs ca{a.gamma, a.beta, a.param};
    switch (a.act) {
    case 0: return launch_channel<AffineOp<ReLU>, T, MODE>(a, ca, a.dgamma, a.dbeta);
    case 1: return launch_channel<AffineOp<LeakyReLU>, T, MODE>(a, ca, a.dgamma, a.dbeta);
    case 2: return launch_channel<AffineOp<Sigmoid>, T, MODE>(a, ca, a.dgamma, a.dbeta);
    case 3: return launch_channel<AffineOp<Tanh>, T, MODE>(a, ca, a.dgamma, a.dbeta);
    case 4: return launch_channel<AffineOp<GeluErf>, T, MODE>(a, ca, a.dgamma, a.dbeta);
    case 5: return launch_channel<AffineOp<GeluTanh>, T, MODE>(a, ca, a.dgamma, a.dbeta);
    case 6: return launch_channel<AffineOp<Swish>, T, MODE>(a, ca, a.dgamma, a.dbeta);
    }
    return cudaErrorInvalidValue;
}

size_t affine_bwd_workspace_bytes(int dtype, int layout, int64_t N, int64_t C, int64_t H, int64_t W)
{
    return chan_bwd_workspace_bytes(AffineOp<Swish>::NR, dtype, layout, N, C, H, W);
}

cudaError_t launch_affine_fwd(const AffineLaunch &a)
{
    return a.dtype == kBF16 ? by_act<Bf16, 0>(a) : by_act<float, 0>(a);
}

cudaError_t launch_affine_bwd(const AffineLaunch &a)
{
    return a.dtype == kBF16 ? by_act<Bf16, 1>(a) : by_act<float, 1>(a);
}

cudaError_t launch_affine_bwd_wait_selftest(const AffineLaunch &a)
{
    const ChanArgs ca{a.gamma, a.beta, 1.f};
    return a.dtype == kBF16 ? launch_channel_wait_selftest<AffineOp<Swish>, Bf16>(a, ca)
                            : launch_channel_wait_selftest<AffineOp<Swish>, float>(a, ca);
}

}  // namespace mea
