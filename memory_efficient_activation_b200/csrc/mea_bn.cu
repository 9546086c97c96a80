// mea_bn.cu -- channel concatenation + batch normalization (batch
// statistics) + ReLU without the concatenated tensor, and with its output
// only in a caller-owned buffer that the backward re-populates.
//
// "A memory-efficient implementation of DenseNets", section "Motivation":
// every concatenation and batch-normalization output of a DenseNet goes into
// shared allocations reused by all layers, and the backward re-populates
// them from the layer inputs, which turns the feature-map memory from
// quadratic to linear in depth.  Here the concatenation is never formed:
// the kernels read the pieces in place through a table of (pointer, channel
// offset), so the only per-layer state kept for the backward is the batch
// mean and inverse standard deviation (2 C floats).
//
//   forward   bn_stats_kernel      per (channel, batch slice): sums of d =
//                                  x - shift and d^2 (shift: one element of
//                                  the channel), fp32 within a 16-byte
//                                  vector, fp64 across -> partials
//             bn_apply_kernel      in its prologue, per channel, slices in
//                                  order: mean, invstd = 1 / sqrt(var +
//                                  eps), running statistics (momentum;
//                                  unbiased variance); then y = max(gamma' x
//                                  + beta', 0), gamma' = gamma invstd, beta'
//                                  = beta - mean gamma'
//   backward  bn_bwd_reduce_kernel per (channel, slice): recompute the ReLU
//                                  mask from x; sums of dz and dz xhat
//                                  (fp32 within a vector, fp64 across)
//             bn_dx_kernel         in its prologue dbeta, dgamma and the
//                                  coefficients of dx; then dx = gamma invstd
//                                  (dz - dbeta / n - xhat dgamma / n),
//                                  written or added into the pieces'
//                                  gradients
// Blocks own (channel c, slice s of the batch) and stream the contiguous
// H W planes of that channel (16-byte vectors when a plane is a multiple of
// 16 bytes and the pieces are aligned), four items in flight per thread,
// (sample, position) from the item index by a multiply-shift division.  All sums are per block in a fixed
// order and combined per channel in slice order: bitwise reproducible.
#include <cuda_runtime.h>

#include <cstdint>

#include "mea_bn_api.h"
#include "mea_device.cuh"
#include "mea_internal.h"
#include "mea_math.cuh"
#include "mea_stream.cuh"

namespace mea {
namespace {

constexpr int kBnThreads = 256;
constexpr int kBnBlocksTarget = 1184;     // C * S is sized to about this many blocks (148 x 8)

int bn_slices(int64_t N, int64_t C)
{
    int64_t s = (kBnBlocksTarget + C - 1) / C;
    if (s > N) s = N;
    if (s < 1) s = 1;
    return (int)s;
}

// Piece holding global channel c (one thread searches, the block shares it).
__device__ __forceinline__ int piece_of(const BnPieces &t, int c)
{
    int lo = 0, hi = t.npieces - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (t.off[mid] <= c) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

struct PlaneJob {
    int64_t c, n0, n1;
    int piece, j, k;     // piece index, channel within the piece, channels of the piece
};

__device__ __forceinline__ PlaneJob plane_job(const BnPieces &t, int64_t N, int slices)
{
    __shared__ int sp;
    PlaneJob p;
    p.c = blockIdx.x / slices;
    const int s = blockIdx.x % slices;
    p.n0 = (int64_t)s * N / slices;
    p.n1 = (int64_t)(s + 1) * N / slices;
    if (threadIdx.x == 0) sp = piece_of(t, (int)p.c);
    __syncthreads();
    p.piece = sp;
    p.j = (int)p.c - t.off[p.piece];
    p.k = t.off[p.piece + 1] - t.off[p.piece];
    return p;
}

// L2 priority of a pass's loads.  Within one call the statistics pass and
// the apply pass (and the backward's sums and dx) read the same x (and dy)
// back to back.  The first pass loads with an evict-last policy and the
// second with evict-first, so the lines the second pass needs outrank the
// rest of the traffic while it runs and are released as it consumes them;
// part of its reads then come from the 126 MB L2 instead of HBM.  (A hint
// only: the results are the same.)
__device__ __forceinline__ uint64_t l2_policy_last()
{
    uint64_t p;
    asm("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t l2_policy_first()
{
    uint64_t p;
    asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
template <typename T, int VL>
__device__ __forceinline__ typename Item<T, VL>::Raw load_hint(const void *p, int64_t i, uint64_t pol)
{
    if constexpr (VL == 1) {
        return Item<T, VL>::load(p, i);
    } else {
        uint4 r;
        asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                     : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                     : "l"(static_cast<const uint4 *>(p) + i), "l"(pol));
        return r;
    }
}

constexpr int kBnUnroll = 4;     // items in flight per thread

// Runs f over the block's planes in items of VL elements (one 16-byte vector,
// or one element), kBnUnroll items per thread per step: f.step gets each
// item's index in the piece (ii) and in the concatenation (io), in item
// units, and whether it exists (ok).  Thread t takes items t, t + bd, t + 2
// bd, ... of the block's planes laid end to end.
//
// When a plane holds at least bd items (and every index fits in 32 bits),
// one step of bd items crosses at most one plane boundary, so the plane
// offset and both indices advance by additions alone; otherwise each item's
// (plane, offset) comes from a multiply-shift division.  Both visit the same
// items in the same order.
template <int VL, class F>
__device__ __forceinline__ void stream_items(const PlaneJob &p, int64_t C, int64_t HW, F &f)
{
    const uint32_t per = (uint32_t)(HW / VL);
    const uint32_t total = (uint32_t)(p.n1 - p.n0) * per;
    const uint32_t bd = blockDim.x;
    const bool fits = (uint64_t)(p.n1 * C) * per < (1ull << 31);
    if (per >= bd && fits) {
        uint32_t v = threadIdx.x;
        uint32_t ii = (uint32_t)((p.n0 * p.k + p.j) * per) + v;
        uint32_t io = (uint32_t)((p.n0 * C + p.c) * per) + v;
        const uint32_t ii_skip = (uint32_t)(p.k - 1) * per, io_skip = (uint32_t)(C - 1) * per;
        for (uint32_t q0 = threadIdx.x; q0 < total; q0 += kBnUnroll * bd) {
            int64_t iu[kBnUnroll], ou[kBnUnroll];
            bool ok[kBnUnroll];
#pragma unroll
            for (int u = 0; u < kBnUnroll; ++u) {
                ok[u] = q0 + u * bd < total;
                iu[u] = ii;
                ou[u] = io;
                v += bd;
                ii += bd;
                io += bd;
                if (v >= per) {
                    v -= per;
                    ii += ii_skip;
                    io += io_skip;
                }
            }
            f.step(iu, ou, ok);
        }
        return;
    }
    const DivU32 div(per);
    for (uint32_t q0 = threadIdx.x; q0 < total; q0 += kBnUnroll * bd) {
        int64_t ii[kBnUnroll], io[kBnUnroll];
        bool ok[kBnUnroll];
#pragma unroll
        for (int u = 0; u < kBnUnroll; ++u) {
            const uint32_t q = q0 + u * bd;
            ok[u] = q < total;
            uint32_t nr, v;
            div.divmod(ok[u] ? q : 0u, nr, v);
            const int64_t n = p.n0 + nr;
            ii[u] = (n * p.k + p.j) * per + v;
            io[u] = (n * C + p.c) * per + v;
        }
        f.step(ii, io, ok);
    }
}

// One 16-byte item as packed .f32x2 pairs (4 for bf16, 2 for fp32), so the
// per-element arithmetic of the vector path takes half the instructions.
template <typename T>
struct Pairs;
template <>
struct Pairs<Bf16> {
    static constexpr int N = 4;
    static __device__ __forceinline__ void unpack(const uint4 &w, F2 (&p)[N])
    {
        const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) p[q] = pk(__uint_as_float(u[q] << 16), __uint_as_float(u[q] & 0xffff0000u));
    }
    static __device__ __forceinline__ uint4 pack(const F2 (&p)[N])
    {
        uint32_t u[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float lo, hi;
            upk(p[q], lo, hi);
            u[q] = pack_bf16x2(lo, hi);
        }
        return make_uint4(u[0], u[1], u[2], u[3]);
    }
};
template <>
struct Pairs<float> {
    static constexpr int N = 2;
    static __device__ __forceinline__ void unpack(const uint4 &w, F2 (&p)[N])
    {
        p[0] = pk(__uint_as_float(w.x), __uint_as_float(w.y));
        p[1] = pk(__uint_as_float(w.z), __uint_as_float(w.w));
    }
    static __device__ __forceinline__ uint4 pack(const F2 (&p)[N])
    {
        float a, b, c, d;
        upk(p[0], a, b);
        upk(p[1], c, d);
        return make_uint4(__float_as_uint(a), __float_as_uint(b), __float_as_uint(c), __float_as_uint(d));
    }
};

// A ReLU mask on two elements: d where z > 0, else 0 (the forward's test).
__device__ __forceinline__ F2 relu_pass2(F2 z, F2 d)
{
    float z0, z1, d0, d1;
    upk(z, z0, z1);
    upk(d, d0, d1);
    return pk(z0 > 0.f ? d0 : 0.f, z1 > 0.f ? d1 : 0.f);
}

template <typename T, class F>
__device__ __forceinline__ void for_planes(const PlaneJob &p, int64_t C, int64_t HW, bool vec, F &f)
{
    if (vec) {
        auto fv = f.template items<Store<T>::V>();
        stream_items<Store<T>::V>(p, C, HW, fv);
        f.absorb(fv);
    } else {
        auto fs = f.template items<1>();
        stream_items<1>(p, C, HW, fs);
        f.absorb(fs);
    }
}

// ------------------------------------------------------------ forward

// Sums of d = x - shift and d^2: fp32 within an item, fp64 across items.
// shift is one element of the channel (the same for every block of the
// channel), which keeps E[d^2] near the variance however large the mean.
template <typename T>
struct StatsF {
    const void *x;
    float shift;
    double s1 = 0.0, s2 = 0.0;
    template <int VL>
    struct It {
        const void *x;
        float shift;
        double s1 = 0.0, s2 = 0.0;
        __device__ __forceinline__ void step(const int64_t (&ii)[kBnUnroll], const int64_t (&)[kBnUnroll],
                                             const bool (&ok)[kBnUnroll])
        {
            typename Item<T, VL>::Raw xr[kBnUnroll];
#pragma unroll
            for (int u = 0; u < kBnUnroll; ++u)
                if (ok[u]) xr[u] = load_hint<T, VL>(x, ii[u], l2_policy_last());
#pragma unroll
            for (int u = 0; u < kBnUnroll; ++u) {
                if (!ok[u]) continue;
                float a = 0.f, b = 0.f;
                if constexpr (VL == 1) {
                    const float d = xr[u] - shift;
                    a = d;
                    b = d * d;
                } else {
                    // fp32 within the item: each lane sums every other element
                    F2 xp[Pairs<T>::N];
                    Pairs<T>::unpack(xr[u], xp);
                    F2 a2 = sp2(0.f), b2 = sp2(0.f);
#pragma unroll
                    for (int q = 0; q < Pairs<T>::N; ++q) {
                        const F2 d = add2(xp[q], sp2(-shift));
                        a2 = add2(a2, d);
                        b2 = fma2(d, d, b2);
                    }
                    float a0, a1, b0, b1;
                    upk(a2, a0, a1);
                    upk(b2, b0, b1);
                    a = a0 + a1;
                    b = b0 + b1;
                }
                s1 += (double)a;
                s2 += (double)b;
            }
        }
    };
    template <int VL>
    __device__ __forceinline__ It<VL> items() const
    {
        return It<VL>{x, shift};
    }
    template <class I>
    __device__ __forceinline__ void absorb(const I &i)
    {
        s1 = i.s1;
        s2 = i.s2;
    }
};

__device__ __forceinline__ int64_t first_of_channel(const BnPieces &t, const PlaneJob &p, int64_t HW)
{
    (void)t;
    return (int64_t)p.j * HW;       // sample 0, channel j of the piece, element 0
}

template <typename T>
__global__ void __launch_bounds__(kBnThreads, 6)
bn_stats_kernel(BnPieces t, int64_t N, int64_t C, int64_t HW, int slices, int vec, double *__restrict__ partials)
{
    pdl_wait();
    const PlaneJob p = plane_job(t, N, slices);
    const void *x = t.ptr[p.piece];
    StatsF<T> f{x, Store<T>::load1(x, first_of_channel(t, p, HW))};
    for_planes<T>(p, C, HW, vec, f);
    pdl_trigger();
    __shared__ double red[32];
    const double a = block_sum(f.s1, red);
    const double b = block_sum(f.s2, red);
    if (threadIdx.x == 0) {
        partials[3 * blockIdx.x] = a;
        partials[3 * blockIdx.x + 1] = b;
        partials[3 * blockIdx.x + 2] = (double)f.shift;
    }
}

// Batch statistics of channel c from its slices' partials, slices in order:
// mean, invstd = 1 / sqrt(var + eps) (rounded to fp32), and with `write` the
// stored mean, invstd and running statistics (momentum; unbiased variance).
struct BnFin {
    double n;
    float eps, momentum;
    float *running_mean, *running_var;
};

__device__ __forceinline__ void bn_finalize(const double *__restrict__ partials, int64_t c, int slices, const BnFin &f,
                                         bool write, float *__restrict__ mean, float *__restrict__ invstd,
                                         float &mu_out, float &r_out)
{
    double s1 = 0.0, s2 = 0.0;
    for (int s = 0; s < slices; ++s) {
        s1 += __ldcg(partials + 3 * (c * slices + s));
        s2 += __ldcg(partials + 3 * (c * slices + s) + 1);
    }
    const double shift = __ldcg(partials + 3 * c * slices + 2);
    const double md = s1 / f.n;               // mean of d = x - shift
    double var = s2 / f.n - md * md;
    if (var < 0.0) var = 0.0;
    const double mu = shift + md;
    mu_out = (float)mu;
    r_out = (float)(1.0 / sqrt(var + (double)f.eps));
    if (!write) return;
    mean[c] = mu_out;
    invstd[c] = r_out;
    if (f.running_mean) {
        const double unbiased = f.n > 1.0 ? var * f.n / (f.n - 1.0) : var;
        f.running_mean[c] = (float)((1.0 - f.momentum) * f.running_mean[c] + f.momentum * mu);
        f.running_var[c] = (float)((1.0 - f.momentum) * f.running_var[c] + f.momentum * unbiased);
    }
}

template <typename T>
struct ApplyF {
    const void *x;
    void *y;
    float g, b;
    template <int VL>
    struct It {
        const void *x;
        void *y;
        float g, b;
        __device__ __forceinline__ void step(const int64_t (&ii)[kBnUnroll], const int64_t (&io)[kBnUnroll],
                                             const bool (&ok)[kBnUnroll])
        {
            typename Item<T, VL>::Raw xr[kBnUnroll];
#pragma unroll
            for (int u = 0; u < kBnUnroll; ++u)
                if (ok[u]) xr[u] = load_hint<T, VL>(x, ii[u], l2_policy_first());
#pragma unroll
            for (int u = 0; u < kBnUnroll; ++u) {
                if (!ok[u]) continue;
                if constexpr (VL == 1) {
                    const float of[1] = {fmaxf(fmaf(g, xr[u], b), 0.f)};
                    Item<T, VL>::store(y, io[u], of);
                } else {
                    F2 xp[Pairs<T>::N];
                    Pairs<T>::unpack(xr[u], xp);
#pragma unroll
                    for (int q = 0; q < Pairs<T>::N; ++q) {
                        float z0, z1;
                        upk(fma2(sp2(g), xp[q], sp2(b)), z0, z1);
                        xp[q] = pk(fmaxf(z0, 0.f), fmaxf(z1, 0.f));
                    }
                    st_v4(static_cast<uint4 *>(y) + io[u], Pairs<T>::pack(xp));
                }
            }
        }
    };
    template <int VL>
    __device__ __forceinline__ It<VL> items() const
    {
        return It<VL>{x, y, g, b};
    }
    template <class I>
    __device__ __forceinline__ void absorb(const I &)
    {
    }
};

// With partials (the forward): the block's thread 0 first forms the
// channel's statistics from them (bn_finalize), and the slice-0 block of
// each channel stores them; without (the re-population): mean and invstd
// are read.  Either way the same fp32 values enter the same arithmetic.
template <typename T>
__global__ void __launch_bounds__(kBnThreads, 6)
bn_apply_kernel(BnPieces t, int64_t N, int64_t C, int64_t HW, int slices, int vec, const float *__restrict__ gamma,
                const float *__restrict__ beta, float *__restrict__ mean, float *__restrict__ invstd,
                void *__restrict__ y, const double *__restrict__ partials, BnFin fin)
{
    __shared__ float stat[2];
    pdl_wait();
    const PlaneJob p = plane_job(t, N, slices);
    float mu, r;
    if (partials) {
        if (threadIdx.x == 0)
            bn_finalize(partials, p.c, slices, fin, blockIdx.x % slices == 0, mean, invstd, stat[0], stat[1]);
        __syncthreads();
        mu = stat[0];
        r = stat[1];
    } else {
        mu = mean[p.c];
        r = invstd[p.c];
    }
    const float gp = gamma[p.c] * r;
    ApplyF<T> f{t.ptr[p.piece], y, gp, fmaf(-mu, gp, beta[p.c])};
    for_planes<T>(p, C, HW, vec, f);
    pdl_trigger();
}

// ------------------------------------------------------------ backward

// dz and xhat of one element, recomputed from x: z = gamma' x + beta' (the
// forward's arithmetic, so the ReLU mask is the forward's).
struct BwdCoef {
    float gp, bp, mu, r;
};

__device__ __forceinline__ BwdCoef bwd_coef(const float *gamma, const float *beta, const float *mean,
                                            const float *invstd, int64_t c)
{
    BwdCoef k;
    k.mu = mean[c];
    k.r = invstd[c];
    k.gp = gamma[c] * k.r;
    k.bp = fmaf(-k.mu, k.gp, beta[c]);
    return k;
}

template <typename T>
struct ReduceF {
    const void *x;
    const void *dy;
    BwdCoef k;
    double s1 = 0.0, s2 = 0.0;
    template <int VL>
    struct It {
        const void *x;
        const void *dy;
        BwdCoef k;
        double s1 = 0.0, s2 = 0.0;
        __device__ __forceinline__ void step(const int64_t (&ii)[kBnUnroll], const int64_t (&io)[kBnUnroll],
                                             const bool (&ok)[kBnUnroll])
        {
            typename Item<T, VL>::Raw xr[kBnUnroll], gr[kBnUnroll];
#pragma unroll
            for (int u = 0; u < kBnUnroll; ++u)
                if (ok[u]) {
                    xr[u] = load_hint<T, VL>(x, ii[u], l2_policy_last());
                    gr[u] = load_hint<T, VL>(dy, io[u], l2_policy_last());
                }
#pragma unroll
            for (int u = 0; u < kBnUnroll; ++u) {
                if (!ok[u]) continue;
                float a = 0.f, b = 0.f;
                if constexpr (VL == 1) {
                    const float dz = fmaf(k.gp, xr[u], k.bp) > 0.f ? gr[u] : 0.f;
                    a = dz;
                    b = dz * ((xr[u] - k.mu) * k.r);
                } else {
                    F2 xp[Pairs<T>::N], gp[Pairs<T>::N];
                    Pairs<T>::unpack(xr[u], xp);
                    Pairs<T>::unpack(gr[u], gp);
                    F2 a2 = sp2(0.f), b2 = sp2(0.f);
#pragma unroll
                    for (int q = 0; q < Pairs<T>::N; ++q) {
                        const F2 dz = relu_pass2(fma2(sp2(k.gp), xp[q], sp2(k.bp)), gp[q]);
                        a2 = add2(a2, dz);
                        b2 = fma2(dz, mul2(add2(xp[q], sp2(-k.mu)), sp2(k.r)), b2);
                    }
                    float a0, a1, b0, b1;
                    upk(a2, a0, a1);
                    upk(b2, b0, b1);
                    a = a0 + a1;
                    b = b0 + b1;
                }
                s1 += (double)a;
                s2 += (double)b;
            }
        }
    };
    template <int VL>
    __device__ __forceinline__ It<VL> items() const
    {
        return It<VL>{x, dy, k};
    }
    template <class I>
    __device__ __forceinline__ void absorb(const I &i)
    {
        s1 = i.s1;
        s2 = i.s2;
    }
};

template <typename T>
__global__ void __launch_bounds__(kBnThreads, 4)
bn_bwd_reduce_kernel(BnPieces t, const void *__restrict__ dy, int64_t N, int64_t C, int64_t HW, int slices, int vec,
                     const float *__restrict__ gamma, const float *__restrict__ beta, const float *__restrict__ mean,
                     const float *__restrict__ invstd, double *__restrict__ partials)
{
    pdl_wait();
    const PlaneJob p = plane_job(t, N, slices);
    ReduceF<T> f{t.ptr[p.piece], dy, bwd_coef(gamma, beta, mean, invstd, p.c)};
    for_planes<T>(p, C, HW, vec, f);
    pdl_trigger();
    __shared__ double red[32];
    const double a = block_sum(f.s1, red);
    const double b = block_sum(f.s2, red);
    if (threadIdx.x == 0) {
        partials[3 * blockIdx.x] = a;
        partials[3 * blockIdx.x + 1] = b;
    }
}

// dbeta, dgamma (stored with `write`), and the coefficients of dx = a dz + b +
// c xhat: a = gamma r, b = -a dbeta / n, c = -a dgamma / n, from channel c's
// slices in order.
__device__ __forceinline__ void bn_bwd_finalize(const double *__restrict__ partials, int64_t c, int slices, double n,
                                             const float *__restrict__ gamma, const float *__restrict__ invstd,
                                             bool write, float *__restrict__ dgamma, float *__restrict__ dbeta,
                                             float (&coef)[3])
{
    double s1 = 0.0, s2 = 0.0;
    for (int s = 0; s < slices; ++s) {
        s1 += __ldcg(partials + 3 * (c * slices + s));
        s2 += __ldcg(partials + 3 * (c * slices + s) + 1);
    }
    if (write) {
        dbeta[c] = (float)s1;
        dgamma[c] = (float)s2;
    }
    const double a = (double)gamma[c] * (double)invstd[c];
    coef[0] = (float)a;
    coef[1] = (float)(-a * s1 / n);
    coef[2] = (float)(-a * s2 / n);
}

// ACC: add d to what dx already holds (a fixed choice per launch, so the
// plain instance carries no read of dx).
template <typename T, bool ACC>
struct DxF {
    const void *x;
    const void *dy;
    void *dx;
    BwdCoef k;
    float a, b, cc;
    template <int VL>
    struct It {
        const void *x;
        const void *dy;
        void *dx;
        BwdCoef k;
        float a, b, cc;
        __device__ __forceinline__ void step(const int64_t (&ii)[kBnUnroll], const int64_t (&io)[kBnUnroll],
                                             const bool (&ok)[kBnUnroll])
        {
            typename Item<T, VL>::Raw xr[kBnUnroll], gr[kBnUnroll];
#pragma unroll
            for (int u = 0; u < kBnUnroll; ++u)
                if (ok[u]) {
                    xr[u] = load_hint<T, VL>(x, ii[u], l2_policy_first());
                    gr[u] = load_hint<T, VL>(dy, io[u], l2_policy_first());
                }
#pragma unroll
            for (int u = 0; u < kBnUnroll; ++u) {
                if (!ok[u]) continue;
                if constexpr (VL == 1) {
                    const float dz = fmaf(k.gp, xr[u], k.bp) > 0.f ? gr[u] : 0.f;
                    const float d = fmaf(a, dz, fmaf(cc, (xr[u] - k.mu) * k.r, b));
                    const float of[1] = {ACC ? Item<T, VL>::load_rw(dx, ii[u]) + d : d};
                    Item<T, VL>::store(dx, ii[u], of);
                } else {
                    F2 xp[Pairs<T>::N], gp[Pairs<T>::N], pp[Pairs<T>::N];
                    Pairs<T>::unpack(xr[u], xp);
                    Pairs<T>::unpack(gr[u], gp);
                    if constexpr (ACC) Pairs<T>::unpack(Item<T, VL>::load_rw(dx, ii[u]), pp);
#pragma unroll
                    for (int q = 0; q < Pairs<T>::N; ++q) {
                        const F2 dz = relu_pass2(fma2(sp2(k.gp), xp[q], sp2(k.bp)), gp[q]);
                        const F2 xh = mul2(add2(xp[q], sp2(-k.mu)), sp2(k.r));
                        const F2 d = fma2(sp2(a), dz, fma2(sp2(cc), xh, sp2(b)));
                        if constexpr (ACC) xp[q] = add2(pp[q], d);
                        else xp[q] = d;
                    }
                    st_v4(static_cast<uint4 *>(dx) + ii[u], Pairs<T>::pack(xp));
                }
            }
        }
    };
    template <int VL>
    __device__ __forceinline__ It<VL> items() const
    {
        return It<VL>{x, dy, dx, k, a, b, cc};
    }
    template <class I>
    __device__ __forceinline__ void absorb(const I &)
    {
    }
};

// The block's thread 0 first forms the channel's coefficients from the
// reduce kernel's partials (bn_bwd_finalize); the slice-0 block of each
// channel stores dgamma and dbeta.
template <typename T, bool ACC>
__global__ void __launch_bounds__(kBnThreads, 4)
bn_dx_kernel(BnPieces t, BnOutPieces d, const void *__restrict__ dy, int64_t N, int64_t C, int64_t HW, int slices,
             int vec, const float *__restrict__ gamma, const float *__restrict__ beta, const float *__restrict__ mean,
             const float *__restrict__ invstd, const double *__restrict__ partials, float *__restrict__ dgamma,
             float *__restrict__ dbeta)
{
    __shared__ float cf[3];
    pdl_wait();
    const PlaneJob p = plane_job(t, N, slices);
    if (threadIdx.x == 0) {
        float k3[3];
        bn_bwd_finalize(partials, p.c, slices, (double)(N * HW), gamma, invstd, blockIdx.x % slices == 0, dgamma,
                        dbeta, k3);
        cf[0] = k3[0];
        cf[1] = k3[1];
        cf[2] = k3[2];
    }
    __syncthreads();
    DxF<T, ACC> f{t.ptr[p.piece], dy, d.ptr[p.piece], bwd_coef(gamma, beta, mean, invstd, p.c), cf[0], cf[1], cf[2]};
    for_planes<T>(p, C, HW, vec, f);
    pdl_trigger();
}

// ------------------------------------------------------------ launchers

bool vec_ok(const BnLaunch &a, int bytes, bool with_d)
{
    if ((a.HW * bytes) % 16) return false;
    uintptr_t al = 0;
    for (int i = 0; i < a.in.npieces; ++i) {
        al |= reinterpret_cast<uintptr_t>(a.in.ptr[i]);
        if (with_d) al |= reinterpret_cast<uintptr_t>(a.din.ptr[i]);
    }
    al |= reinterpret_cast<uintptr_t>(a.y) | reinterpret_cast<uintptr_t>(a.dy);
    return (al & 15u) == 0;
}

template <typename T>
cudaError_t fwd_t(const BnLaunch &a, bool stats)
{
    const int slices = bn_slices(a.N, a.C);
    const int64_t grid = a.C * slices;
    if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
    const int vec = vec_ok(a, Store<T>::kBytes, false);
    double *partials = reinterpret_cast<double *>(static_cast<char *>(a.workspace) + kWsHeader);
    if (stats) {
        cudaError_t e = launch_pdl(bn_stats_kernel<T>, dim3((unsigned)grid), dim3(kBnThreads), 0, a.stream, a.in,
                                   a.N, a.C, a.HW, slices, vec, partials);
        if (e != cudaSuccess) return e;
    }
    const BnFin fin{(double)(a.N * a.HW), a.eps, a.momentum, a.running_mean, a.running_var};
    return launch_pdl(bn_apply_kernel<T>, dim3((unsigned)grid), dim3(kBnThreads), 0, a.stream, a.in, a.N, a.C, a.HW,
                      slices, vec, a.gamma, a.beta, a.mean, a.invstd, a.y,
                      stats ? static_cast<const double *>(partials) : nullptr, fin);
}

template <typename T>
cudaError_t bwd_t(const BnLaunch &a)
{
    const int slices = bn_slices(a.N, a.C);
    const int64_t grid = a.C * slices;
    if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
    const int vec = vec_ok(a, Store<T>::kBytes, true);
    double *partials = reinterpret_cast<double *>(static_cast<char *>(a.workspace) + kWsHeader);
    cudaError_t e = launch_pdl(bn_bwd_reduce_kernel<T>, dim3((unsigned)grid), dim3(kBnThreads), 0, a.stream, a.in,
                               a.dy, a.N, a.C, a.HW, slices, vec, a.gamma, a.beta,
                               static_cast<const float *>(a.mean), static_cast<const float *>(a.invstd), partials);
    if (e != cudaSuccess) return e;
    auto dx_kernel = a.accumulate ? bn_dx_kernel<T, true> : bn_dx_kernel<T, false>;
    return launch_pdl(dx_kernel, dim3((unsigned)grid), dim3(kBnThreads), 0, a.stream, a.in, a.din, a.dy, a.N, a.C,
                      a.HW, slices, vec, a.gamma, a.beta, static_cast<const float *>(a.mean),
                      static_cast<const float *>(a.invstd), static_cast<const double *>(partials), a.dgamma,
                      a.dbeta);
}

}  // namespace

size_t bn_workspace_bytes(int64_t N, int64_t C)
{
    const size_t grid = (size_t)C * (size_t)bn_slices(N, C);
    return kWsHeader + sizeof(double) * 3 * grid + sizeof(float) * 3 * (size_t)C + 16;
}

cudaError_t launch_bn_fwd(const BnLaunch &a)
{
    return a.dtype == kBF16 ? fwd_t<Bf16>(a, true) : fwd_t<float>(a, true);
}

cudaError_t launch_bn_apply(const BnLaunch &a)
{
    return a.dtype == kBF16 ? fwd_t<Bf16>(a, false) : fwd_t<float>(a, false);
}

cudaError_t launch_bn_bwd(const BnLaunch &a)
{
    return a.dtype == kBF16 ? bwd_t<Bf16>(a) : bwd_t<float>(a);
}

}  // namespace mea
