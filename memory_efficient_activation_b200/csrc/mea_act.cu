// mea_act.cu -- streaming kernels of the save-input-only activation family.
//
// One template serves every activation, dtype and pass:
//   MODE 0  forward:            y  = f(x)
//   MODE 1  backward:           dx = dy f'(x), f' recomputed from x
//   MODE 2  backward + d alpha: as MODE 1, plus sum dy x^2 s (1 - s) (Swish)
//
// The work is HBM-bound (problem B07 of "What activations cost, in memory and
// in arithmetic": about c/4 FLOP per byte), so the kernel is built around the
// memory system: 16-byte vector loads through the non-coherent path without
// L1 allocation, kUnroll independent vectors per thread (2 kUnroll in the
// backward) all issued before any arithmetic, one tile per block so that
// short-lived blocks keep every SM's memory pipeline full, and stores straight
// from registers.  (Measured on B200 at 67M bf16 elements: this shape reaches
// the speed of a compute-free copy with the same access pattern; persistent
// grid-stride loops, register double-buffering and a TMA bulk-copy pipeline
// through shared memory were each 3-15% slower.)  Pointers that are not
// 16-byte aligned take the scalar loop of the same kernel; so does the ragged
// tail of n mod V elements.
//
// The d alpha reduction is deterministic: its grid is a function of n only,
// each thread accumulates fp32 vector sums into an fp64 register, blocks
// reduce through a fixed xor-butterfly, every block writes one fp64 partial,
// and the last block to finish (found with an atomic ticket, no waiting)
// adds the partials in index order and writes the fp32 result.  The ticket
// wraps back to zero, so the workspace is left as it was found.
#include "mea_device.cuh"
#include "mea_internal.h"
#include "mea_math.cuh"

#include <cmath>
#include <cstdint>
#include <type_traits>

namespace mea {

// Writes this block's partial; the last block to arrive sums all partials in
// index order and stores the fp32 result.  No block ever waits.
// bid / nblk: this block's index among the nblk blocks of its reduction.
__device__ __forceinline__ void finish_reduction(double acc, float *out, void *ws, int bid, int nblk)
{
    __shared__ double red[32];
    unsigned int *ticket = static_cast<unsigned int *>(ws);
    double *partials = reinterpret_cast<double *>(static_cast<char *>(ws) + kWsHeader);

    double b = block_sum(acc, red);
    if (threadIdx.x == 0) partials[bid] = b;
    if (!last_block_done(ticket, nblk)) return;
    double v = 0.0;
    for (int i = threadIdx.x; i < nblk; i += blockDim.x) v += __ldcg(partials + i);
    double total = block_sum(v, red);
    if (threadIdx.x == 0) *out = (float)total;
}

// ------------------------------------------------------------ the kernel

// Writes this block's partial only (the grouped kernel: a second kernel adds
// each segment's partials, so its workspace needs no counter).
__device__ __forceinline__ void block_partial(double acc, void *ws, int bid)
{
    __shared__ double red[32];
    double *partials = reinterpret_cast<double *>(static_cast<char *>(ws) + kWsHeader);
    const double b = block_sum(acc, red);
    if (threadIdx.x == 0) partials[bid] = b;
}

// The work of block bid of nblk over one tensor (the grid of act_kernel, or
// one segment's share of the grouped kernel's grid).  kTicket: the d alpha
// reduction ends in this grid (last block by ticket) rather than in a
// separate kernel.
template <class A, typename T, int MODE, bool kTicket = true>
__device__ __forceinline__ void act_body(const void *__restrict__ x, const void *__restrict__ dy,
                                         void *__restrict__ out, int64_t n, int vec_ok, float param,
                                         const float *__restrict__ param_dev, float *__restrict__ dparam,
                                         void *__restrict__ ws, int bid, int nblk)
{
    using S = Store<T>;
    constexpr int V = S::V;
    constexpr bool P = S::P;
    pdl_wait();
    const Coef k = A::coef(param_dev ? __ldg(param_dev) : param);
    const int64_t nvec = vec_ok ? n / V : 0;
    const int tid = threadIdx.x;
    const int64_t tile = (int64_t)kThreads * kUnroll;
    double acc = 0.0;

    if constexpr (MODE != 2) {
        // One tile of kThreads * kUnroll vectors per block (the grid covers
        // every tile): all loads of the tile are issued before any math, and
        // blocks retire and refill the SM independently.
        const int64_t base = (int64_t)bid * tile + tid;
        uint4 xv[kUnroll], gv[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t i = base + (int64_t)u * kThreads;
            if (i < nvec) {
                xv[u] = ld_nc_v4(static_cast<const uint4 *>(x) + i);
                if constexpr (MODE != 0) gv[u] = ld_nc_v4(static_cast<const uint4 *>(dy) + i);
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t i = base + (int64_t)u * kThreads;
            if (i < nvec) {
                float xf[V], gf[V], of[V];
                S::unpack(xv[u], xf);
                if constexpr (MODE != 0) S::unpack(gv[u], gf);
                bool tail = false;
                constexpr bool kPairs = MODE == 0 ? HasPairs<A, P>::value : HasPairsBwd<A, P>::value;
                if constexpr (kPairs) {
#pragma unroll
                    for (int j = 0; j < V; j += 2) {
                        if constexpr (MODE == 0)
                            A::f2(xf[j], xf[j + 1], k, tail, of[j], of[j + 1]);
                        else
                            A::df2(xf[j], xf[j + 1], gf[j], gf[j + 1], k, tail, of[j], of[j + 1]);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < V; ++j) {
                        if constexpr (MODE == 0)
                            of[j] = A::template f<P>(xf[j], k, tail);
                        else
                            of[j] = A::template df<P>(xf[j], gf[j], k, tail);
                    }
                }
                if (tail) {
#pragma unroll
                    for (int j = 0; j < V; ++j) {
                        if constexpr (MODE == 0) {
                            if (A::is_tail(xf[j], k)) of[j] = A::template f_tail<P>(xf[j], k);
                        } else {
                            if (A::template is_tail_bwd<P>(xf[j], k)) of[j] = A::template df_tail<P>(xf[j], gf[j], k);
                        }
                    }
                }
                st_v4(static_cast<uint4 *>(out) + i, S::pack(of));
            }
        }
    } else {
        // d alpha: grid-stride over a grid fixed by n (one resident wave on a
        // B200), so that every element's place in the summation order is
        // fixed too.  The next iteration's x and dy are loaded before the
        // current one is worked on.
        constexpr int R = kRedUnroll;
        const int64_t rtile = (int64_t)kThreads * R;
        const int64_t rstride = (int64_t)nblk * rtile;
        int64_t rb = (int64_t)bid * rtile + tid;
        uint4 xv[R], gv[R];
#pragma unroll
        for (int u = 0; u < R; ++u) {
            const int64_t i = rb + (int64_t)u * kThreads;
            if (i < nvec) {
                xv[u] = ld_nc_v4(static_cast<const uint4 *>(x) + i);
                gv[u] = ld_nc_v4(static_cast<const uint4 *>(dy) + i);
            }
        }
        for (; rb < nvec; rb += rstride) {
            uint4 xn[R], gn[R];
#pragma unroll
            for (int u = 0; u < R; ++u) {
                const int64_t i = rb + rstride + (int64_t)u * kThreads;
                if (i < nvec) {
                    xn[u] = ld_nc_v4(static_cast<const uint4 *>(x) + i);
                    gn[u] = ld_nc_v4(static_cast<const uint4 *>(dy) + i);
                }
            }
#pragma unroll
            for (int u = 0; u < R; ++u) {
                const int64_t i = rb + (int64_t)u * kThreads;
                if (i < nvec) {
                    float xf[V], gf[V], of[V], tf[V];
                    S::unpack(xv[u], xf);
                    S::unpack(gv[u], gf);
                    bool tail = false;
#pragma unroll
                    for (int j = 0; j < V; ++j) of[j] = A::template df_da<P>(xf[j], gf[j], k, tail, tf[j]);
                    if (tail) {
#pragma unroll
                        for (int j = 0; j < V; ++j)
                            if (A::template is_tail_bwd<P>(xf[j], k))
                                of[j] = A::template df_da_tail<P>(xf[j], gf[j], k, tf[j]);
                    }
                    st_v4(static_cast<uint4 *>(out) + i, S::pack(of));
                    acc += (double)tree_sum<V>(tf);
                }
            }
#pragma unroll
            for (int u = 0; u < R; ++u) {
                xv[u] = xn[u];
                gv[u] = gn[u];
            }
        }
    }

    pdl_trigger();

    // Scalar loop: the n mod V tail of the vector path, or every element when
    // a pointer is not 16-byte aligned.
    for (int64_t i = nvec * V + (int64_t)bid * kThreads + tid; i < n;
         i += (int64_t)nblk * kThreads) {
        const float xi = S::load1(x, i);
        bool tail = false;
        float o, term = 0.f;
        if constexpr (MODE == 0) {
            o = A::template f<P>(xi, k, tail);
            if (tail) o = A::template f_tail<P>(xi, k);
        } else {
            const float gi = S::load1(dy, i);
            if constexpr (MODE == 1) {
                o = A::template df<P>(xi, gi, k, tail);
                if (tail) o = A::template df_tail<P>(xi, gi, k);
            } else {
                o = A::template df_da<P>(xi, gi, k, tail, term);
                if (tail) o = A::template df_da_tail<P>(xi, gi, k, term);
            }
        }
        S::store1(out, i, o);
        if constexpr (MODE == 2) acc += (double)term;
    }

    if constexpr (MODE == 2) {
        if constexpr (kTicket)
            finish_reduction(acc, dparam, ws, bid, nblk);
        else
            block_partial(acc, ws, bid);
    }
}

template <class A, typename T, int MODE>
__global__ void __launch_bounds__(kThreads, MODE == 2 ? 3 : 4)
act_kernel(const void *__restrict__ x, const void *__restrict__ dy, void *__restrict__ out, int64_t n,
           int vec_ok, float param, const float *__restrict__ param_dev, float *__restrict__ dparam,
           void *__restrict__ ws)
{
    act_body<A, T, MODE>(x, dy, out, n, vec_ok, param, param_dev, dparam, ws, (int)blockIdx.x, (int)gridDim.x);
}

// Several independent tensors in one grid: block b works on the segment
// whose block range holds b, exactly as block b - start of that segment's
// own act_kernel launch would (same block count, same element assignment,
// same summation order), so every output and d alpha is bitwise what the
// separate launches give.  One launch instead of several removes the ramp,
// drain and launch gaps of each small tensor.  With d alpha each block
// writes its partial and act_group_dalpha_kernel adds them.
template <class A, typename T, int MODE>
__global__ void __launch_bounds__(kThreads, MODE == 2 ? 3 : 4)
act_group_kernel(const __grid_constant__ ActSegTable tab)
{
    int s = 0;
    while (s + 1 < tab.nseg && (int)blockIdx.x >= tab.start[s + 1]) ++s;
    const ActSeg &g = tab.seg[s];
    act_body<A, T, MODE, false>(g.x, g.dy, g.out, g.n, g.vec_ok, g.param, g.param_dev, g.dparam, g.ws,
                                (int)blockIdx.x - tab.start[s], tab.start[s + 1] - tab.start[s]);
}

// d alpha of segment blockIdx.x from its blocks' partials: the sum the last
// block of a single launch forms (finish_reduction), in the same order with
// the same block size, so the result is bitwise the same.
__global__ void __launch_bounds__(kThreads)
act_group_dalpha_kernel(const __grid_constant__ ActSegTable tab)
{
    __shared__ double red[32];
    pdl_wait();
    const ActSeg &g = tab.seg[blockIdx.x];
    const int nblk = tab.start[blockIdx.x + 1] - tab.start[blockIdx.x];
    const double *partials = reinterpret_cast<const double *>(static_cast<const char *>(g.ws) + kWsHeader);
    double v = 0.0;
    for (int i = threadIdx.x; i < nblk; i += blockDim.x) v += __ldcg(partials + i);
    const double total = block_sum(v, red);
    if (threadIdx.x == 0) *g.dparam = (float)total;
}


// ------------------------------------------------------------ launchers

int sm_count()
{
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev < 0 || dev >= 64) return 148;
    if (cached[dev] == 0) {
        int c = 0;
        if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c <= 0)
            c = 148;
        cached[dev] = c;
    }
    return cached[dev];
}

template <class A, typename T, int MODE>
struct KernelTag {};

template <class A, typename T, int MODE>
static cudaError_t launch_one(const ActLaunch &a)
{
    constexpr int V = Store<T>::V;
    auto kernel = act_kernel<A, T, MODE>;
    uintptr_t align = reinterpret_cast<uintptr_t>(a.x) | reinterpret_cast<uintptr_t>(a.out);
    if (MODE != 0) align |= reinterpret_cast<uintptr_t>(a.dy);
    const int vec_ok = (align & 15u) == 0;
    int64_t g;
    if (MODE == 2) {
        g = red_grid(a.n);
    } else if (vec_ok) {
        // one tile per block; the n mod V tail goes to block 0's scalar loop
        g = (a.n / V + (int64_t)kThreads * kUnroll - 1) / ((int64_t)kThreads * kUnroll);
    } else {
        // scalar path: a grid-stride loop over a resident-sized grid
        const int64_t units = (a.n + kThreads - 1) / kThreads;
        const int64_t cap = (int64_t)sm_count() * resident_blocks<KernelTag<A, T, MODE>>(kernel, kThreads);
        g = units < cap ? units : cap;
    }
    if (g < 1) g = 1;
    if (g > 0x7fffffff) return cudaErrorInvalidConfiguration;
    const int grid = (int)g;
    return launch_pdl(kernel, dim3((unsigned)grid), dim3(kThreads), 0, a.stream, a.x, a.dy, a.out, a.n, vec_ok,
                      a.param, a.param_dev, a.dparam, a.workspace);
}

template <class A, int MODE>
static cudaError_t by_dtype(const ActLaunch &a)
{
    return a.dtype == kBF16 ? launch_one<A, Bf16, MODE>(a) : launch_one<A, float, MODE>(a);
}

// alpha = 0 or +-2^k: alpha x is exact for bf16 x (see SwishT).
static bool exact_scale(float alpha)
{
    if (alpha == 0.f) return true;
    int e = 0;
    return std::isfinite(alpha) && std::fabs(std::frexp(alpha, &e)) == 0.5f;
}

template <int MODE>
static cudaError_t by_act(const ActLaunch &a)
{
    if (MODE != 0 && a.act == 6 && a.dtype == kBF16 && !a.param_dev && exact_scale(a.param))
        return launch_one<SwishT<false>, Bf16, MODE>(a);
    switch (a.act) {
    case 0: return by_dtype<ReLU, MODE>(a);
    case 1: return by_dtype<LeakyReLU, MODE>(a);
    case 2: return by_dtype<Sigmoid, MODE>(a);
    case 3: return by_dtype<Tanh, MODE>(a);
    case 4: return by_dtype<GeluErf, MODE>(a);
    case 5: return by_dtype<GeluTanh, MODE>(a);
    case 6: return by_dtype<Swish, MODE>(a);
    }
    return cudaErrorInvalidValue;
}

// ------------------------------------------------------ grouped launches

// The grid launch_one gives the segment's tensor on its own (0: nothing to do).
template <class A, typename T, int MODE>
static int64_t seg_blocks(const ActSeg &g)
{
    constexpr int V = Store<T>::V;
    if (MODE == 2) return red_grid(g.n);
    if (g.n == 0) return 0;
    int64_t b;
    if (g.vec_ok) {
        b = (g.n / V + (int64_t)kThreads * kUnroll - 1) / ((int64_t)kThreads * kUnroll);
    } else {
        const int64_t units = (g.n + kThreads - 1) / kThreads;
        const int64_t cap = (int64_t)sm_count() *
                            resident_blocks<KernelTag<A, T, MODE>>(act_kernel<A, T, MODE>, kThreads);
        b = units < cap ? units : cap;
    }
    return b < 1 ? 1 : b;
}

template <class A, typename T, int MODE>
static cudaError_t launch_group(const ActGroupLaunch &a)
{
    for (int c0 = 0; c0 < a.nseg; c0 += kMaxSegs) {
        const int cnt = a.nseg - c0 < kMaxSegs ? a.nseg - c0 : kMaxSegs;
        ActSegTable tab{};
        int64_t total = 0;
        int k = 0;
        for (int i = 0; i < cnt; ++i) {
            ActSeg g = a.segs[c0 + i];
            uintptr_t align = reinterpret_cast<uintptr_t>(g.x) | reinterpret_cast<uintptr_t>(g.out);
            if (MODE != 0) align |= reinterpret_cast<uintptr_t>(g.dy);
            g.vec_ok = (align & 15u) == 0;
            const int64_t b = seg_blocks<A, T, MODE>(g);
            if (b == 0) continue;
            tab.seg[k] = g;
            tab.start[k] = (int)total;
            total += b;
            ++k;
            if (total > 0x7fffffff) return cudaErrorInvalidConfiguration;
        }
        if (k == 0) continue;
        tab.start[k] = (int)total;
        tab.nseg = k;
        cudaError_t e =
            launch_pdl(act_group_kernel<A, T, MODE>, dim3((unsigned)total), dim3(kThreads), 0, a.stream, tab);
        if (e == cudaSuccess && MODE == 2)
            e = launch_pdl(act_group_dalpha_kernel, dim3((unsigned)k), dim3(kThreads), 0, a.stream, tab);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

template <class A, int MODE>
static cudaError_t group_by_dtype(const ActGroupLaunch &a)
{
    return a.dtype == kBF16 ? launch_group<A, Bf16, MODE>(a) : launch_group<A, float, MODE>(a);
}

template <int MODE>
static cudaError_t group_by_act(const ActGroupLaunch &a)
{
    if (a.act == 6) {
        bool exact = a.dtype == kBF16;
        for (int i = 0; exact && i < a.nseg; ++i) exact = !a.segs[i].param_dev && exact_scale(a.segs[i].param);
        if (MODE != 0 && exact) return launch_group<SwishT<false>, Bf16, MODE>(a);
        return group_by_dtype<Swish, MODE>(a);
    }
    if constexpr (MODE == 2) {
        return cudaErrorInvalidValue;   // d alpha exists for Swish only
    } else {
        switch (a.act) {
        case 0: return group_by_dtype<ReLU, MODE>(a);
        case 1: return group_by_dtype<LeakyReLU, MODE>(a);
        case 2: return group_by_dtype<Sigmoid, MODE>(a);
        case 3: return group_by_dtype<Tanh, MODE>(a);
        case 4: return group_by_dtype<GeluErf, MODE>(a);
        case 5: return group_by_dtype<GeluTanh, MODE>(a);
        }
        return cudaErrorInvalidValue;
    }
}

cudaError_t launch_act_fwd_grouped(const ActGroupLaunch &a) { return group_by_act<0>(a); }

cudaError_t launch_act_bwd_grouped(const ActGroupLaunch &a)
{
    const bool da = a.nseg > 0 && a.segs[0].dparam != nullptr;
    return da ? group_by_act<2>(a) : group_by_act<1>(a);
}

cudaError_t launch_act_fwd(const ActLaunch &a) { return by_act<0>(a); }

cudaError_t launch_act_bwd(const ActLaunch &a)
{
    if (a.dparam) {   // the C-ABI admits d alpha for Swish only
        if (a.dtype == kBF16 && !a.param_dev && exact_scale(a.param)) return launch_one<SwishT<false>, Bf16, 2>(a);
        return by_dtype<Swish, 2>(a);
    }
    return by_act<1>(a);
}

}  // namespace mea
