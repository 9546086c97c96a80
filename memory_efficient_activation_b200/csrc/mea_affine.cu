// mea_affine.cu -- fused per-channel affine + Swish, forward and backward.
//
//   z = gamma_c x + beta_c,  y = z Sigmoid(z)
//   dz = dy (s + z s Sigmoid(-z)),  dx = gamma_c dz,
//   dgamma_c = sum dz x,  dbeta_c = sum dz        (over all N H W positions)
//
// Only x is kept between the passes; the backward recomputes z and the
// sigmoid from it (the save-input-only idea of "Memory efficient Swish",
// section "What makes this implementation save GPU memory?", applied to the
// affine + Swish pair that EfficientNet-style blocks run back to back).
//
// NHWC fast path (C a multiple of the 16-byte vector width, aligned
// pointers): a block has a multiple of G = C / V threads, so the grid-stride
// step is a multiple of G and every thread keeps the same V channels for the
// whole loop.  Its gamma / beta live in registers and its dgamma / dbeta
// partial sums in fp64 registers (fp32 inside one unrolled step).  The block
// folds its threads' sums per channel through shared memory in a fixed
// order and writes one fp64 partial per channel; the last block to finish
// (atomic ticket, no waiting) adds the per-block partials in block order.
// The backward grid is fixed by the shape, so the result is bitwise
// reproducible on any device.
//
// Plane path (NCHW, and NHWC shapes the fast path does not take): block
// (c, s) owns channel c and the s-th slice of the batch; for NCHW it streams
// the contiguous H W planes of that channel (16-byte vectors when H W is a
// multiple of the vector width and the pointers are aligned).
#include "mea_device.cuh"
#include "mea_internal.h"
#include "mea_math.cuh"

#include <cstdint>

namespace mea {

constexpr int kAffUnroll = 4;
constexpr int kNhwcMaxThreads = 640;
constexpr int kAffGridMax = 148;         // NHWC backward blocks (fixed, not device-derived)
constexpr int kPlaneThreads = 256;
constexpr int kPlaneBlocksTarget = 1184; // C * S is sized to about this many blocks

// Threads per NHWC block: lcm(G, 32) times the largest m that keeps it within
// kNhwcMaxThreads, where G = C / V is the number of channel groups.  Returns
// 0 when lcm(G, 32) itself is too large (the NHWC fast path is then not
// taken), so a block is always whole warps and a multiple of G.
static int nhwc_threads(int groups)
{
    int a = groups, b = 32;
    while (b) { int t = a % b; a = b; b = t; }
    const long lcm = (long)groups / a * 32;
    if (lcm > kNhwcMaxThreads) return 0;
    long m = kNhwcMaxThreads / lcm;
    if (m < 1) m = 1;
    return (int)(lcm * m);
}

static int plane_slices(int64_t N, int64_t C)
{
    int64_t s = (kPlaneBlocksTarget + C - 1) / C;
    if (s > N) s = N;
    if (s < 1) s = 1;
    return (int)s;
}

// ------------------------------------------------------------ NHWC fast

template <typename T, int MODE>
__global__ void __launch_bounds__(kNhwcMaxThreads)
affine_nhwc_kernel(const void *__restrict__ x, const void *__restrict__ dy, const float *__restrict__ gamma,
                   const float *__restrict__ beta, void *__restrict__ out, int64_t nvec, int groups, int C,
                   float *__restrict__ dgamma, float *__restrict__ dbeta, void *__restrict__ ws)
{
    using S = Store<T>;
    constexpr int V = S::V;
    constexpr bool P = S::P;
    const int tid = threadIdx.x;
    const int g = tid % groups;
    const Coef k = Swish::coef(1.f);
    float ga[V], be[V];
#pragma unroll
    for (int j = 0; j < V; ++j) {
        ga[j] = __ldg(gamma + g * V + j);
        be[j] = __ldg(beta + g * V + j);
    }
    // MODE 1: this thread's fp64 dgamma / dbeta sums live in shared memory,
    // acc[(kind * V + j) * blockDim.x + tid], which frees 2 V fp64 registers.
    extern __shared__ double acc[];
    if constexpr (MODE == 1) {
#pragma unroll
        for (int j = 0; j < 2 * V; ++j) acc[j * blockDim.x + tid] = 0.0;
    }

    const int64_t step = (int64_t)blockDim.x * kAffUnroll;
    for (int64_t base = (int64_t)blockIdx.x * step + tid; base < nvec; base += (int64_t)gridDim.x * step) {
        uint4 xv[kAffUnroll], gv[kAffUnroll];
#pragma unroll
        for (int u = 0; u < kAffUnroll; ++u) {
            const int64_t i = base + (int64_t)u * blockDim.x;
            if (i < nvec) {
                xv[u] = ld_nc_v4(static_cast<const uint4 *>(x) + i);
                if constexpr (MODE == 1) gv[u] = ld_nc_v4(static_cast<const uint4 *>(dy) + i);
            }
        }
        float sg[V], sb[V];
#pragma unroll
        for (int j = 0; j < V; ++j) sg[j] = sb[j] = 0.f;
#pragma unroll
        for (int u = 0; u < kAffUnroll; ++u) {
            const int64_t i = base + (int64_t)u * blockDim.x;
            if (i < nvec) {
                float xf[V], gf[V], zf[V], of[V];
                S::unpack(xv[u], xf);
                if constexpr (MODE == 1) S::unpack(gv[u], gf);
                bool tail = false;
#pragma unroll
                for (int j = 0; j < V; ++j) {
                    zf[j] = fmaf(ga[j], xf[j], be[j]);
                    if constexpr (MODE == 0)
                        of[j] = Swish::f<P>(zf[j], k, tail);
                    else
                        of[j] = Swish::df<P>(zf[j], gf[j], k, tail);   // dz
                }
                if (tail) {
#pragma unroll
                    for (int j = 0; j < V; ++j) {
                        if (Swish::is_tail(zf[j], k)) {
                            if constexpr (MODE == 0)
                                of[j] = Swish::f_tail<P>(zf[j], k);
                            else
                                of[j] = Swish::df_tail<P>(zf[j], gf[j], k);
                        }
                    }
                }
                if constexpr (MODE == 1) {
#pragma unroll
                    for (int j = 0; j < V; ++j) {
                        sg[j] = fmaf(of[j], xf[j], sg[j]);
                        sb[j] += of[j];
                        of[j] = ga[j] * of[j];
                    }
                }
                st_v4(static_cast<uint4 *>(out) + i, S::pack(of));
            }
        }
        if constexpr (MODE == 1) {
#pragma unroll
            for (int j = 0; j < V; ++j) {
                acc[j * blockDim.x + tid] += (double)sg[j];
                acc[(V + j) * blockDim.x + tid] += (double)sb[j];
            }
        }
    }
    if constexpr (MODE == 0) return;

    // Fold the rows of threads that share a channel group, in row order.
    unsigned int *ticket = static_cast<unsigned int *>(ws);
    double *partials = reinterpret_cast<double *>(static_cast<char *>(ws) + kWsHeader);
    const int rows = blockDim.x / groups;
    __syncthreads();
    for (int o = tid; o < 2 * C; o += blockDim.x) {
        const int kind = o / C, c = o % C;
        const int cg = c / V, cj = c % V;
        const double *col = acc + (kind * V + cj) * blockDim.x + cg;
        double s = 0.0;
        for (int r = 0; r < rows; ++r) s += col[r * groups];
        partials[(int64_t)o * gridDim.x + blockIdx.x] = s;
    }
    if (!last_block_done(ticket)) return;

    // Last block: output o (kind * C + c) is the sum over blocks in order;
    // one warp per output, lanes take blocks lane, lane + 32, ... and meet in
    // a fixed butterfly.
    const int lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    for (int o = warp; o < 2 * C; o += nwarps) {
        double s = 0.0;
        for (int b = lane; b < (int)gridDim.x; b += 32) s += __ldcg(partials + (int64_t)o * gridDim.x + b);
        s = warp_sum(s);
        if (lane == 0) {
            if (o < C) dgamma[o] = (float)s;
            else dbeta[o - C] = (float)s;
        }
    }
}

// ------------------------------------------------------------ plane path

template <typename T, int MODE, bool NHWC>
__global__ void __launch_bounds__(kPlaneThreads)
affine_plane_kernel(const void *__restrict__ x, const void *__restrict__ dy, const float *__restrict__ gamma,
                    const float *__restrict__ beta, void *__restrict__ out, int64_t N, int64_t C, int64_t HW,
                    int slices, int vec_ok, float *__restrict__ dgamma, float *__restrict__ dbeta,
                    void *__restrict__ ws)
{
    using S = Store<T>;
    constexpr int V = S::V;
    constexpr bool P = S::P;
    const int64_t c = blockIdx.x / slices;
    const int s = blockIdx.x % slices;
    const int64_t n0 = (int64_t)s * N / slices, n1 = (int64_t)(s + 1) * N / slices;
    const float ga = __ldg(gamma + c), be = __ldg(beta + c);
    const Coef k = Swish::coef(1.f);
    double ag = 0.0, ab = 0.0;

    auto one = [&](float xi, float gi, float &o) {
        const float z = fmaf(ga, xi, be);
        bool tail = false;
        if constexpr (MODE == 0) {
            o = Swish::f<P>(z, k, tail);
            if (tail) o = Swish::f_tail<P>(z, k);
        } else {
            float dz = Swish::df<P>(z, gi, k, tail);
            if (tail) dz = Swish::df_tail<P>(z, gi, k);
            o = ga * dz;
            ag += (double)(dz * xi);
            ab += (double)dz;
        }
    };

    if (!NHWC && vec_ok) {
        // NCHW planes are contiguous and each starts on a 16-byte boundary.
        const int64_t hwv = HW / V;
        const int64_t total = (n1 - n0) * hwv;
        for (int64_t q = threadIdx.x; q < total; q += blockDim.x) {
            const int64_t n = n0 + q / hwv;
            const int64_t vi = (n * C + c) * hwv + q % hwv;
            float xf[V], gf[V], of[V];
            S::unpack(ld_nc_v4(static_cast<const uint4 *>(x) + vi), xf);
            if constexpr (MODE == 1) S::unpack(ld_nc_v4(static_cast<const uint4 *>(dy) + vi), gf);
#pragma unroll
            for (int j = 0; j < V; ++j) one(xf[j], MODE == 1 ? gf[j] : 0.f, of[j]);
            st_v4(static_cast<uint4 *>(out) + vi, S::pack(of));
        }
    } else {
        const int64_t total = (n1 - n0) * HW;
        for (int64_t p = threadIdx.x; p < total; p += blockDim.x) {
            const int64_t n = n0 + p / HW, hw = p % HW;
            const int64_t i = NHWC ? (n * HW + hw) * C + c : (n * C + c) * HW + hw;
            const float xi = S::load1(x, i);
            const float gi = MODE == 1 ? S::load1(dy, i) : 0.f;
            float o;
            one(xi, gi, o);
            S::store1(out, i, o);
        }
    }
    if constexpr (MODE == 0) return;

    __shared__ double red[32];
    unsigned int *ticket = static_cast<unsigned int *>(ws);
    double *partials = reinterpret_cast<double *>(static_cast<char *>(ws) + kWsHeader);
    const double bg = block_sum(ag, red);
    const double bb = block_sum(ab, red);
    if (threadIdx.x == 0) {
        partials[(0 * C + c) * slices + s] = bg;
        partials[(1 * C + c) * slices + s] = bb;
    }
    if (!last_block_done(ticket)) return;
    for (int64_t o = threadIdx.x; o < 2 * C; o += blockDim.x) {
        double t = 0.0;
        for (int q = 0; q < slices; ++q) t += __ldcg(partials + o * slices + q);
        if (o < C) dgamma[o] = (float)t;
        else dbeta[o - C] = (float)t;
    }
}

// ------------------------------------------------------------ launchers

template <typename T>
static bool nhwc_fast(const AffineLaunch &a)
{
    constexpr int V = Store<T>::V;
    uintptr_t al = reinterpret_cast<uintptr_t>(a.x) | reinterpret_cast<uintptr_t>(a.out);
    if (a.dy) al |= reinterpret_cast<uintptr_t>(a.dy);
    return a.layout == 1 && a.C % V == 0 && (a.C / V) <= 1024 && nhwc_threads((int)(a.C / V)) > 0 &&
           (al & 15u) == 0;
}

template <typename T>
static int nhwc_bwd_grid(const AffineLaunch &a, int threads)
{
    constexpr int V = Store<T>::V;
    const int64_t nvec = a.N * a.C * a.H * a.W / V;
    int64_t g = (nvec + (int64_t)threads * kAffUnroll - 1) / ((int64_t)threads * kAffUnroll);
    if (g > kAffGridMax) g = kAffGridMax;
    if (g < 1) g = 1;
    return (int)g;
}

template <typename T, int MODE>
static cudaError_t launch_affine(const AffineLaunch &a)
{
    constexpr int V = Store<T>::V;
    const int64_t HW = a.H * a.W;
    const int64_t n = a.N * a.C * HW;
    if (nhwc_fast<T>(a)) {
        const int groups = (int)(a.C / V);
        const int threads = nhwc_threads(groups);
        auto kernel = affine_nhwc_kernel<T, MODE>;
        const int64_t nvec = n / V;
        int grid;
        size_t smem = 0;
        if (MODE == 1) {
            grid = nhwc_bwd_grid<T>(a, threads);
            smem = sizeof(double) * 2 * V * threads;
            if (smem > 48 * 1024) {
                cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
                if (e != cudaSuccess) return e;
            }
        } else {
            int b = 0;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kernel, threads, 0) != cudaSuccess || b < 1) b = 1;
            int64_t units = (nvec + (int64_t)threads * kAffUnroll - 1) / ((int64_t)threads * kAffUnroll);
            int64_t cap = (int64_t)sm_count() * b;
            grid = (int)(units < cap ? (units < 1 ? 1 : units) : cap);
        }
        kernel<<<grid, threads, smem, a.stream>>>(a.x, a.dy, a.gamma, a.beta, a.out, nvec, groups, (int)a.C,
                                                  a.dgamma, a.dbeta, a.workspace);
        return cudaGetLastError();
    }
    uintptr_t al = reinterpret_cast<uintptr_t>(a.x) | reinterpret_cast<uintptr_t>(a.out);
    if (a.dy) al |= reinterpret_cast<uintptr_t>(a.dy);
    const int vec_ok = a.layout == 0 && HW % V == 0 && (al & 15u) == 0;
    const int slices = plane_slices(a.N, a.C);
    const int64_t grid = a.C * slices;
    if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
    if (a.layout == 1)
        affine_plane_kernel<T, MODE, true><<<(unsigned)grid, kPlaneThreads, 0, a.stream>>>(
            a.x, a.dy, a.gamma, a.beta, a.out, a.N, a.C, HW, slices, vec_ok, a.dgamma, a.dbeta, a.workspace);
    else
        affine_plane_kernel<T, MODE, false><<<(unsigned)grid, kPlaneThreads, 0, a.stream>>>(
            a.x, a.dy, a.gamma, a.beta, a.out, a.N, a.C, HW, slices, vec_ok, a.dgamma, a.dbeta, a.workspace);
    return cudaGetLastError();
}

size_t affine_bwd_workspace_bytes(int dtype, int layout, int64_t N, int64_t C, int64_t H, int64_t W)
{
    // Mirrors the launch decision; pointer alignment is not known here, so
    // the larger of the two layouts' needs is returned for NHWC.
    const int V = dtype == kBF16 ? 8 : 4;
    size_t plane = kWsHeader + sizeof(double) * 2 * (size_t)C * (size_t)plane_slices(N, C);
    if (layout == 1 && C % V == 0 && C / V <= 1024 && nhwc_threads((int)(C / V)) > 0) {
        const int threads = nhwc_threads((int)(C / V));
        const int64_t nvec = N * C * H * W / V;
        int64_t g = (nvec + (int64_t)threads * kAffUnroll - 1) / ((int64_t)threads * kAffUnroll);
        if (g > kAffGridMax) g = kAffGridMax;
        if (g < 1) g = 1;
        size_t fast = kWsHeader + sizeof(double) * 2 * (size_t)C * (size_t)g;
        return fast > plane ? fast : plane;
    }
    return plane;
}

cudaError_t launch_affine_fwd(const AffineLaunch &a)
{
    return a.dtype == kBF16 ? launch_affine<Bf16, 0>(a) : launch_affine<float, 0>(a);
}

cudaError_t launch_affine_bwd(const AffineLaunch &a)
{
    return a.dtype == kBF16 ? launch_affine<Bf16, 1>(a) : launch_affine<float, 1>(a);
}

}  // namespace mea
