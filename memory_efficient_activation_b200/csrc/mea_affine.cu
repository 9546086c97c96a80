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
// NHWC fast path (C a multiple of 4, aligned pointers): a block is a
// multiple of G = C / 4 threads, so every thread keeps the same 4 channels,
// with gamma / beta in registers.  The forward handles one tile per block.
// The backward runs a fixed grid (a function of the shape) that walks the
// tiles with register prefetch, keeps fp64 per-channel sums per thread,
// folds them per block in row order and writes one row of fp64 partials per
// block; a second kernel adds each channel's column in block order.  So
// dgamma / dbeta are bitwise reproducible on any device.
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

constexpr int kNhwcMaxThreads = 512;
constexpr int kNhwcTargetThreads = 256;
constexpr int kColsumThreads = 256;
constexpr int kNhwcBwdGridCap = 888;     // 148 x 6
constexpr int kPlaneThreads = 256;
constexpr int kPlaneBlocksTarget = 1184; // C * S is sized to about this many blocks

// Threads per NHWC block: lcm(G, 32) times the largest m that keeps it at
// or below kNhwcTargetThreads (at least one lcm), where G = C / V is the
// number of channel groups.  A block is then whole warps and a multiple of
// G, so every thread of a block keeps the same V channels.  Returns 0 when
// lcm(G, 32) exceeds kNhwcMaxThreads (the NHWC fast path is then not taken).
static int nhwc_threads(int groups)
{
    int a = groups, b = 32;
    while (b) { int t = a % b; a = b; b = t; }
    const long lcm = (long)groups / a * 32;
    if (lcm > kNhwcMaxThreads) return 0;
    long m = kNhwcTargetThreads / lcm;
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

// Load units of the NHWC kernels: VE elements per thread per access (bf16:
// 4 elements in 8 bytes or 8 in 16; fp32: 4 in 16 bytes).  Fewer channels
// per thread keep the per-thread gamma / beta / partial-sum registers small,
// which is what sets the occupancy of these kernels.
template <typename T, int VE>
struct Unit;

template <>
struct Unit<Bf16, 8> {
    using W = uint4;
    static constexpr bool P = false;
    static __device__ __forceinline__ W load(const void *p, int64_t i) { return ld_nc_v4(static_cast<const uint4 *>(p) + i); }
    static __device__ __forceinline__ void store(void *p, int64_t i, const W &w) { st_v4(static_cast<uint4 *>(p) + i, w); }
    static __device__ __forceinline__ void unpack(const W &w, float (&f)[8]) { Store<Bf16>::unpack(w, f); }
    static __device__ __forceinline__ W pack(const float (&f)[8]) { return Store<Bf16>::pack(f); }
};

template <>
struct Unit<Bf16, 4> {
    using W = uint2;
    static constexpr bool P = false;
    static __device__ __forceinline__ W load(const void *p, int64_t i)
    {
        W r;
        asm("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y)
            : "l"(static_cast<const uint2 *>(p) + i));
        return r;
    }
    static __device__ __forceinline__ void store(void *p, int64_t i, const W &w)
    {
        asm volatile("st.global.v2.u32 [%0], {%1, %2};" ::"l"(static_cast<uint2 *>(p) + i), "r"(w.x), "r"(w.y)
                     : "memory");
    }
    static __device__ __forceinline__ void unpack(const W &w, float (&f)[4])
    {
        f[0] = __uint_as_float(w.x << 16);
        f[1] = __uint_as_float(w.x & 0xffff0000u);
        f[2] = __uint_as_float(w.y << 16);
        f[3] = __uint_as_float(w.y & 0xffff0000u);
    }
    static __device__ __forceinline__ W pack(const float (&f)[4])
    {
        return make_uint2(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]));
    }
};

template <>
struct Unit<float, 4> {
    using W = uint4;
    static constexpr bool P = true;
    static __device__ __forceinline__ W load(const void *p, int64_t i) { return ld_nc_v4(static_cast<const uint4 *>(p) + i); }
    static __device__ __forceinline__ void store(void *p, int64_t i, const W &w) { st_v4(static_cast<uint4 *>(p) + i, w); }
    static __device__ __forceinline__ void unpack(const W &w, float (&f)[4]) { Store<float>::unpack(w, f); }
    static __device__ __forceinline__ W pack(const float (&f)[4]) { return Store<float>::pack(f); }
};

// Forward: one tile of blockDim.x * U units per block (as the plain
// activation kernels), y = z Sigmoid(z), z = gamma_c x + beta_c.
template <typename T, int U, int VE>
__global__ void __launch_bounds__(kNhwcMaxThreads)
affine_nhwc_fwd_kernel(const void *__restrict__ x, const float *__restrict__ gamma, const float *__restrict__ beta,
                       void *__restrict__ out, int64_t nunits, int groups)
{
    using L = Unit<T, VE>;
    constexpr bool P = L::P;
    const int tid = threadIdx.x;
    const int g = tid % groups;
    const Coef k = Swish::coef(1.f);
    pdl_wait();
    float ga[VE], be[VE];
#pragma unroll
    for (int j = 0; j < VE; ++j) {
        ga[j] = __ldg(gamma + g * VE + j);
        be[j] = __ldg(beta + g * VE + j);
    }
    const int64_t base = (int64_t)blockIdx.x * blockDim.x * U + tid;
    typename L::W xv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int64_t i = base + (int64_t)u * blockDim.x;
        if (i < nunits) xv[u] = L::load(x, i);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int64_t i = base + (int64_t)u * blockDim.x;
        if (i < nunits) {
            float xf[VE], of[VE];
            L::unpack(xv[u], xf);
            bool tail = false;
#pragma unroll
            for (int j = 0; j < VE; ++j) of[j] = Swish::f<P>(fmaf(ga[j], xf[j], be[j]), k, tail);
            if (tail) {
#pragma unroll
                for (int j = 0; j < VE; ++j) {
                    const float z = fmaf(ga[j], xf[j], be[j]);
                    if (Swish::is_tail(z, k)) of[j] = Swish::f_tail<P>(z, k);
                }
            }
            L::store(out, i, L::pack(of));
        }
    }
    pdl_trigger();
}

// Backward: a fixed grid of blocks (a function of the shape only) walks the
// tiles of blockDim.x * U units with a grid stride, loading the next tile's
// x and dy before working on the current one.  Each thread keeps the same VE
// channels throughout; its dz x and dz sums go from fp32 per tile into fp64
// registers.  At the end the block folds its threads' sums per channel in
// row order (fp64, through shared memory) and writes one row of partials:
//   partials[blockIdx.x * 2C + kind * C + c],  kind 0 = dgamma, 1 = dbeta.
template <typename T, int U, int VE>
__global__ void __launch_bounds__(kNhwcMaxThreads)
affine_nhwc_bwd_kernel(const void *__restrict__ x, const void *__restrict__ dy, const float *__restrict__ gamma,
                       const float *__restrict__ beta, void *__restrict__ dx, int64_t nunits, int groups, int C,
                       double *__restrict__ partials)
{
    using L = Unit<T, VE>;
    constexpr bool P = L::P;
    const int tid = threadIdx.x;
    const int g = tid % groups;
    const Coef k = Swish::coef(1.f);
    pdl_wait();
    float ga[VE], be[VE];
#pragma unroll
    for (int j = 0; j < VE; ++j) {
        ga[j] = __ldg(gamma + g * VE + j);
        be[j] = __ldg(beta + g * VE + j);
    }
    double ag[VE], ab[VE];
#pragma unroll
    for (int j = 0; j < VE; ++j) ag[j] = ab[j] = 0.0;
    const int64_t tile = (int64_t)blockDim.x * U;
    const int64_t stride = (int64_t)gridDim.x * tile;
    int64_t base = (int64_t)blockIdx.x * tile + tid;
    typename L::W xv[U], gv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int64_t i = base + (int64_t)u * blockDim.x;
        if (i < nunits) {
            xv[u] = L::load(x, i);
            gv[u] = L::load(dy, i);
        }
    }
    for (; base < nunits; base += stride) {
        typename L::W xn[U], gn[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = base + stride + (int64_t)u * blockDim.x;
            if (i < nunits) {
                xn[u] = L::load(x, i);
                gn[u] = L::load(dy, i);
            }
        }
        float sg[VE], sb[VE];
#pragma unroll
        for (int j = 0; j < VE; ++j) sg[j] = sb[j] = 0.f;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = base + (int64_t)u * blockDim.x;
            if (i < nunits) {
                float xf[VE], gf[VE], of[VE];
                L::unpack(xv[u], xf);
                L::unpack(gv[u], gf);
                bool tail = false;
#pragma unroll
                for (int j = 0; j < VE; ++j) of[j] = Swish::df<P>(fmaf(ga[j], xf[j], be[j]), gf[j], k, tail);
                if (tail) {
#pragma unroll
                    for (int j = 0; j < VE; ++j) {
                        const float z = fmaf(ga[j], xf[j], be[j]);
                        if (Swish::is_tail(z, k)) of[j] = Swish::df_tail<P>(z, gf[j], k);
                    }
                }
#pragma unroll
                for (int j = 0; j < VE; ++j) {
                    sg[j] = fmaf(of[j], xf[j], sg[j]);   // dz x
                    sb[j] += of[j];                      // dz
                    of[j] = ga[j] * of[j];               // dx
                }
                L::store(dx, i, L::pack(of));
            }
        }
#pragma unroll
        for (int j = 0; j < VE; ++j) {
            ag[j] += (double)sg[j];
            ab[j] += (double)sb[j];
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            xv[u] = xn[u];
            gv[u] = gn[u];
        }
    }
    pdl_trigger();
    extern __shared__ double red[];   // 2 VE * blockDim.x doubles
#pragma unroll
    for (int j = 0; j < VE; ++j) {
        red[j * blockDim.x + tid] = ag[j];
        red[(VE + j) * blockDim.x + tid] = ab[j];
    }
    __syncthreads();
    const int rows = blockDim.x / groups;
    for (int o = tid; o < 2 * C; o += blockDim.x) {
        const int kind = o / C, c = o % C;
        const double *col = red + (kind * VE + c % VE) * blockDim.x + c / VE;
        double s = 0.0;
        for (int r = 0; r < rows; ++r) s += col[r * groups];
        partials[(int64_t)blockIdx.x * 2 * C + o] = s;
    }
}

// Output o (kind * C + c) = sum over the nb rows of partials, column o, in
// fp64: thread t adds rows t, t + kColsumThreads, ... in order, then a fixed
// block-wide tree.  One block per output.
__global__ void __launch_bounds__(kColsumThreads)
affine_colsum_kernel(const double *__restrict__ partials, int nb, int C, float *__restrict__ dgamma,
                     float *__restrict__ dbeta)
{
    __shared__ double red[32];
    const int o = blockIdx.x;
    pdl_wait();
    pdl_trigger();
    double s = 0.0;
    for (int b = threadIdx.x; b < nb; b += kColsumThreads) s += partials[(int64_t)b * 2 * C + o];
    s = block_sum(s, red);
    if (threadIdx.x == 0) {
        if (o < C) dgamma[o] = (float)s;
        else dbeta[o - C] = (float)s;
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
    pdl_wait();
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
    pdl_trigger();
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

// NHWC launch shape per storage dtype: elements per thread access (VE) and
// accesses per thread (U) for the forward and the backward (measured on B200
// at [128, 56, 56, 144] bf16 against 8 / 16-byte units, 1-16 accesses,
// tile-per-block and fixed-grid backward variants).
template <typename T>
struct NhwcCfg;
template <>
struct NhwcCfg<Bf16> {
    static constexpr int VE = 4, U_FWD = 16, U_BWD = 2;
};
template <>
struct NhwcCfg<float> {
    static constexpr int VE = 4, U_FWD = 8, U_BWD = 2;
};

template <typename T>
static bool nhwc_fast(const AffineLaunch &a)
{
    constexpr int VE = NhwcCfg<T>::VE;
    constexpr int bytes = VE * (sizeof(T) == 4 ? 4 : 2);
    uintptr_t al = reinterpret_cast<uintptr_t>(a.x) | reinterpret_cast<uintptr_t>(a.out);
    if (a.dy) al |= reinterpret_cast<uintptr_t>(a.dy);
    return a.layout == 1 && a.C % VE == 0 && nhwc_threads((int)(a.C / VE)) > 0 && (al % bytes) == 0;
}

static int64_t nhwc_blocks(int64_t nunits, int threads, int U)
{
    const int64_t per = (int64_t)threads * U;
    const int64_t nb = (nunits + per - 1) / per;
    return nb < 1 ? 1 : nb;
}

// Backward grid: one block per tile up to kNhwcBwdGridCap blocks (a function
// of the shape only, so the summation order is fixed).
static int nhwc_bwd_grid(int64_t nunits, int threads, int U)
{
    const int64_t nb = nhwc_blocks(nunits, threads, U);
    return (int)(nb < kNhwcBwdGridCap ? nb : kNhwcBwdGridCap);
}

template <typename T, int MODE>
static cudaError_t launch_affine(const AffineLaunch &a)
{
    constexpr int V = Store<T>::V;
    const int64_t HW = a.H * a.W;
    const int64_t n = a.N * a.C * HW;
    if (nhwc_fast<T>(a)) {
        constexpr int VE = NhwcCfg<T>::VE;
        const int groups = (int)(a.C / VE);
        const int threads = nhwc_threads(groups);
        const int64_t nunits = n / VE;
        if (MODE == 0) {
            constexpr int U = NhwcCfg<T>::U_FWD;
            const int64_t nb = nhwc_blocks(nunits, threads, U);
            if (nb > 0x7fffffff) return cudaErrorInvalidConfiguration;
            return launch_pdl(affine_nhwc_fwd_kernel<T, U, VE>, dim3((unsigned)nb), dim3(threads), 0, a.stream, a.x,
                              a.gamma, a.beta, a.out, nunits, groups);
        }
        constexpr int U = NhwcCfg<T>::U_BWD;
        auto kernel = affine_nhwc_bwd_kernel<T, U, VE>;
        const int nb = nhwc_bwd_grid(nunits, threads, U);
        double *partials = reinterpret_cast<double *>(static_cast<char *>(a.workspace) + kWsHeader);
        const size_t smem = sizeof(double) * 2 * VE * threads;
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                             (int)cudaSharedmemCarveoutMaxShared);
        if (e == cudaSuccess && smem > 48 * 1024)
            e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        e = launch_pdl(kernel, dim3((unsigned)nb), dim3(threads), smem, a.stream, a.x, a.dy, a.gamma, a.beta, a.out,
                       nunits, groups, (int)a.C, partials);
        if (e != cudaSuccess) return e;
        return launch_pdl(affine_colsum_kernel, dim3((unsigned)(2 * a.C)), dim3(kColsumThreads), 0, a.stream,
                          partials, nb, (int)a.C, a.dgamma, a.dbeta);
    }
    uintptr_t al = reinterpret_cast<uintptr_t>(a.x) | reinterpret_cast<uintptr_t>(a.out);
    if (a.dy) al |= reinterpret_cast<uintptr_t>(a.dy);
    const int vec_ok = a.layout == 0 && HW % V == 0 && (al & 15u) == 0;
    const int slices = plane_slices(a.N, a.C);
    const int64_t grid = a.C * slices;
    if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
    if (a.layout == 1)
        return launch_pdl(affine_plane_kernel<T, MODE, true>, dim3((unsigned)grid), dim3(kPlaneThreads), 0, a.stream,
                          a.x, a.dy, a.gamma, a.beta, a.out, a.N, a.C, HW, slices, vec_ok, a.dgamma, a.dbeta,
                          a.workspace);
    return launch_pdl(affine_plane_kernel<T, MODE, false>, dim3((unsigned)grid), dim3(kPlaneThreads), 0, a.stream,
                      a.x, a.dy, a.gamma, a.beta, a.out, a.N, a.C, HW, slices, vec_ok, a.dgamma, a.dbeta,
                      a.workspace);
}

size_t affine_bwd_workspace_bytes(int dtype, int layout, int64_t N, int64_t C, int64_t H, int64_t W)
{
    // Mirrors the launch decision; pointer alignment is not known here, so
    // the larger of the two layouts' needs is returned for NHWC.
    const int VE = dtype == kBF16 ? NhwcCfg<Bf16>::VE : NhwcCfg<float>::VE;
    const int U = dtype == kBF16 ? NhwcCfg<Bf16>::U_BWD : NhwcCfg<float>::U_BWD;
    size_t plane = kWsHeader + sizeof(double) * 2 * (size_t)C * (size_t)plane_slices(N, C);
    if (layout == 1 && C % VE == 0 && nhwc_threads((int)(C / VE)) > 0) {
        const int threads = nhwc_threads((int)(C / VE));
        const int64_t nunits = N * C * H * W / VE;
        size_t fast = kWsHeader + sizeof(double) * 2 * (size_t)C * (size_t)nhwc_bwd_grid(nunits, threads, U);
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
