// mea_channel.cuh -- per-channel elementwise kernels (fused affine + any
// activation; Swish with one alpha per channel), forward and backward.
//
// A per-channel operation Op supplies the arithmetic; the kernels here supply
// the data movement and the deterministic per-channel reductions.  Op has:
//   NR                     reductions per channel (affine: dgamma, dbeta;
//                          channel alpha: dalpha)
//   K  kcoef(ChanArgs)     constants shared by every channel
//   Ch load(ChanArgs, c)   constants of channel c
//   f<P>, f_tail<P>, is_tail      forward value, deep-tail recompute, test
//   bwd<P>(x, dy, ..., o, t)      backward main path -> raw results o, t
//   flag_bwd<P>, bwd_tail<P>      per-element test for, and recompute of,
//                                 every element a backward main path may flag
//                                 (deep tails, packed-form overflow guards;
//                                 with bf16 storage the neighbourhood of the
//                                 zero of f')
//   finish(x, o, t, ch, acc[NR])  dx, and adds the channel's reduction terms
//   Ch2, pair(ch, ch), bwd2<P>, finish2   the same for two adjacent channels
//                          in packed .f32x2 registers (pipelined backward)
//
// Only x is kept between the passes; the backward recomputes everything from
// it (the save-input-only idea of "Memory efficient Swish", section "What
// makes this implementation save GPU memory?", applied to the per-channel op
// that precedes the activation in EfficientNet-style blocks).
//
// NHWC fast path (C a multiple of 4, aligned pointers): a block is a
// multiple of G = C / 4 threads, so every thread keeps the same 4 channels,
// with their constants in registers.  The forward handles one tile per block.
// The backward runs a fixed grid (a function of the shape) that walks the
// tiles with register prefetch, keeps fp64 per-channel sums per thread,
// folds them per block in row order and writes one row of fp64 partials per
// block; a second kernel adds each channel's column in block order.  So the
// reductions are bitwise reproducible on any device.
//
// Plane path (NCHW, and NHWC shapes the fast path does not take): block
// (c, s) owns channel c and the s-th slice of the batch; for NCHW it streams
// the contiguous H W planes of that channel (16-byte vectors when H W is a
// multiple of the vector width and the pointers are aligned), and the last
// block to finish (atomic ticket) adds the per-block partials in order.
#pragma once

#include <cstdint>

#include "mea_channel_api.h"
#include "mea_device.cuh"
#include "mea_internal.h"
#include "mea_math.cuh"
#include "mea_pipe.cuh"
#include "mea_stream.cuh"

namespace mea {

constexpr int kNhwcMaxThreads = 512;
constexpr int kNhwcTargetThreads = 256;
constexpr int kColsumThreads = 256;
constexpr int kNhwcBwdGridCap = 888;     // 148 x 6
// Register cap of the NHWC backward.  Registers are allocated per warp in
// granules of 8 per thread, so with 288-thread blocks (C = 144: lcm(36, 32))
// 72 registers keep three blocks resident per SM and 56 keep four.
#ifndef MEA_NHWC_BWD_MAXREGS
#define MEA_NHWC_BWD_MAXREGS 72
#endif
constexpr int kNhwcBwdMaxRegs = MEA_NHWC_BWD_MAXREGS;
// Register cap of the NHWC forward: 64 keeps three 288-thread blocks per SM.
#ifndef MEA_NHWC_FWD_MAXREGS
#define MEA_NHWC_FWD_MAXREGS 64
#endif
constexpr int kNhwcFwdMaxRegs = MEA_NHWC_FWD_MAXREGS;
constexpr int kPlaneThreads = 256;
constexpr int kPlaneBlocksTarget = 1184; // C * S is sized to about this many blocks

// Parameter arrays and scalar of a per-channel operation (device pointers).
struct ChanArgs {
    const float *p0;   // gamma (affine) or alpha (channel Swish), [C]
    const float *p1;   // beta (affine), [C]; unused otherwise
    float scalar;      // activation parameter (LeakyReLU slope, Swish alpha)
};

// Threads per NHWC block: lcm(G, 32) times the largest m that keeps it at
// or below kNhwcTargetThreads (at least one lcm), where G = C / 4 is the
// number of channel groups.  A block is then whole warps and a multiple of
// G, so every thread of a block keeps the same channels.  Returns 0 when
// lcm(G, 32) exceeds kNhwcMaxThreads (the NHWC fast path is then not taken).
inline int nhwc_threads(int groups)
{
    int a = groups, b = 32;
    while (b) {
        int t = a % b;
        a = b;
        b = t;
    }
    const long lcm = (long)groups / a * 32;
    if (lcm > kNhwcMaxThreads) return 0;
    long m = kNhwcTargetThreads / lcm;
    if (m < 1) m = 1;
    return (int)(lcm * m);
}

inline int plane_slices(int64_t N, int64_t C)
{
    int64_t s = (kPlaneBlocksTarget + C - 1) / C;
    if (s > N) s = N;
    if (s < 1) s = 1;
    return (int)s;
}


// ------------------------------------------------------------ load units

// VE elements per thread per access (bf16: 4 elements in 8 bytes; fp32: 4 in
// 16 bytes).  Few channels per thread keep the per-thread constants and
// partial sums in few registers, which is what sets the occupancy here.
template <typename T, int VE>
struct Unit;

template <>
struct Unit<Bf16, 4> {
    using W = uint2;
    static constexpr bool P = false;
    static __device__ __forceinline__ W load(const void *p, int64_t i)
    {
        W r;
        asm("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];"
            : "=r"(r.x), "=r"(r.y)
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

// NHWC launch shape per storage dtype: elements per thread access (VE) and
// accesses per thread (U) for the forward and the backward (measured on B200
// at [128, 56, 56, 144] bf16 against 8 / 16-byte units, 1-16 accesses,
// tile-per-block and fixed-grid backward variants).
template <typename T>
struct NhwcCfg;
#ifndef MEA_NHWC_BWD_U
#define MEA_NHWC_BWD_U 2
#endif
// U_PIPE: units per consumer thread per tile of the pipelined backward.
#ifndef MEA_PIPE_UT_BF16
#define MEA_PIPE_UT_BF16 4
#endif
#ifndef MEA_NHWC_FWD_U_BF16
#define MEA_NHWC_FWD_U_BF16 16
#endif
template <>
struct NhwcCfg<Bf16> {
    static constexpr int VE = 4, U_FWD = MEA_NHWC_FWD_U_BF16, U_BWD = MEA_NHWC_BWD_U, U_PIPE = MEA_PIPE_UT_BF16;
};
template <>
struct NhwcCfg<float> {
    static constexpr int VE = 4, U_FWD = 8, U_BWD = MEA_NHWC_BWD_U, U_PIPE = 2;
};

// ------------------------------------------------------------ NHWC kernels

// Forward: one tile of blockDim.x * U units per block (as the plain
// activation kernels); pairs of channels in packed .f32x2 registers.
template <class Op, typename T, int U, int VE>
__global__ void __maxnreg__(kNhwcFwdMaxRegs)
chan_nhwc_fwd_kernel(const void *__restrict__ x, ChanArgs ca, void *__restrict__ out, int64_t nunits, int groups)
{
    using L = Unit<T, VE>;
    using W = typename L::W;
    constexpr bool P = L::P;
    const int tid = threadIdx.x;
    const int g = tid % groups;
    pdl_wait();
    const typename Op::K k = Op::kcoef(ca);
    typename Op::Ch ch[VE];
#pragma unroll
    for (int j = 0; j < VE; ++j) ch[j] = Op::load(ca, g * VE + j);
    typename Op::Ch2 ch2[VE / 2];
#pragma unroll
    for (int p = 0; p < VE / 2; ++p) ch2[p] = Op::pair(ch[2 * p], ch[2 * p + 1]);
    const int64_t base = (int64_t)blockIdx.x * blockDim.x * U + tid;
    const bool whole = (int64_t)(blockIdx.x + 1) * blockDim.x * U <= nunits;
    auto unit = [&](const W &w) -> W {
        float xf[VE], of[VE];
        L::unpack(w, xf);
        bool tail = false;
#pragma unroll
        for (int p = 0; p < VE / 2; ++p)
            upk(Op::template f2<P>(pk(xf[2 * p], xf[2 * p + 1]), k, ch2[p], tail), of[2 * p], of[2 * p + 1]);
        if (tail) {
#pragma unroll
            for (int j = 0; j < VE; ++j)
                if (Op::is_tail(xf[j], k, ch[j])) of[j] = Op::template f_tail<P>(xf[j], k, ch[j]);
        }
        return L::pack(of);
    };
    W xv[U];
    if (whole) {
        const W *src = static_cast<const W *>(x) + base;
#pragma unroll
        for (int u = 0; u < U; ++u) xv[u] = L::load(src, u * blockDim.x);
        W *dst = static_cast<W *>(out) + base;
#pragma unroll
        for (int u = 0; u < U; ++u) L::store(dst, u * blockDim.x, unit(xv[u]));
    } else {
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = base + (int64_t)u * blockDim.x;
            if (i < nunits) xv[u] = L::load(x, i);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = base + (int64_t)u * blockDim.x;
            if (i < nunits) L::store(out, i, unit(xv[u]));
        }
    }
    pdl_trigger();
}

// Backward: a fixed grid of blocks (a function of the shape only) walks the
// tiles of blockDim.x * U units with a grid stride, loading the next tile's
// x and dy before working on the current one.  Each thread keeps the same VE
// channels throughout; its reduction terms go from fp32 per tile into fp64
// registers.  At the end the block folds its threads' sums per channel in
// row order (fp64, through shared memory) and writes one row of partials:
//   partials[blockIdx.x * NR C + r * C + c].
template <class Op, typename T, int U, int VE>
__global__ void __maxnreg__(kNhwcBwdMaxRegs)
chan_nhwc_bwd_kernel(const void *__restrict__ x, const void *__restrict__ dy, ChanArgs ca, void *__restrict__ dx,
                     int64_t nunits, int groups, int C, double *__restrict__ partials)
{
    using L = Unit<T, VE>;
    constexpr bool P = L::P;
    constexpr int NR = Op::NR;
    const int tid = threadIdx.x;
    const int g = tid % groups;
    pdl_wait();
    const typename Op::K k = Op::kcoef(ca);
    typename Op::Ch ch[VE];
#pragma unroll
    for (int j = 0; j < VE; ++j) ch[j] = Op::load(ca, g * VE + j);
    // fp64 running sums, one slot per (reduction, channel of the thread,
    // thread): each thread owns its slots, so no synchronisation until the
    // fold.  Kept in shared memory rather than registers, which leaves room
    // for four blocks of 288 threads per SM.
    extern __shared__ double acc[];   // NR VE * blockDim.x doubles
#pragma unroll
    for (int r = 0; r < NR; ++r)
#pragma unroll
        for (int j = 0; j < VE; ++j) acc[(r * VE + j) * blockDim.x + tid] = 0.0;
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
        float accf[VE][NR];
#pragma unroll
        for (int j = 0; j < VE; ++j)
#pragma unroll
            for (int r = 0; r < NR; ++r) accf[j][r] = 0.f;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = base + (int64_t)u * blockDim.x;
            if (i < nunits) {
                float xf[VE], gf[VE], o[VE], t[VE], of[VE];
                L::unpack(xv[u], xf);
                L::unpack(gv[u], gf);
                bool tail = false;
#pragma unroll
                for (int j = 0; j < VE; ++j) Op::template bwd<P>(xf[j], gf[j], k, ch[j], tail, o[j], t[j]);
                if (tail) {
#pragma unroll
                    for (int j = 0; j < VE; ++j)
                        if (Op::template flag_bwd<P>(xf[j], k, ch[j]))
                            Op::template bwd_tail<P>(xf[j], gf[j], k, ch[j], o[j], t[j]);
                }
#pragma unroll
                for (int j = 0; j < VE; ++j) of[j] = Op::finish(xf[j], o[j], t[j], ch[j], accf[j]);
                L::store(dx, i, L::pack(of));
            }
        }
#pragma unroll
        for (int r = 0; r < NR; ++r)
#pragma unroll
            for (int j = 0; j < VE; ++j) acc[(r * VE + j) * blockDim.x + tid] += (double)accf[j][r];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            xv[u] = xn[u];
            gv[u] = gn[u];
        }
    }
    pdl_trigger();
    __syncthreads();
    const double *red = acc;
    const int rows = blockDim.x / groups;
    for (int o = tid; o < NR * C; o += blockDim.x) {
        const int r = o / C, c = o % C;
        const double *col = red + (r * VE + c % VE) * blockDim.x + c / VE;
        double s = 0.0;
        for (int q = 0; q < rows; ++q) s += col[q * groups];
        partials[(int64_t)blockIdx.x * NR * C + o] = s;
    }
}

// Backward, pipelined: the same work split and summation order as
// chan_nhwc_bwd_kernel (block b owns tiles b, b + grid, ...; fp32 sums per
// tile, fp64 per thread, one row of fp64 partials per block), but the x and
// dy tiles reach shared memory by 1-D bulk copies (cp.async.bulk) that one
// producer thread keeps `stages` tiles ahead, so the bytes in flight no
// longer cost registers.  Warp 0 is the producer; warps 1.. are consumers
// (blockDim.x - 32 of them, a multiple of the G = C / VE channel groups, so
// every consumer thread keeps the same VE channels).  A consumer copies its
// UT units of the tile from shared memory to registers, releases the stage
// (one arrival per warp on the stage's `empty` barrier), computes, and
// stores dx to global memory directly.  The partial tile at the end (fewer
// than a tile's units) is done with plain loads by the block that owns its
// index.  Waits are bounded: one that expires sets err[0] and the kernel
// finishes without computing further tiles.
//
// Shared memory: [0, 256) barriers; then NR VE * consumers fp64 running sums;
// then `stages` x {x tile, dy tile}.
constexpr int kPipeMaxStages = 8;
constexpr int kPipeHeader = 256;
// 96 registers: two blocks of 288 + 32 threads (C = 144) per SM.  Against
// three blocks of 64 registers (3 stages each), two blocks of 96 with 5
// stages each keep more bytes in flight and more independent elements per
// thread: measured on [128, 56, 56, 144] bf16, Swish 0.83 -> 0.87 of copy
// bandwidth, GELU-tanh 0.79 -> 0.84, ReLU unchanged.
#ifndef MEA_PIPE_MAXREGS
#define MEA_PIPE_MAXREGS 96
#endif
constexpr int kPipeMaxRegs = MEA_PIPE_MAXREGS;
// Tiles whose fp32 sums a consumer thread carries before adding them to its
// fp64 sums (kPipeFlushTiles * UT terms per channel in fp32).
constexpr int kPipeFlushTiles = 4;

// kWaitOut: the bounded-wait self-test.  The producer announces each stage's
// bytes but issues no copy, so no stage barrier ever completes (a flag that
// nothing sets); every wait gives up after kMbarSpinsSelfTest polls, records
// the error word and lets its role finish.  No copy is in flight when the
// block exits, and dx is not written.
template <class Op, typename T, int VE, int UT, bool kWaitOut = false>
__global__ void __maxnreg__(kPipeMaxRegs)
chan_nhwc_bwd_pipe_kernel(const void *__restrict__ x, const void *__restrict__ dy, ChanArgs ca,
                          void *__restrict__ dx, int64_t nunits, int groups, int C, int stages,
                          double *__restrict__ partials, unsigned int *__restrict__ err)
{
    using L = Unit<T, VE>;
    using W = typename L::W;
    constexpr bool P = L::P;
    constexpr int NR = Op::NR;
    constexpr int UB = sizeof(W);
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem);
    uint64_t *empty = full + kPipeMaxStages;
    const int consumers = blockDim.x - 32;
    double *acc = reinterpret_cast<double *>(smem + kPipeHeader);
    const size_t acc_bytes = ((size_t)NR * VE * consumers * sizeof(double) + 127) & ~(size_t)127;
    unsigned char *buf = smem + kPipeHeader + acc_bytes;
    const int64_t tile_units = (int64_t)consumers * UT;
    const uint32_t tile_bytes = (uint32_t)(tile_units * UB);
    const int64_t ntiles = nunits / tile_units;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr uint32_t spins = kWaitOut ? kMbarSpinsSelfTest : kMbarSpins;

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(smem_addr(full + s), 1);
            mbar_init(smem_addr(empty + s), consumers / 32);
        }
        mbar_init_fence();
    }
    __syncthreads();
    pdl_wait();

    if (warp == 0) {
        if (lane == 0) {
            // stage s of pass `phase` (it = phase * stages + s), stepped
            // without a division
            int it = 0, s = 0;
            uint32_t phase = 0;
            for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x, ++it) {
                if (it >= stages && !mbar_wait(smem_addr(empty + s), (phase & 1) ^ 1, spins)) {
                    atomicExch(err, 1u);
                    break;
                }
                const uint32_t fb = smem_addr(full + s);
                mbar_arrive_expect_tx(fb, 2 * tile_bytes);
                if constexpr (!kWaitOut) {
                    unsigned char *bx = buf + (size_t)s * 2 * tile_bytes;
                    bulk_load(smem_addr(bx), static_cast<const unsigned char *>(x) + t * tile_bytes, tile_bytes, fb);
                    bulk_load(smem_addr(bx + tile_bytes), static_cast<const unsigned char *>(dy) + t * tile_bytes,
                              tile_bytes, fb);
                }
                if (++s == stages) {
                    s = 0;
                    ++phase;
                }
            }
            // Every issued copy lands before the block may exit.
            for (int j = it > stages ? it - stages : 0; j < it; ++j)
                if (!mbar_wait(smem_addr(full + j % stages), (j / stages) & 1, spins)) atomicExch(err, 1u);
        }
        return;
    }

    const int ct = threadIdx.x - 32;
    const int g = ct % groups;
    const typename Op::K k = Op::kcoef(ca);
    typename Op::Ch ch[VE];
#pragma unroll
    for (int j = 0; j < VE; ++j) ch[j] = Op::load(ca, g * VE + j);
    typename Op::Ch2 ch2[VE / 2];
#pragma unroll
    for (int p = 0; p < VE / 2; ++p) ch2[p] = Op::pair(ch[2 * p], ch[2 * p + 1]);
#pragma unroll
    for (int r = 0; r < NR; ++r)
#pragma unroll
        for (int j = 0; j < VE; ++j) acc[(r * VE + j) * consumers + ct] = 0.0;

    // fp32 sums of up to kPipeFlushTiles tiles (UT terms per channel each),
    // then added to the thread's fp64 sums in shared memory.
    F2 accf[VE / 2][NR];
    auto clear = [&]() {
#pragma unroll
        for (int p = 0; p < VE / 2; ++p)
#pragma unroll
            for (int r = 0; r < NR; ++r) accf[p][r] = sp2(0.f);
    };
    auto flush = [&]() {
#pragma unroll
        for (int r = 0; r < NR; ++r)
#pragma unroll
            for (int p = 0; p < VE / 2; ++p) {
                float a0, a1;
                upk(accf[p][r], a0, a1);
                acc[(r * VE + 2 * p) * consumers + ct] += (double)a0;
                acc[(r * VE + 2 * p + 1) * consumers + ct] += (double)a1;
            }
        clear();
    };
    // One unit: VE elements of VE consecutive channels.
    auto unit = [&](const W &xw, const W &gw) -> W {
        float xf[VE], gf[VE], o[VE], tt[VE], of[VE];
        L::unpack(xw, xf);
        L::unpack(gw, gf);
        bool tail = false;
#pragma unroll
        for (int p = 0; p < VE / 2; ++p) {
            F2 o2, t2 = sp2(0.f);
            Op::template bwd2<P>(pk(xf[2 * p], xf[2 * p + 1]), pk(gf[2 * p], gf[2 * p + 1]), k, ch2[p], tail, o2,
                                 t2);
            upk(o2, o[2 * p], o[2 * p + 1]);
            upk(t2, tt[2 * p], tt[2 * p + 1]);
        }
        if (tail) {
            // only the flagged elements: bwd_tail picks the near-zero,
            // deep-tail or scalar form (the packed forms also flag elements
            // whose products could overflow)
#pragma unroll
            for (int j = 0; j < VE; ++j)
                if (Op::template flag_bwd<P>(xf[j], k, ch[j]))
                    Op::template bwd_tail<P>(xf[j], gf[j], k, ch[j], o[j], tt[j]);
        }
#pragma unroll
        for (int p = 0; p < VE / 2; ++p)
            upk(Op::finish2(pk(xf[2 * p], xf[2 * p + 1]), pk(o[2 * p], o[2 * p + 1]),
                            pk(tt[2 * p], tt[2 * p + 1]), ch2[p], accf[p]),
                of[2 * p], of[2 * p + 1]);
        return L::pack(of);
    };
    clear();

    int it = 0, s = 0;
    uint32_t phase = 0;
    for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x, ++it) {
        if (!mbar_wait(smem_addr(full + s), phase & 1, spins)) {
            atomicExch(err, 1u);
            break;
        }
        const W *sx = reinterpret_cast<const W *>(buf + (size_t)s * 2 * tile_bytes) + ct;
        const W *sg = reinterpret_cast<const W *>(buf + (size_t)s * 2 * tile_bytes + tile_bytes) + ct;
        W xv[UT], gv[UT];
#pragma unroll
        for (int u = 0; u < UT; ++u) {
            xv[u] = sx[u * consumers];
            gv[u] = sg[u * consumers];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(empty + s));
        // a whole tile: every unit is in range
        W *out = static_cast<W *>(dx) + t * tile_units + ct;
#pragma unroll
        for (int u = 0; u < UT; ++u) L::store(out, u * consumers, unit(xv[u], gv[u]));
        if ((it + 1) % kPipeFlushTiles == 0) flush();
        if (++s == stages) {
            s = 0;
            ++phase;
        }
    }
    // The partial tile at the end, if any, belongs to block ntiles % grid.
    if (ntiles * tile_units < nunits && blockIdx.x == ntiles % gridDim.x) {
        const int64_t base = ntiles * tile_units + ct;
#pragma unroll
        for (int u = 0; u < UT; ++u) {
            const int64_t i = base + (int64_t)u * consumers;
            if (i < nunits) L::store(dx, i, unit(L::load(x, i), L::load(dy, i)));
        }
    }
    flush();
    pdl_trigger();
    named_sync(1, consumers);
    const int rows = consumers / groups;
    for (int o = ct; o < NR * C; o += consumers) {
        const int r = o / C, c = o % C;
        const double *col = acc + (r * VE + c % VE) * consumers + c / VE;
        double sum = 0.0;
        for (int q = 0; q < rows; ++q) sum += col[q * groups];
        partials[(int64_t)blockIdx.x * NR * C + o] = sum;
    }
}

// Output o (r * C + c) = sum over the nb rows of partials, column o, in
// fp64: thread t adds rows t, t + kColsumThreads, ... in order, then a fixed
// block-wide tree.  One block per output; r = 0 goes to out0, r = 1 to out1.
template <int NR>
__global__ void __launch_bounds__(kColsumThreads)
chan_colsum_kernel(const double *__restrict__ partials, int nb, int C, float *__restrict__ out0,
                   float *__restrict__ out1)
{
    __shared__ double red[32];
    const int o = blockIdx.x;
    pdl_wait();
    pdl_trigger();
    double s = 0.0;
    for (int b = threadIdx.x; b < nb; b += kColsumThreads) s += partials[(int64_t)b * NR * C + o];
    s = block_sum(s, red);
    if (threadIdx.x == 0) {
        if (o < C) out0[o] = (float)s;
        else out1[o - C] = (float)s;
    }
}

// ------------------------------------------------------------ plane path

constexpr int kPlaneUnroll = 4;   // items in flight per thread

template <class Op, typename T, int MODE, bool NHWC>
__global__ void __launch_bounds__(kPlaneThreads, 3)
chan_plane_kernel(const void *__restrict__ x, const void *__restrict__ dy, ChanArgs ca, void *__restrict__ out,
                  int64_t N, int64_t C, int64_t HW, int slices, int vec_ok, float *__restrict__ out0,
                  float *__restrict__ out1, void *__restrict__ ws)
{
    constexpr bool P = Store<T>::P;
    constexpr int NR = Op::NR;
    const int64_t c = blockIdx.x / slices;
    const int s = blockIdx.x % slices;
    const int64_t n0 = (int64_t)s * N / slices, n1 = (int64_t)(s + 1) * N / slices;
    pdl_wait();
    const typename Op::K k = Op::kcoef(ca);
    const typename Op::Ch ch = Op::load(ca, (int)c);
    double acc[NR];
#pragma unroll
    for (int r = 0; r < NR; ++r) acc[r] = 0.0;

    // The block's planes in items of VL elements (a 16-byte vector, or one
    // element), kPlaneUnroll items per thread per step, loads first; the
    // reduction terms of an item are added in fp32, then in fp64.
    auto run = [&](auto vl) {
        constexpr int VL = decltype(vl)::value;
        using I = Item<T, VL>;
        const uint32_t per = (uint32_t)(HW / VL);
        const uint32_t total = (uint32_t)(n1 - n0) * per;
        const DivU32 div(per);
        const uint32_t bd = blockDim.x;
        for (uint32_t q0 = threadIdx.x; q0 < total; q0 += kPlaneUnroll * bd) {
            int64_t idx[kPlaneUnroll];
            typename I::Raw xr[kPlaneUnroll], gr[kPlaneUnroll];
#pragma unroll
            for (int u = 0; u < kPlaneUnroll; ++u) {
                const uint32_t q = q0 + u * bd;
                uint32_t nr, v;
                div.divmod(q < total ? q : 0u, nr, v);
                const int64_t n = n0 + nr;
                idx[u] = NHWC ? (n * HW + v) * C + c : (n * C + c) * per + v;
                if (q < total) {
                    xr[u] = I::load(x, idx[u]);
                    if constexpr (MODE == 1) gr[u] = I::load(dy, idx[u]);
                }
            }
#pragma unroll
            for (int u = 0; u < kPlaneUnroll; ++u) {
                if (q0 + u * bd >= total) continue;
                float xf[VL], gf[VL], of[VL];
                I::unpack(xr[u], xf);
                if constexpr (MODE == 1) I::unpack(gr[u], gf);
                bool tail = false;
                if constexpr (MODE == 0) {
#pragma unroll
                    for (int j = 0; j < VL; ++j) of[j] = Op::template f<P>(xf[j], k, ch, tail);
                    if (tail) {
#pragma unroll
                        for (int j = 0; j < VL; ++j)
                            if (Op::is_tail(xf[j], k, ch)) of[j] = Op::template f_tail<P>(xf[j], k, ch);
                    }
                } else {
                    float o[VL], t[VL];
#pragma unroll
                    for (int j = 0; j < VL; ++j) Op::template bwd<P>(xf[j], gf[j], k, ch, tail, o[j], t[j]);
                    if (tail) {
#pragma unroll
                        for (int j = 0; j < VL; ++j)
                            if (Op::template flag_bwd<P>(xf[j], k, ch))
                                Op::template bwd_tail<P>(xf[j], gf[j], k, ch, o[j], t[j]);
                    }
                    float tmp[NR];
#pragma unroll
                    for (int r = 0; r < NR; ++r) tmp[r] = 0.f;
#pragma unroll
                    for (int j = 0; j < VL; ++j) of[j] = Op::finish(xf[j], o[j], t[j], ch, tmp);
#pragma unroll
                    for (int r = 0; r < NR; ++r) acc[r] += (double)tmp[r];
                }
                I::store(out, idx[u], of);
            }
        }
    };
    if (!NHWC && vec_ok) run(std::integral_constant<int, Store<T>::V>{});
    else run(std::integral_constant<int, 1>{});
    pdl_trigger();
    if constexpr (MODE == 0) {
        return;
    } else {
        __shared__ double red[32];
        unsigned int *ticket = static_cast<unsigned int *>(ws);
        double *partials = reinterpret_cast<double *>(static_cast<char *>(ws) + kWsHeader);
#pragma unroll
        for (int r = 0; r < NR; ++r) {
            const double b = block_sum(acc[r], red);
            if (threadIdx.x == 0) partials[(r * C + c) * slices + s] = b;
        }
        if (!last_block_done(ticket, gridDim.x)) return;
        for (int64_t o = threadIdx.x; o < NR * C; o += blockDim.x) {
            double t = 0.0;
            for (int q = 0; q < slices; ++q) t += __ldcg(partials + o * slices + q);
            if (o < C) out0[o] = (float)t;
            else out1[o - C] = (float)t;
        }
    }
}

// ------------------------------------------------------------ launchers

inline int64_t nhwc_blocks(int64_t nunits, int threads, int U)
{
    const int64_t per = (int64_t)threads * U;
    const int64_t nb = (nunits + per - 1) / per;
    return nb < 1 ? 1 : nb;
}

// Backward grid: one block per tile up to kNhwcBwdGridCap blocks (a function
// of the shape only, so the summation order is fixed).
inline int nhwc_bwd_grid(int64_t nunits, int threads, int U)
{
    const int64_t nb = nhwc_blocks(nunits, threads, U);
    return (int)(nb < kNhwcBwdGridCap ? nb : kNhwcBwdGridCap);
}

template <typename T>
inline bool nhwc_fast(const AffineLaunch &a)
{
    constexpr int VE = NhwcCfg<T>::VE;
    constexpr int bytes = VE * (sizeof(T) == 4 ? 4 : 2);
    uintptr_t al = reinterpret_cast<uintptr_t>(a.x) | reinterpret_cast<uintptr_t>(a.out);
    if (a.dy) al |= reinterpret_cast<uintptr_t>(a.dy);
    return a.layout == 1 && a.C % VE == 0 && nhwc_threads((int)(a.C / VE)) > 0 && (al % bytes) == 0;
}

// Pipelined backward: shared memory per block is held to kPipeSmemBudget so
// that two blocks fit an SM (228 KB, 1 KB of it reserved per block), and
// the grid is at most kPipeGrid blocks (one wave of two per SM on a B200;
// a constant, so the summation order does not depend on the device).
#ifndef MEA_PIPE_SMEM_KB
#define MEA_PIPE_SMEM_KB 110
#endif
#ifndef MEA_PIPE_GRID
#define MEA_PIPE_GRID 296
#endif
constexpr int kPipeSmemBudget = MEA_PIPE_SMEM_KB * 1024;
constexpr int kPipeGrid = MEA_PIPE_GRID;

struct PipeShape {
    int stages;          // 0: the pipelined kernel is not used
    int grid;
    size_t smem;
};

template <typename T>
inline PipeShape pipe_shape(int nr, int64_t nunits, int consumers)
{
    constexpr int VE = NhwcCfg<T>::VE, UT = NhwcCfg<T>::U_PIPE;
    constexpr int UB = VE * (sizeof(T) == 4 ? 4 : 2);
    const size_t acc = ((size_t)nr * VE * consumers * sizeof(double) + 127) & ~(size_t)127;
    const size_t tile = (size_t)consumers * UT * UB;
    const long room = (long)kPipeSmemBudget - kPipeHeader - (long)acc;
    long stages = room > 0 ? room / (long)(2 * tile) : 0;
    if (stages > kPipeMaxStages) stages = kPipeMaxStages;
    if (stages < 2) return PipeShape{0, 0, 0};
    const int64_t ntiles = nunits / ((int64_t)consumers * UT);
    const int64_t grid = ntiles < 1 ? 1 : (ntiles < kPipeGrid ? ntiles : kPipeGrid);
    return PipeShape{(int)stages, (int)grid, kPipeHeader + acc + (size_t)stages * 2 * tile};
}

// Workspace of the backward of a per-channel operation with nr reductions:
// the larger of the NHWC fast path's and the plane path's needs (pointer
// alignment, which decides between them, is not known here).
inline size_t chan_bwd_workspace_bytes(int nr, int dtype, int layout, int64_t N, int64_t C, int64_t H, int64_t W)
{
    const int VE = dtype == kBF16 ? NhwcCfg<Bf16>::VE : NhwcCfg<float>::VE;
    const int U = dtype == kBF16 ? NhwcCfg<Bf16>::U_BWD : NhwcCfg<float>::U_BWD;
    size_t plane = kWsHeader + sizeof(double) * nr * (size_t)C * (size_t)plane_slices(N, C);
    if (layout == 1 && C % VE == 0 && nhwc_threads((int)(C / VE)) > 0) {
        const int threads = nhwc_threads((int)(C / VE));
        const int64_t nunits = N * C * H * W / VE;
        const int reg_rows = nhwc_bwd_grid(nunits, threads, U);
        const int pipe_rows = dtype == kBF16 ? pipe_shape<Bf16>(nr, nunits, threads).grid
                                             : pipe_shape<float>(nr, nunits, threads).grid;
        const int rows = reg_rows > pipe_rows ? reg_rows : pipe_rows;
        size_t fast = kWsHeader + sizeof(double) * nr * (size_t)C * (size_t)rows;
        return fast > plane ? fast : plane;
    }
    return plane;
}

template <class Op, typename T, int MODE>
cudaError_t launch_channel(const AffineLaunch &a, const ChanArgs &ca, float *out0, float *out1)
{
    constexpr int V = Store<T>::V;
    constexpr int NR = Op::NR;
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
            return launch_pdl(chan_nhwc_fwd_kernel<Op, T, U, VE>, dim3((unsigned)nb), dim3(threads), 0, a.stream, a.x,
                              ca, a.out, nunits, groups);
        }
        double *partials = reinterpret_cast<double *>(static_cast<char *>(a.workspace) + kWsHeader);
        unsigned int *err = reinterpret_cast<unsigned int *>(static_cast<char *>(a.workspace) + 4);
        const bool bulk_ok = ((reinterpret_cast<uintptr_t>(a.x) | reinterpret_cast<uintptr_t>(a.dy)) & 15u) == 0;
        const PipeShape ps = pipe_shape<T>(NR, nunits, threads);
        int nb;
        cudaError_t e;
        if (bulk_ok && ps.stages > 0) {
            auto kernel = chan_nhwc_bwd_pipe_kernel<Op, T, VE, NhwcCfg<T>::U_PIPE>;
            nb = ps.grid;
            e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                     (int)cudaSharedmemCarveoutMaxShared);
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ps.smem);
            if (e != cudaSuccess) return e;
            e = launch_pdl(kernel, dim3((unsigned)nb), dim3(threads + 32), ps.smem, a.stream, a.x, a.dy, ca, a.out,
                           nunits, groups, (int)a.C, ps.stages, partials, err);
        } else {
            constexpr int U = NhwcCfg<T>::U_BWD;
            auto kernel = chan_nhwc_bwd_kernel<Op, T, U, VE>;
            nb = nhwc_bwd_grid(nunits, threads, U);
            const size_t smem = sizeof(double) * NR * VE * threads;
            e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                     (int)cudaSharedmemCarveoutMaxShared);
            if (e == cudaSuccess && smem > 48 * 1024)
                e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
            e = launch_pdl(kernel, dim3((unsigned)nb), dim3(threads), smem, a.stream, a.x, a.dy, ca, a.out, nunits,
                           groups, (int)a.C, partials);
        }
        if (e != cudaSuccess) return e;
        return launch_pdl(chan_colsum_kernel<NR>, dim3((unsigned)(NR * a.C)), dim3(kColsumThreads), 0, a.stream,
                          partials, nb, (int)a.C, out0, out1);
    }
    uintptr_t al = reinterpret_cast<uintptr_t>(a.x) | reinterpret_cast<uintptr_t>(a.out);
    if (a.dy) al |= reinterpret_cast<uintptr_t>(a.dy);
    const int vec_ok = a.layout == 0 && HW % V == 0 && (al & 15u) == 0;
    const int slices = plane_slices(a.N, a.C);
    const int64_t grid = a.C * slices;
    if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
    if (a.layout == 1)
        return launch_pdl(chan_plane_kernel<Op, T, MODE, true>, dim3((unsigned)grid), dim3(kPlaneThreads), 0,
                          a.stream, a.x, a.dy, ca, a.out, a.N, a.C, HW, slices, vec_ok, out0, out1, a.workspace);
    return launch_pdl(chan_plane_kernel<Op, T, MODE, false>, dim3((unsigned)grid), dim3(kPlaneThreads), 0, a.stream,
                      a.x, a.dy, ca, a.out, a.N, a.C, HW, slices, vec_ok, out0, out1, a.workspace);
}

// The bounded-wait self-test: the pipelined NHWC backward of Op with its
// copies withheld (see kWaitOut).  cudaErrorNotSupported when the shape or
// the alignment does not take the pipelined path.
template <class Op, typename T>
cudaError_t launch_channel_wait_selftest(const AffineLaunch &a, const ChanArgs &ca)
{
    if (!nhwc_fast<T>(a)) return cudaErrorNotSupported;
    constexpr int VE = NhwcCfg<T>::VE;
    const int groups = (int)(a.C / VE);
    const int threads = nhwc_threads(groups);
    const int64_t nunits = a.N * a.C * a.H * a.W / VE;
    const bool bulk_ok = ((reinterpret_cast<uintptr_t>(a.x) | reinterpret_cast<uintptr_t>(a.dy)) & 15u) == 0;
    const PipeShape ps = pipe_shape<T>(Op::NR, nunits, threads);
    if (!bulk_ok || ps.stages <= 0) return cudaErrorNotSupported;
    double *partials = reinterpret_cast<double *>(static_cast<char *>(a.workspace) + kWsHeader);
    unsigned int *err = reinterpret_cast<unsigned int *>(static_cast<char *>(a.workspace) + 4);
    auto kernel = chan_nhwc_bwd_pipe_kernel<Op, T, VE, NhwcCfg<T>::U_PIPE, true>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                         (int)cudaSharedmemCarveoutMaxShared);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ps.smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(kernel, dim3((unsigned)ps.grid), dim3(threads + 32), ps.smem, a.stream, a.x, a.dy, ca, a.out,
                      nunits, groups, (int)a.C, ps.stages, partials, err);
}

}  // namespace mea
