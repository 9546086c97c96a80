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
// Row path (NCHW with planes of at most kRowMaxHW elements, aligned
// pointers): a block streams a contiguous run of whole planes in 16-byte
// vectors whatever H W is, finds each element's channel from its position,
// and sums each plane's reduction terms in fixed order (chan_row_kernel).
//
// Plane path (larger NCHW planes, unaligned NCHW tensors, and NHWC shapes the
// fast path does not take): block (c, s) owns channel c and the s-th slice
// of the batch; for NCHW it streams the contiguous H W planes of that
// channel (16-byte vectors when H W is a multiple of the vector width and
// the pointers are aligned), and the last block to finish (atomic ticket)
// adds the per-block partials in order.
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
constexpr int kPlaneBlocksTarget = 1184; // C * S is sized to about this many blocks (backward)
// The forward, with no reduction at its end, measured best with twice as many
// (NCHW fp32, Swish with alpha per channel: [64, 96, 112, 112] 0.834 -> 0.901
// of copy bandwidth, [64, 144, 56, 56] 0.797 -> 0.835, [64, 32, 112, 112]
// 0.837 -> 0.851); the backward lost 3-7% there and more with fewer.
constexpr int kPlaneBlocksTargetFwd = 2368;

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

// Slices of N per channel, so that C S is about `target` blocks: the
// backward's kPlaneBlocksTarget, or kPlaneBlocksTargetFwd for the forward.
inline int plane_slices(int64_t N, int64_t C, int64_t target = kPlaneBlocksTarget)
{
    int64_t s = (target + C - 1) / C;
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

// Backward, pipelined: a fixed work split (a function of the shape and the
// grid only; fp32 sums per few tiles, fp64 per thread, one row of fp64
// partials per block) in which the x and dy tiles reach shared memory by
// 1-D bulk copies (cp.async.bulk) that one producer thread keeps `stages`
// tiles ahead, so the bytes in flight cost no registers.  Warp 0 is the
// producer; warps 1.. are consumers (blockDim.x - 32 of them, a multiple of
// the G = C / VE channel groups, so every consumer thread keeps the same VE
// channels).  Block b owns tiles b, b + grid, ... below the last whole round
// of the grid (rounds * grid tiles).  A consumer copies its UT units of a
// tile from shared memory to registers, releases the stage (one arrival per
// warp on the stage's `empty` barrier), computes, and stores dx to global
// memory directly.  What is left after the whole rounds (the last
// ntiles % grid tiles and the partial tile) is cut into rows of `consumers`
// units, row r going to block r % grid, so that every block ends within a
// row of the others instead of ntiles % grid blocks taking one more tile;
// the consumers load their rows before the producer's first copies and
// compute them while the first stages are in flight.  Waits are bounded:
// one that expires sets err[0] and the kernel finishes without computing
// further tiles.
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
    // tiles of the whole rounds, which go through the stages
    const int64_t piped = nunits / tile_units / gridDim.x * gridDim.x;
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
    // The consumers' rows of the remainder are loaded before the producer
    // issues its first copies, so that they are not queued behind them.  The
    // remainder is under grid whole tiles (ntiles - piped < grid, plus a
    // partial tile), i.e. at most grid * UT rows: at most UT per block.
    constexpr int kLeft = UT;
    const int64_t r0 = piped * tile_units;
    const int ct = threadIdx.x - 32;
    W lx[kLeft], lg[kLeft];
    if (!kWaitOut && warp != 0) {
#pragma unroll
        for (int q = 0; q < kLeft; ++q) {
            const int64_t i = r0 + (blockIdx.x + (int64_t)q * gridDim.x) * consumers + ct;
            if (i < nunits) {
                lx[q] = L::load(x, i);
                lg[q] = L::load(dy, i);
            }
        }
    }
    __syncthreads();

    if (warp == 0) {
        if (lane == 0) {
            // stage s of pass `phase` (it = phase * stages + s), stepped
            // without a division
            int it = 0, s = 0;
            uint32_t phase = 0;
            for (int64_t t = blockIdx.x; t < piped; t += gridDim.x, ++it) {
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

    // This block's rows of the remainder, while the first stages are in
    // flight; none in the self-test, which writes no dx.
    if constexpr (!kWaitOut) {
#pragma unroll
        for (int q = 0; q < kLeft; ++q) {
            const int64_t i = r0 + (blockIdx.x + (int64_t)q * gridDim.x) * consumers + ct;
            if (i < nunits) L::store(dx, i, unit(lx[q], lg[q]));
        }
    }

    int it = 0, s = 0;
    uint32_t phase = 0;
    for (int64_t t = blockIdx.x; t < piped; t += gridDim.x, ++it) {
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

// ------------------------------------------------------------ row path
// NCHW with small planes (EfficientNet's 7 x 7 to 28 x 28 stages): the
// tensor read as N C planes of H W contiguous elements.  Block b owns the
// whole planes [b P, b P + P), a contiguous range of P H W elements that it
// streams in 16-byte vectors, so a plane of 49 elements costs no scalar
// loads and no stride.  P is a multiple of the vector width over
// gcd(H W, vector width), so every block starts on a 16-byte boundary; only
// the last block can end inside a vector (its ragged end goes element by
// element).  The constants of the block's planes sit in shared memory and
// each element finds its plane by counting positions within the vector.
//
// Backward: each element's reduction terms (fp32) are staged in shared
// memory; once the block's elements are done, warp w adds up planes w,
// w + 8, ... in fp64 (lane l takes positions l, l + 32, ...; then a fixed
// shuffle tree) and writes one value per plane and reduction to row n,
// column r C + c of the partials; a second kernel adds each column over the
// N rows in fixed order, one warp per column.  P depends only on the shape,
// so the sums are bitwise reproducible on any device.
constexpr int kRowThreads = 256;
constexpr int kRowUnroll = 4;            // vectors in flight per thread
// Blocks the row path aims at (148 SMs x 4), each of about N C / 592 planes.
// Measured on NCHW fp32, Swish with alpha per channel, batch 64, against
// 1184: forward at 14^2 0.603 -> 0.649 of copy bandwidth, 7^2 0.510 ->
// 0.539; backward at 14^2 0.524 -> 0.531, 7^2 0.412 -> 0.427; the three
// small stages grouped 0.840 -> 0.857 forward and 0.707 -> 0.734 backward;
// 28^2 level (its backward is held by the staging buffer).  Targets of 296
// to 4736 were measured; more blocks lost up to 40% in the forward, and 888
// lost 8% in the 7^2 backward.
constexpr int kRowBlocksTarget = 592;
constexpr int kRowTerms = 8192;          // fp32 terms staged per block (32 KB)
constexpr int kRowMaxPlanes = 256;
#ifndef MEA_ROW_MAX_HW
#define MEA_ROW_MAX_HW 1024
#endif
constexpr int64_t kRowMaxHW = MEA_ROW_MAX_HW;   // larger planes take the plane path

struct RowShape {
    int planes;          // P; 0: the row path is not taken
    int64_t grid;
};

// Lanes that add up one plane's terms: the largest power of two at most
// H W / 16, within 1 .. 32.
__device__ __forceinline__ uint32_t row_team(uint32_t hw)
{
    uint32_t ts = 1;
    while (ts < 32 && ts * 2 * 16 <= hw) ts *= 2;
    return ts;
}
// The lanes of lane's team of ts (a power of two) within its warp.
__device__ __forceinline__ unsigned row_team_mask(uint32_t lane, uint32_t ts)
{
    return ts == 32 ? 0xffffffffu : ((1u << ts) - 1u) << (lane & ~(ts - 1u));
}

// P for nr reductions and vl elements per 16-byte vector: about
// N C / kRowBlocksTarget planes, rounded up to the alignment multiple, at
// most what the staging buffer and the constants table hold.
inline RowShape row_shape(int nr, int vl, int64_t N, int64_t C, int64_t HW)
{
    const int64_t np = N * C;
    if (np < 1 || HW < 1 || HW > kRowMaxHW) return RowShape{0, 0};
    int64_t a = HW % vl, b = vl;
    while (a) {
        const int64_t t = b % a;
        b = a;
        a = t;
    }
    const int64_t m = vl / b;                 // planes per 16-byte-aligned step
    int64_t pmax = kRowMaxPlanes;
    if (nr > 0 && kRowTerms / (HW * nr) < pmax) pmax = kRowTerms / (HW * nr);
    pmax -= pmax % m;
    if (pmax < m) return RowShape{0, 0};
    int64_t p = (np + kRowBlocksTarget - 1) / kRowBlocksTarget;
    p = (p + m - 1) / m * m;
    if (p > pmax) p = pmax;
    return RowShape{(int)p, (np + p - 1) / p};
}

// Block `blk` of the row path over one tensor (the single-tensor kernel and
// every segment of the grouped one run this).  Dynamic shared memory: NR P
// H W floats in the backward.  The first vectors are requested before the
// constants table is filled, so the two memory round trips overlap.
template <class Op, typename T, int MODE>
__device__ __forceinline__ void row_body(const void *__restrict__ x, const void *__restrict__ dy, const ChanArgs &ca,
                                         void *__restrict__ out, int64_t C, int64_t HW, int64_t nplanes, int P,
                                         double *__restrict__ partials, int64_t blk)
{
    constexpr bool Pk = Store<T>::P;
    constexpr int NR = Op::NR;
    constexpr int VL = Store<T>::V;
    using I = Item<T, VL>;
    using I1 = Item<T, 1>;
    using Ch = typename Op::Ch;
    extern __shared__ float terms[];   // [NR][P H W], MODE 1 only
    __shared__ Ch chs[kRowMaxPlanes];
    const int64_t g0 = blk * P;
    const uint32_t np = (uint32_t)(nplanes - g0 < P ? nplanes - g0 : P);
    const uint32_t hw = (uint32_t)HW;
    const uint32_t L = np * hw;               // elements of the block
    const uint32_t ld = (uint32_t)P * hw;     // stride of terms between reductions
    const int64_t e0 = g0 * HW;
    const uint32_t nv = L / VL;
    const int64_t v0g = e0 / VL;
    typename I::Raw xr[kRowUnroll], gr[kRowUnroll];
    auto load_batch = [&](uint32_t q0) {
#pragma unroll
        for (int u = 0; u < kRowUnroll; ++u) {
            const uint32_t q = q0 + u * kRowThreads;
            if (q < nv) {
                xr[u] = I::load(x, v0g + q);
                if constexpr (MODE == 1) gr[u] = I::load(dy, v0g + q);
            }
        }
    };
    pdl_wait();
    load_batch(threadIdx.x);
    const typename Op::K k = Op::kcoef(ca);
    for (uint32_t i = threadIdx.x; i < np; i += kRowThreads) chs[i] = Op::load(ca, (int)((g0 + i) % C));
    __syncthreads();
    const DivU32 div(hw);
    const bool in_plane = hw % VL == 0;

    // One element of a plane whose constants are h: the value (MODE 0) or
    // dx and its reduction terms, written to tm[NR].
    auto elem = [&](float xv, float gv, const Ch &h, float (&tm)[NR]) -> float {
        bool tail = false;
        if constexpr (MODE == 0) {
            const float y = Op::template f<Pk>(xv, k, h, tail);
            return tail && Op::is_tail(xv, k, h) ? Op::template f_tail<Pk>(xv, k, h) : y;
        } else {
            float o, t;
            Op::template bwd<Pk>(xv, gv, k, h, tail, o, t);
            if (tail && Op::template flag_bwd<Pk>(xv, k, h)) Op::template bwd_tail<Pk>(xv, gv, k, h, o, t);
#pragma unroll
            for (int r = 0; r < NR; ++r) tm[r] = 0.f;
            return Op::finish(xv, o, t, h, tm);
        }
    };

    for (uint32_t q0 = threadIdx.x; q0 < nv; q0 += kRowUnroll * kRowThreads) {
        if (q0 != threadIdx.x) load_batch(q0);
#pragma unroll
        for (int u = 0; u < kRowUnroll; ++u) {
            const uint32_t q = q0 + u * kRowThreads;
            if (q >= nv) continue;
            float xf[VL], gf[VL], of[VL], tv[NR][VL];
            I::unpack(xr[u], xf);
            if constexpr (MODE == 1) I::unpack(gr[u], gf);
            uint32_t lp, pos;
            div.divmod(q * VL, lp, pos);
            // the backward reads the plane's constants again only where the
            // vector crosses into the next plane (measured: backward 28^2
            // 0.649 -> 0.659 of copy bandwidth), and when H W is a multiple
            // of VL (every vector then lies in one plane; the choice is the
            // same for the whole block, so no warp runs both forms) counts
            // no positions (28^2 0.646 -> 0.690); the forward reads them per
            // element, which measured faster there
            Ch h = chs[lp];
            if (MODE == 1 && in_plane) {
#pragma unroll
                for (int j = 0; j < VL; ++j) {
                    float tm[NR];
                    of[j] = elem(xf[j], MODE == 1 ? gf[j] : 0.f, h, tm);
#pragma unroll
                    for (int r = 0; r < NR; ++r) tv[r][j] = tm[r];
                }
            } else {
#pragma unroll
                for (int j = 0; j < VL; ++j) {
                    float tm[NR];
                    if constexpr (MODE == 0) {
                        if (j > 0) h = chs[lp];
                    }
                    of[j] = elem(xf[j], MODE == 1 ? gf[j] : 0.f, h, tm);
                    if constexpr (MODE == 1) {
#pragma unroll
                        for (int r = 0; r < NR; ++r) tv[r][j] = tm[r];
                    }
                    if (j + 1 < VL && ++pos == hw) {
                        pos = 0;
                        ++lp;
                        if constexpr (MODE == 1) h = chs[lp];
                    }
                }
            }
            I::store(out, v0g + q, of);
            if constexpr (MODE == 1) {
#pragma unroll
                for (int r = 0; r < NR; ++r)
#pragma unroll
                    for (int j = 0; j < VL; j += 4)
                        *reinterpret_cast<float4 *>(terms + r * ld + q * VL + j) =
                            make_float4(tv[r][j], tv[r][j + 1], tv[r][j + 2], tv[r][j + 3]);
            }
        }
    }
    // The ragged end of the last block (fewer than VL elements).
    for (uint32_t l = nv * VL + threadIdx.x; l < L; l += kRowThreads) {
        float tm[NR];
        const float xv = I1::load(x, e0 + l);
        const float gv = MODE == 1 ? (float)I1::load(dy, e0 + l) : 0.f;
        const float of[1] = {elem(xv, gv, chs[l / hw], tm)};
        I1::store(out, e0 + l, of);
        if constexpr (MODE == 1) {
#pragma unroll
            for (int r = 0; r < NR; ++r) terms[r * ld + l] = tm[r];
        }
    }
    pdl_trigger();
    if constexpr (MODE == 1) {
        __syncthreads();
        // A team of ts lanes per plane (about 16 terms per lane; a power of
        // two from 1 to 32, fixed by H W): lane i of a team adds positions
        // i, i + ts, ... in fp64, then a fixed shuffle tree within the team.
        auto sums = [&](auto tsc) {
            constexpr uint32_t TS = decltype(tsc)::value;
            const uint32_t lane = threadIdx.x & 31, sub = lane & (TS - 1);
            const unsigned mask = row_team_mask(lane, TS);
            for (uint32_t lp = threadIdx.x / TS; lp < np; lp += kRowThreads / TS) {
                const int64_t g = g0 + lp;
                const int64_t n = g / C, c = g - n * C;
#pragma unroll
                for (int r = 0; r < NR; ++r) {
                    double v = 0.0;
                    const float *tp = terms + r * ld + lp * hw;
#pragma unroll 4
                    for (uint32_t i = sub; i < hw; i += TS) v += (double)tp[i];
#pragma unroll
                    for (uint32_t off = TS >> 1; off >= 1; off >>= 1) v += __shfl_xor_sync(mask, v, off);
                    if (sub == 0) partials[(n * NR + r) * C + c] = v;
                }
            }
        };
        switch (row_team(hw)) {
        case 1: sums(std::integral_constant<uint32_t, 1>{}); break;
        case 2: sums(std::integral_constant<uint32_t, 2>{}); break;
        case 4: sums(std::integral_constant<uint32_t, 4>{}); break;
        case 8: sums(std::integral_constant<uint32_t, 8>{}); break;
        case 16: sums(std::integral_constant<uint32_t, 16>{}); break;
        default: sums(std::integral_constant<uint32_t, 32>{}); break;
        }
    }
}

// Column o of the row path's [N][NR C] partials: lane l adds rows l, l + 32,
// ... in order, then a fixed shuffle tree (one warp per column).
__device__ __forceinline__ double row_colsum(const double *__restrict__ partials, int64_t N, int64_t ld, int64_t o)
{
    double v = 0.0;
    for (int64_t n = threadIdx.x & 31; n < N; n += 32) v += partials[n * ld + o];
    return warp_sum(v);
}

template <class Op, typename T, int MODE>
__global__ void __launch_bounds__(kRowThreads)
chan_row_kernel(const void *__restrict__ x, const void *__restrict__ dy, ChanArgs ca, void *__restrict__ out,
                int64_t C, int64_t HW, int64_t nplanes, int P, double *__restrict__ partials)
{
    row_body<Op, T, MODE>(x, dy, ca, out, C, HW, nplanes, P, partials, blockIdx.x);
}

// Output o (r C + c) of the row path: r = 0 to out0, r = 1 to out1.
template <int NR>
__global__ void __launch_bounds__(kRowThreads)
chan_row_colsum_kernel(const double *__restrict__ partials, int64_t N, int64_t C, float *__restrict__ out0,
                       float *__restrict__ out1)
{
    pdl_wait();
    pdl_trigger();
    const int64_t o = (int64_t)blockIdx.x * (kRowThreads / 32) + (threadIdx.x >> 5);
    if (o >= NR * C) return;
    const double v = row_colsum(partials, N, NR * C, o);
    if ((threadIdx.x & 31) == 0) {
        if (o < C) out0[o] = (float)v;
        else out1[o - C] = (float)v;
    }
}

// Grouped row path: segments laid end to end in one grid (block ranges
// start[s] .. start[s + 1]); the column sums of segment s are outputs
// ostart[s] .. ostart[s + 1] of the second kernel.  Each segment's blocks
// and sums are those of its single-tensor launch, so its results are
// bitwise the same.
constexpr int kMaxRowSegs = 32;
struct RowSeg {
    const void *x;
    const void *dy;
    void *out;
    const float *p0;
    const float *p1;
    double *partials;
    float *out0;
    float *out1;
    int64_t N, C, HW;
    int P;
};
struct RowSegTable {
    RowSeg seg[kMaxRowSegs];
    int start[kMaxRowSegs + 1];
    int ostart[kMaxRowSegs + 1];
    int nseg;
    float scalar;
};
static_assert(sizeof(RowSegTable) < 4000, "kernel parameter space");

template <class Op, typename T, int MODE>
__global__ void __launch_bounds__(kRowThreads)
chan_row_group_kernel(const __grid_constant__ RowSegTable tab)
{
    int s = 0;
    while (s + 1 < tab.nseg && (int)blockIdx.x >= tab.start[s + 1]) ++s;
    const RowSeg &g = tab.seg[s];
    const ChanArgs ca{g.p0, g.p1, tab.scalar};
    row_body<Op, T, MODE>(g.x, g.dy, ca, g.out, g.C, g.HW, g.N * g.C, g.P, g.partials,
                          (int64_t)blockIdx.x - tab.start[s]);
}

template <int NR>
__global__ void __launch_bounds__(kRowThreads)
chan_row_group_colsum_kernel(const __grid_constant__ RowSegTable tab)
{
    pdl_wait();
    pdl_trigger();
    const int64_t og = (int64_t)blockIdx.x * (kRowThreads / 32) + (threadIdx.x >> 5);
    if (og >= tab.ostart[tab.nseg]) return;
    int s = 0;
    while (s + 1 < tab.nseg && og >= tab.ostart[s + 1]) ++s;
    const RowSeg &g = tab.seg[s];
    const int64_t o = og - tab.ostart[s];
    const double v = row_colsum(g.partials, g.N, NR * g.C, o);
    if ((threadIdx.x & 31) == 0) {
        if (o < g.C) g.out0[o] = (float)v;
        else g.out1[o - g.C] = (float)v;
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
    if (layout == 0 && row_shape(nr, dtype == kBF16 ? Store<Bf16>::V : Store<float>::V, N, C, H * W).planes > 0) {
        const size_t row = kWsHeader + sizeof(double) * nr * (size_t)C * (size_t)N;
        if (row > plane) plane = row;
    }
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
    const RowShape rs = a.layout == 0 ? row_shape(NR, V, a.N, a.C, HW) : RowShape{0, 0};
    if (rs.planes > 0 && (al & 15u) == 0) {
        if (rs.grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
        double *partials = reinterpret_cast<double *>(static_cast<char *>(a.workspace) + kWsHeader);
        const size_t smem = MODE == 1 ? sizeof(float) * NR * (size_t)rs.planes * (size_t)HW : 0;
        cudaError_t e = launch_pdl(chan_row_kernel<Op, T, MODE>, dim3((unsigned)rs.grid), dim3(kRowThreads), smem,
                                   a.stream, a.x, a.dy, ca, a.out, a.C, HW, a.N * a.C, rs.planes, partials);
        if (e != cudaSuccess || MODE == 0) return e;
        const int64_t cb = (NR * a.C + kRowThreads / 32 - 1) / (kRowThreads / 32);
        return launch_pdl(chan_row_colsum_kernel<NR>, dim3((unsigned)cb), dim3(kRowThreads), 0, a.stream,
                          static_cast<const double *>(partials), a.N, a.C, out0, out1);
    }
    const int vec_ok = a.layout == 0 && HW % V == 0 && (al & 15u) == 0;
    const int slices = plane_slices(a.N, a.C, MODE == 0 ? kPlaneBlocksTargetFwd : kPlaneBlocksTarget);
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
