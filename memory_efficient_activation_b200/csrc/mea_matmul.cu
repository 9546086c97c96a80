// mea_matmul.cu -- a matrix multiply with the activation fused into its
// epilogue, on the fifth-generation tensor cores (tcgen05, accumulators in
// tensor memory, operands staged by TMA).
//
//   forward:   Z = X W^T (fp32 accumulation), stored in bf16, and
//              Y = f(Z as stored)
//   backward:  dZ = (G W^T) f'(Z), Z the stored bf16 pre-activation
//
// Problem B07 of "What activations cost, in memory and in arithmetic"
// (SOLUTION, step 4) sets the activation after a d x d matrix multiply on
// the same tensor and observes that the activation's arithmetic is free
// beside it while its memory is not.  Fusing it into the matmul's epilogue
// keeps only Z for the backward, writes f(Z) without a second pass over Z,
// and in the backward multiplies the product by f'(Z) before it ever
// reaches memory (no G W^T tensor is written or re-read).
//
// Kernel (persistent, clusters of two CTAs on two SMs, 192 threads each):
// a CTA pair owns a 256 x 256 output tile and multiplies it with the
// two-SM form of the tensor-core instruction (tcgen05.mma.cta_group::2):
// each CTA stages its own 128 rows of X and its own 128 rows of W per K
// step, and one instruction issued by the pair's first CTA reads A from
// both CTAs' shared memory (M 256) and B from both (N 256), writing a
// 128 x 256 fp32 accumulator into each CTA's tensor memory.  Per CTA:
//   warp 0      one thread issues TMA loads of 128 x 64 tiles of X and W
//               (128-byte swizzle, no multicast) into a 7-stage ring; the
//               loads of both CTAs complete on the first CTA's barrier
//   warp 1      allocates 512 tensor-memory columns (two accumulators) in
//               both CTAs; in the first CTA one thread issues the MMAs and
//               commits each stage and each finished accumulator to the
//               barriers of both CTAs (tcgen05.commit multicast)
//   warps 2..5  read this CTA's accumulator rows (tcgen05.ld, one row per
//               thread), apply the epilogue, store, and release the
//               accumulator to the first CTA, while the other is filled
// Tiles are assigned round-robin to CTA pairs; each tile's sum runs over k
// in one fixed order, so results do not depend on the grid.  Every barrier
// wait is bounded: one that expires sets g_matmul_error and the roles stop
// issuing work.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "mea_device.cuh"
#include "mea_internal.h"
#include "mea_math.cuh"
#include "mea_matmul_api.h"
#include "mea_pipe.cuh"

namespace mea {

__device__ unsigned int g_matmul_error = 0;

namespace {

constexpr int kBM = kMatmulBM, kBN = kMatmulBN, kBK = kMatmulBK;   // tile of a CTA pair: 256 x 256
constexpr int kHalf = 128;                                  // rows of X and of W one CTA stages
constexpr int kUmmaK = 16;                                  // K of one bf16 MMA
constexpr int kStages = 7;
constexpr int kThreadsMM = 192;
constexpr uint32_t kStageA = kHalf * kBK * 2;                // 16 KB
constexpr uint32_t kStageB = kHalf * kBK * 2;                // 16 KB
constexpr uint32_t kStageBytes = kStageA + kStageB;
constexpr uint32_t kAccCols = kBN;                           // fp32 columns per accumulator
constexpr uint32_t kTmemCols = 2 * kAccCols;                 // 512: all of tensor memory
constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kStageBytes + 256;

// Instruction descriptor of tcgen05.mma.kind::f16: fp32 accumulator (bits
// 4-5 = 1), A and B bf16 (bits 7-9 = 1, 10-12 = 1), both K-major (bits 15,
// 16 = 0), N / 8 in bits 17-22, M / 16 in bits 24-28 (M 256: the pair).
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) |
                            ((uint32_t)(kBM >> 4) << 24);

// Shared-memory matrix descriptor of a K-major operand tile written by TMA
// with the 128-byte swizzle: rows of 64 bf16 (128 bytes), 8-row groups
// 1024 bytes apart.  Fields: start address / 16 (bits 0-13), leading byte
// offset / 16 (bits 16-29; not used by swizzled K-major layouts, set to 1),
// stride byte offset / 16 (bits 32-45), descriptor version 1 (bits 46-47),
// base offset 0 (tiles are 1024-byte aligned), swizzle mode 2 = 128-byte
// (bits 61-63).  A K step of 16 elements inside the 128-byte row advances
// the start address by 32 bytes.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// TMA load into this CTA's shared memory that completes on `bar`, a
// shared::cluster address that may lie in the other CTA of the pair.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, int x, int y, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
        "%3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// shared::cluster address of the variable at `saddr` in CTA `rank` of the
// cluster.
__device__ __forceinline__ uint32_t cluster_addr(uint32_t saddr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cbar)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cbar) : "memory");
}

__device__ __forceinline__ void umma_bf16_pair(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t accumulate)
{
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
            tmem_d),
        "l"(a), "l"(b), "r"(kIdesc), "r"(accumulate)
        : "memory");
}

// Arrives once on the barrier at `bar` in both CTAs of the pair when every
// tcgen05.mma this thread issued so far has completed.
__device__ __forceinline__ void umma_commit_pair(uint32_t bar)
{
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
        "h"((uint16_t)3)
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive fp32 columns of this warp's 32 tensor-memory lanes: thread
// i of the warp receives lane (base lane + i), columns col .. col + 31.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void record_error() { atomicExch(&g_matmul_error, 1u); }

// Epilogue of one row segment of 32 columns.  acc: the fp32 accumulator
// bits; zp: the stored Z (backward); outputs as in MatmulLaunch.
template <class A, int MODE>
__device__ __forceinline__ void epilogue32(const uint32_t (&acc)[32], const Coef &k, const uint16_t *zp,
                                           uint16_t *o0, uint16_t *o1, int ncols)
{
    float zr[32], r[32];
    uint32_t zb[16];
    if constexpr (MODE == 0) {
        // Z rounded to bf16 once; f is evaluated at the stored value.
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            zb[j] = pack_bf16x2(__uint_as_float(acc[2 * j]), __uint_as_float(acc[2 * j + 1]));
            zr[2 * j] = __uint_as_float(zb[j] << 16);
            zr[2 * j + 1] = __uint_as_float(zb[j] & 0xffff0000u);
        }
        bool tail = false;
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] = A::template f<false>(zr[j], k, tail);
        if (tail) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (A::is_tail(zr[j], k)) r[j] = A::template f_tail<false>(zr[j], k);
        }
    } else {
        if (ncols == 32) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 w = ld_nc_v4(reinterpret_cast<const uint4 *>(zp) + q);
                zb[4 * q] = w.x;
                zb[4 * q + 1] = w.y;
                zb[4 * q + 2] = w.z;
                zb[4 * q + 3] = w.w;
            }
        } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const uint32_t lo = 2 * j < ncols ? zp[2 * j] : 0u;
                const uint32_t hi = 2 * j + 1 < ncols ? zp[2 * j + 1] : 0u;
                zb[j] = lo | (hi << 16);
            }
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            zr[2 * j] = __uint_as_float(zb[j] << 16);
            zr[2 * j + 1] = __uint_as_float(zb[j] & 0xffff0000u);
        }
        bool tail = false;
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] = A::template df<false>(zr[j], __uint_as_float(acc[j]), k, tail);
        if (tail) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (A::template is_tail_bwd<false>(zr[j], k))
                    r[j] = A::template df_tail<false>(zr[j], __uint_as_float(acc[j]), k);
        }
    }
    uint32_t rb[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) rb[j] = pack_bf16x2(r[2 * j], r[2 * j + 1]);
    if (ncols == 32) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            if (MODE == 0 && o0)
                st_v4(reinterpret_cast<uint4 *>(o0) + q, make_uint4(zb[4 * q], zb[4 * q + 1], zb[4 * q + 2], zb[4 * q + 3]));
            if (o1)
                st_v4(reinterpret_cast<uint4 *>(o1) + q, make_uint4(rb[4 * q], rb[4 * q + 1], rb[4 * q + 2], rb[4 * q + 3]));
        }
    } else {
        for (int j = 0; j < ncols; ++j) {
            if (MODE == 0 && o0) o0[j] = (uint16_t)(j & 1 ? zb[j >> 1] >> 16 : zb[j >> 1] & 0xffffu);
            if (o1) o1[j] = (uint16_t)(j & 1 ? rb[j >> 1] >> 16 : rb[j >> 1] & 0xffffu);
        }
    }
}

template <class A, int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreadsMM, 1)
matmul_act_kernel(const __grid_constant__ CUtensorMap tma_x, const __grid_constant__ CUtensorMap tma_w, int M,
                  int N, int K, float param, const uint16_t *__restrict__ zin, uint16_t *__restrict__ out0,
                  uint16_t *__restrict__ out1)
{
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    unsigned char *smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);   // 1024-byte aligned tiles
    const uint32_t sbase = smem_addr(smem);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kStages * kStageBytes);
    uint64_t *empty = full + kStages;
    uint64_t *acc_full = empty + kStages;
    uint64_t *acc_empty = acc_full + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();          // 0: issues the MMAs of the pair
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int tiles_m = (M + kBM - 1) / kBM, tiles_n = (N + kBN - 1) / kBN;
    const int ntiles = tiles_m * tiles_n;
    const int kblocks = (K + kBK - 1) / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_addr(full + s), 1);     // the first CTA's producer; bytes of both CTAs
            mbar_init(smem_addr(empty + s), 1);    // one commit from the first CTA
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_addr(acc_full + b), 1);
            mbar_init(smem_addr(acc_empty + b), 8); // four epilogue warps of each CTA
        }
        mbar_init_fence();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync();                                // barriers of both CTAs initialised
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();

    if (warp == 0) {
        if (lane == 0) {
            // TMA producer: this CTA's rows of X and W; completion on the
            // first CTA's barrier
            int it = 0;
            bool ok = true;
            for (int t = pair; t < ntiles && ok; t += npairs) {
                const int tm = t / tiles_n, tn = t % tiles_n;
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const int s = it % kStages, round = it / kStages;
                    if (round > 0 && !mbar_wait(smem_addr(empty + s), (round & 1) ^ 1)) {
                        record_error();
                        ok = false;
                        break;
                    }
                    const uint32_t fb = cluster_addr(smem_addr(full + s), 0);
                    if (rank == 0) mbar_arrive_expect_tx(smem_addr(full + s), 2 * kStageBytes);
                    const uint32_t sa = sbase + s * kStageBytes;
                    tma_load_2d_pair(sa, &tma_x, kb * kBK, tm * kBM + rank * kHalf, fb);
                    tma_load_2d_pair(sa + kStageA, &tma_w, kb * kBK, tn * kBN + rank * kHalf, fb);
                }
            }
            // every load issued has landed before teardown: this CTA's stages
            // are released (empty) once the MMAs that read them complete
            for (int j = it > kStages ? it - kStages : 0; j < it; ++j)
                if (!mbar_wait(smem_addr(empty + j % kStages), (j / kStages) & 1)) record_error();
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // MMA issuer of the pair
            int it = 0, lt = 0;
            bool ok = true;
            for (int t = pair; t < ntiles && ok; t += npairs, ++lt) {
                const int b = lt & 1, use = lt >> 1;
                if (use > 0 && !mbar_wait(smem_addr(acc_empty + b), (use & 1) ^ 1)) {
                    record_error();
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem + b * kAccCols;
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const int s = it % kStages;
                    if (!mbar_wait(smem_addr(full + s), (it / kStages) & 1)) {
                        record_error();
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = sbase + s * kStageBytes;
#pragma unroll
                    for (int k = 0; k < kBK / kUmmaK; ++k)
                        umma_bf16_pair(d, sdesc_sw128(sa + k * kUmmaK * 2),
                                       sdesc_sw128(sa + kStageA + k * kUmmaK * 2), (kb | k) != 0);
                    umma_commit_pair(smem_addr(empty + s));
                }
                if (ok) umma_commit_pair(smem_addr(acc_full + b));
            }
        }
        __syncwarp();
    } else {
        // epilogue: warp w reads tensor-memory lanes 32 (w % 4) .. + 31 of
        // this CTA, i.e. rows rank * 128 + 32 (w % 4) + lane of the tile
        const int q = warp & 3;
        const Coef k = A::coef(param);
        const uint32_t release = cluster_addr(smem_addr(acc_empty), 0);
        int lt = 0;
        for (int t = pair; t < ntiles; t += npairs, ++lt) {
            const int b = lt & 1, use = lt >> 1;
            if (!mbar_wait(smem_addr(acc_full + b), use & 1)) {
                record_error();
                break;
            }
            tc_fence_after();
            const int tm = t / tiles_n, tn = t % tiles_n;
            const int row = tm * kBM + (int)rank * kHalf + q * 32 + lane;
#pragma unroll 1
            for (int c = 0; c < kBN / 32; ++c) {
                uint32_t v[32];
                tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + b * kAccCols + c * 32, v);
                const int col = tn * kBN + c * 32;
                if (row < M && col < N) {
                    const int ncols = N - col < 32 ? N - col : 32;
                    const size_t off = (size_t)row * N + col;
                    epilogue32<A, MODE>(v, k, MODE == 1 ? zin + off : nullptr, out0 ? out0 + off : nullptr,
                                        out1 ? out1 + off : nullptr, ncols);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(release + 8 * b);
        }
    }
    pdl_trigger();
    tc_fence_before();
    cluster_sync();                                // no CTA leaves while its pair may touch its memory
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

// ------------------------------------------------------------ host side

using EncodeTiled = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                 const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encoder()
{
    static EncodeTiled fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(p);
    });
    return fn;
}

// 2-D map of a row-major bf16 [rows x cols] matrix, box of box_rows x 64.
bool make_map(CUtensorMap *map, const void *base, int64_t rows, int64_t cols, uint32_t box_rows)
{
    EncodeTiled enc = encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kBK, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <class A, int MODE>
cudaError_t launch_one(const MatmulLaunch &a, const CUtensorMap &mx, const CUtensorMap &mw)
{
    auto kernel = matmul_act_kernel<A, MODE>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    const int64_t tiles = ((a.M + kBM - 1) / kBM) * ((a.N + kBN - 1) / kBN);
    const int pairs_max = sm_count() / 2;
    const int pairs = (int)(tiles < pairs_max ? tiles : pairs_max);
    return launch_pdl(kernel, dim3((unsigned)(2 * pairs)), dim3(kThreadsMM), kSmemBytes, a.stream, mx, mw, (int)a.M,
                      (int)a.N, (int)a.K, a.param, static_cast<const uint16_t *>(a.zin),
                      static_cast<uint16_t *>(a.out0), static_cast<uint16_t *>(a.out1));
}

template <int MODE>
cudaError_t by_act(const MatmulLaunch &a, const CUtensorMap &mx, const CUtensorMap &mw)
{
    switch (a.act) {
    case 0: return launch_one<ReLU, MODE>(a, mx, mw);
    case 1: return launch_one<LeakyReLU, MODE>(a, mx, mw);
    case 2: return launch_one<Sigmoid, MODE>(a, mx, mw);
    case 3: return launch_one<Tanh, MODE>(a, mx, mw);
    case 4: return launch_one<GeluErf, MODE>(a, mx, mw);
    case 5: return launch_one<GeluTanh, MODE>(a, mx, mw);
    case 6: return launch_one<Swish, MODE>(a, mx, mw);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t matmul_error_word(int clear, unsigned int *word)
{
    cudaError_t e = cudaMemcpyFromSymbol(word, g_matmul_error, sizeof(unsigned int));
    if (e == cudaSuccess && clear) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_matmul_error, &zero, sizeof(unsigned int));
    }
    return e;
}

cudaError_t launch_matmul_act(const MatmulLaunch &a)
{
    CUtensorMap mx, mw;
    if (!make_map(&mx, a.x, a.M, a.K, kHalf) || !make_map(&mw, a.w, a.N, a.K, kHalf)) return cudaErrorInvalidValue;
    return a.mode == 0 ? by_act<0>(a, mx, mw) : by_act<1>(a, mx, mw);
}

}  // namespace mea
