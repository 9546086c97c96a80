// mea_device.cuh -- device-side building blocks shared by the streaming
// kernels: 16-byte global loads and stores, bf16/fp32 storage adapters,
// fixed-order register sums and the deterministic block / grid reduction.
#pragma once

#include <cstdint>

#include "mea_internal.h"

namespace mea {

// ------------------------------------------------- programmatic dependence
//
// Every kernel of the library is launched with programmatic stream
// serialisation (see launch_pdl in mea_internal.h): the next kernel on the
// stream may be scheduled while this one drains.  pdl_wait() must come
// before the first access to memory a preceding kernel may write; it returns
// once every preceding grid on the stream has completed and its memory is
// visible (and at once when the launch carried no such dependence).
// pdl_trigger() tells the hardware that the dependent grid may start
// launching; it does not weaken pdl_wait() in the dependent.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------- memory helpers

// 16-byte load through the non-coherent (read-only) path, not allocated in
// L1: every byte is used exactly once.
__device__ __forceinline__ uint4 ld_nc_v4(const uint4 *p)
{
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p));
    return r;
}

__device__ __forceinline__ void st_v4(uint4 *p, const uint4 &v)
{
    asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};"
                 :
                 : "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// fp32 pair -> bf16x2, round to nearest even (cvt.rn.bf16x2.f32 puts its
// first source in the upper half).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ uint16_t to_bf16(float v)
{
    uint16_t r;
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(v));
    return r;
}

struct Bf16 {};  // tag type for bfloat16 storage

template <typename T>
struct Store;

template <>
struct Store<float> {
    static constexpr int V = 4;          // elements per 16-byte vector
    static constexpr bool P = true;      // precise exponent arguments
    static constexpr int kBytes = 4;
    static __device__ __forceinline__ void unpack(const uint4 &w, float (&f)[V])
    {
        f[0] = __uint_as_float(w.x);
        f[1] = __uint_as_float(w.y);
        f[2] = __uint_as_float(w.z);
        f[3] = __uint_as_float(w.w);
    }
    static __device__ __forceinline__ uint4 pack(const float (&f)[V])
    {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                          __float_as_uint(f[3]));
    }
    static __device__ __forceinline__ float load1(const void *p, int64_t i)
    {
        return __ldg(static_cast<const float *>(p) + i);
    }
    static __device__ __forceinline__ void store1(void *p, int64_t i, float v)
    {
        static_cast<float *>(p)[i] = v;
    }
};

template <>
struct Store<Bf16> {
    static constexpr int V = 8;
    static constexpr bool P = false;
    static constexpr int kBytes = 2;
    static __device__ __forceinline__ void unpack(const uint4 &w, float (&f)[V])
    {
        const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            f[2 * q] = __uint_as_float(u[q] << 16);
            f[2 * q + 1] = __uint_as_float(u[q] & 0xffff0000u);
        }
    }
    static __device__ __forceinline__ uint4 pack(const float (&f)[V])
    {
        return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                          pack_bf16x2(f[6], f[7]));
    }
    static __device__ __forceinline__ float load1(const void *p, int64_t i)
    {
        uint16_t b = __ldg(static_cast<const unsigned short *>(p) + i);
        return __uint_as_float(static_cast<uint32_t>(b) << 16);
    }
    static __device__ __forceinline__ void store1(void *p, int64_t i, float v)
    {
        static_cast<uint16_t *>(p)[i] = to_bf16(v);
    }
};

// ------------------------------------------------------- fixed-order sums

template <int V>
__device__ __forceinline__ float tree_sum(const float (&t)[V])
{
    float s[V];
#pragma unroll
    for (int j = 0; j < V; ++j) s[j] = t[j];
#pragma unroll
    for (int w = V / 2; w >= 1; w /= 2) {
#pragma unroll
        for (int j = 0; j < w; ++j) s[j] = s[j] + s[j + w];
    }
    return s[0];
}

__device__ __forceinline__ double warp_sum(double v)
{
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// Block-wide sum in a fixed order (xor butterfly per warp, then warp 0 over
// the warp results).  Valid in thread 0.  red must hold 32 doubles.  Every
// thread of the block must call it.
__device__ __forceinline__ double block_sum(double v, double *red)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwarps = (blockDim.x + 31) >> 5;
    v = warp_sum(v);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    double r = 0.0;
    if (warp == 0) {
        r = lane < nwarps ? red[lane] : 0.0;
        r = warp_sum(r);
    }
    __syncthreads();
    return r;
}

// Grid completion ticket: returns true in every thread of the one block
// that finishes last (after all other blocks have published their partials
// with a fence).  The counter wraps back to zero, leaving the workspace as
// it was found.  Nothing waits.
__device__ __forceinline__ bool last_block_done(unsigned int *ticket, unsigned int nblk)
{
    __shared__ int is_last;
    __threadfence();          // every thread's partial stores are visible device-wide
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned int t = atomicInc(ticket, nblk - 1);
        is_last = (t == nblk - 1);
    }
    __syncthreads();
    const bool last = is_last != 0;
    if (last) __threadfence();
    return last;
}

}  // namespace mea
