// mea_stream.cuh -- helpers of the plane-streaming kernels: division by a
// fixed divisor without a division instruction, and 16-byte / one-element
// item access that keeps loads raw until they are used.
#pragma once

#include <cstdint>
#include <type_traits>

#include "mea_device.cuh"

namespace mea {

// Unsigned division by a fixed d >= 1 for dividends below 2^31: q = (hi(n m)
// + n) >> s with s = ceil(log2 d), m = floor(2^32 (2^s - d) / d) + 1 (the
// round-up method of Granlund and Montgomery, "Division by invariant integers
// using multiplication", 1994).
struct DivU32 {
    uint32_t d, m, s;
    __device__ __forceinline__ explicit DivU32(uint32_t dd) : d(dd)
    {
        s = 0;
        while ((1u << s) < d && s < 31) ++s;
        m = (uint32_t)((((uint64_t)1 << 32) * (((uint64_t)1 << s) - d)) / d + 1);
    }
    __device__ __forceinline__ void divmod(uint32_t n, uint32_t &q, uint32_t &r) const
    {
        q = (__umulhi(n, m) + n) >> s;
        r = n - q * d;
    }
};

// Item access: VL = V loads a 16-byte vector, VL = 1 one element.  Loads
// keep the raw bits (unpacked when used) so four items in flight cost few
// registers.
template <typename T, int VL>
struct Item {
    using Raw = typename std::conditional<VL == 1, float, uint4>::type;
    static __device__ __forceinline__ Raw load(const void *p, int64_t i)
    {
        if constexpr (VL == 1) {
            return Store<T>::load1(p, i);
        } else {
            return ld_nc_v4(static_cast<const uint4 *>(p) + i);
        }
    }
    static __device__ __forceinline__ Raw load_rw(const void *p, int64_t i)
    {
        if constexpr (VL == 1) {
            return Store<T>::load1(p, i);
        } else {
            return *(static_cast<const uint4 *>(p) + i);
        }
    }
    static __device__ __forceinline__ void unpack(const Raw &r, float (&f)[VL])
    {
        if constexpr (VL == 1) {
            f[0] = r;
        } else {
            Store<T>::unpack(r, f);
        }
    }
    static __device__ __forceinline__ void store(void *p, int64_t i, const float (&f)[VL])
    {
        if constexpr (VL == 1) {
            Store<T>::store1(p, i, f[0]);
        } else {
            st_v4(static_cast<uint4 *>(p) + i, Store<T>::pack(f));
        }
    }
};

}  // namespace mea
