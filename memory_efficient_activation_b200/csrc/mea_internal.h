// mea_internal.h -- launchers shared between the C-ABI layer and the kernels.
// Not installed; the public interface is include/mea.h.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace mea {

// Storage dtype and activation ids follow include/mea.h.
enum Dtype { kF32 = 0, kBF16 = 1 };

constexpr int kThreads = 256;          // threads per block of the streaming kernels
constexpr int kUnroll = 4;             // 16-byte vectors per thread per iteration
constexpr int kRedGridMax = 444;       // 148 SMs x 3 resident blocks: one wave on a B200
constexpr int kRedUnroll = 2;          // vectors per thread per iteration of the d alpha loop
constexpr int64_t kRedElemsPerBlock = 8192;
constexpr size_t kWsHeader = 256;      // ticket counter lives in the first 256 bytes

// Reduction grid of the d alpha backward: a function of n only, so the sum
// order (and hence the bits of the result) never depends on the device.
// With u = ceil(n / kRedElemsPerBlock) work units and k = ceil(u /
// kRedGridMax) units per block, the grid is ceil(u / k): every block gets k
// units (the last ones possibly one fewer), so no block is left with a
// partly empty last pass.
inline int red_grid(int64_t n)
{
    int64_t u = (n + kRedElemsPerBlock - 1) / kRedElemsPerBlock;
    if (u < 1) u = 1;
    const int64_t k = (u + kRedGridMax - 1) / kRedGridMax;
    return (int)((u + k - 1) / k);
}

struct ActLaunch {
    int act;                 // mea_act_t
    int dtype;               // Dtype
    const void *x;
    const void *dy;          // backward only
    void *out;               // y or dx
    int64_t n;
    float param;
    const float *param_dev;  // nullable
    float *dparam;           // nullable (Swish d alpha)
    void *workspace;         // ticket + fp64 partials when dparam is set
    cudaStream_t stream;
};

// Returns a cudaError_t from the launch (cudaSuccess on success).
cudaError_t launch_act_fwd(const ActLaunch &a);
cudaError_t launch_act_bwd(const ActLaunch &a);

// One tensor of a grouped launch (act_group_kernel).
struct ActSeg {
    const void *x;
    const void *dy;          // backward only
    void *out;               // y or dx
    int64_t n;
    const float *param_dev;  // nullable
    float *dparam;           // nullable (Swish d alpha: every segment or none)
    void *ws;                // this segment's ticket + fp64 partials (d alpha)
    float param;
    int vec_ok;              // set by the launcher
};
constexpr int kMaxSegs = 32;  // segments per launch (the table is passed as a kernel parameter)
struct ActSegTable {
    ActSeg seg[kMaxSegs];
    int start[kMaxSegs + 1];  // first block of each segment; start[nseg] is the grid
    int nseg;
};
struct ActGroupLaunch {
    int act;
    int dtype;
    int nseg;                 // any count: launched kMaxSegs at a time
    const ActSeg *segs;
    cudaStream_t stream;
};
cudaError_t launch_act_fwd_grouped(const ActGroupLaunch &a);
cudaError_t launch_act_bwd_grouped(const ActGroupLaunch &a);

// Launch with programmatic stream serialisation: the kernel may begin while
// the previous kernel on the stream drains, and waits (pdl_wait) before it
// touches memory.  Returns the launch's cudaError_t.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Number of SMs of the current device (cached per device).
int sm_count();

// Resident blocks per SM of one kernel instantiation at `threads` threads
// per block.  The Tag type gives every instantiation its own cache (kernels
// of one template share a function-pointer type).  Every GPU this library
// targets is a B200, so the value does not vary between devices.
template <class Tag, typename K>
int resident_blocks(K kernel, int threads)
{
    static int blocks = 0;
    if (blocks == 0) {
        int b = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kernel, threads, 0) != cudaSuccess || b <= 0)
            b = 1;
        blocks = b;
    }
    return blocks;
}

}  // namespace mea
