// mea_noalloc.cu -- the Swish backward with d alpha, with its reduction
// scratch taken from a fixed array in the library instead of a caller buffer.
//
// Who needs it: callers that cannot call cudaMalloc / cudaFree for the small
// reduction workspace.  Examples are code whose device memory is handed out
// entirely by another allocator (a framework's caching allocator or a fixed
// memory plan that must not be bypassed), and latency-sensitive paths that
// cannot accept the device-wide synchronisation cudaFree implies (and that
// cudaMalloc may imply).  This entry point allocates nothing: the scratch is
// a file-scope __device__ array of kNoAllocScratchBytes bytes, created when
// the library's device code is loaded on a GPU and held until the process
// exits.
//
// Host code cannot use the array's name as a device address (on the host it
// names a host-side stand-in), so every call looks the device address up with
// cudaGetSymbolAddress on the current device.  Looking it up per call rather
// than caching it keeps the address right after a device reset (which
// reloads the library's device code at a new address).  The first call on a
// device may load that code, so it should come before any stream capture.
// The array is shared by every call on a device and
// keeps whatever the last call left in it; the completion counter at its
// start is cleared (cudaMemsetAsync on the caller's stream) before every
// launch.  Calls whose kernels overlap on the GPU (different streams, no
// ordering between them) race on the array and must not be issued.
#include <cuda_runtime.h>

#include <nvtx3/nvToolsExt.h>

#include <cstdint>
#include <cstdio>

#include "../../include/mea.h"
#include "mea_internal.h"

// Header (completion counter) plus one fp64 partial per block of the
// largest reduction grid: enough for every element count (3,808 bytes).
static constexpr size_t kNoAllocScratchBytes = mea::kWsHeader + sizeof(double) * mea::kRedGridMax;

static __device__ __align__(256) unsigned char g_dalpha_scratch[kNoAllocScratchBytes];

namespace {

// Device address of the scratch on the current device.
cudaError_t scratch_for_current_device(void **out)
{
    void *p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_dalpha_scratch);
    if (e != cudaSuccess) return e;
    *out = p;
    return cudaSuccess;
}

}  // namespace

namespace mea {
// Records the detail string mea_last_error returns (defined with the rest of
// the C ABI in mea_capi.cu).
void set_last_error_detail(const char *detail);
}  // namespace mea

static mea_status_t noalloc_bwd(mea_act_t act, mea_dtype_t dtype, const void *x, const void *dy, void *dx,
                                int64_t n, float param, const float *param_dev, float *dparam_dev,
                                mea_stream_t stream);

extern "C" mea_status_t mea_act_bwd_dparam_noalloc(mea_act_t act, mea_dtype_t dtype, const void *x,
                                                   const void *dy, void *dx, int64_t n, float param,
                                                   const float *param_dev, float *dparam_dev,
                                                   mea_stream_t stream)
{
    nvtxRangePushA("mea_act_bwd_dparam_noalloc");
    const mea_status_t st = noalloc_bwd(act, dtype, x, dy, dx, n, param, param_dev, dparam_dev, stream);
    nvtxRangePop();
    return st;
}

static mea_status_t noalloc_bwd(mea_act_t act, mea_dtype_t dtype, const void *x, const void *dy, void *dx,
                                int64_t n, float param, const float *param_dev, float *dparam_dev,
                                mea_stream_t stream)
{
    // Without d alpha there is no reduction and no scratch: a plain backward.
    if (!dparam_dev)
        return mea_act_bwd(act, dtype, x, dy, dx, n, param, param_dev, nullptr, nullptr, 0, stream);
    void *scratch = nullptr;
    cudaError_t e = scratch_for_current_device(&scratch);
    if (e != cudaSuccess) {
        char msg[256];
        snprintf(msg, sizeof(msg), "looking up the fixed d alpha scratch: %s (%s)", cudaGetErrorName(e),
                 cudaGetErrorString(e));
        mea::set_last_error_detail(msg);
        return MEA_ERR_CUDA;
    }
    // A negative n, an activation without a parameter gradient, or a
    // reduction needing more scratch than the fixed array holds (not
    // reachable with the capped grid) is refused by the regular entry point,
    // which reports the scratch's real size, before anything is queued.  Any
    // other invalid argument is refused by it after the counter clear below,
    // which is harmless (it only touches the library's own array).
    if (n < 0 || act != MEA_SWISH || mea_act_bwd_workspace_bytes(act, n, 1) > kNoAllocScratchBytes)
        return mea_act_bwd(act, dtype, x, dy, dx, n, param, param_dev, dparam_dev, scratch,
                           kNoAllocScratchBytes, stream);
    // The completion counter must start at zero.
    e = cudaMemsetAsync(scratch, 0, mea::kWsHeader, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        char msg[256];
        snprintf(msg, sizeof(msg), "clearing the fixed d alpha scratch: %s (%s)", cudaGetErrorName(e),
                 cudaGetErrorString(e));
        mea::set_last_error_detail(msg);
        return MEA_ERR_CUDA;
    }
    return mea_act_bwd(act, dtype, x, dy, dx, n, param, param_dev, dparam_dev, scratch, kNoAllocScratchBytes,
                       stream);
}
