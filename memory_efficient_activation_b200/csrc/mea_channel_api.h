// mea_channel_api.h -- host-side interface of the per-channel kernels (fused
// per-channel affine + activation; Swish with one alpha per channel).
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace mea {

// Per-channel operations (affine + activation; Swish with per-channel alpha).
// For the channel Swish, gamma carries alpha and dgamma receives dalpha.
struct AffineLaunch {
    int act;                 // mea_act_t (affine + activation)
    float param;             // activation parameter (affine + activation)
    int dtype;
    int layout;              // mea_layout_t
    int64_t N, C, H, W;
    const void *x;
    const void *dy;
    const float *gamma;
    const float *beta;
    void *out;
    float *dgamma;
    float *dbeta;
    void *workspace;
    cudaStream_t stream;
};

size_t affine_bwd_workspace_bytes(int dtype, int layout, int64_t N, int64_t C, int64_t H, int64_t W);
cudaError_t launch_affine_fwd(const AffineLaunch &a);
cudaError_t launch_affine_bwd(const AffineLaunch &a);
// The bounded-wait self-test (affine + Swish, NHWC pipelined backward with its
// copies withheld); cudaErrorNotSupported off the pipelined path.
cudaError_t launch_affine_bwd_wait_selftest(const AffineLaunch &a);
size_t channel_swish_bwd_workspace_bytes(int dtype, int layout, int64_t N, int64_t C, int64_t H, int64_t W);
cudaError_t launch_channel_swish_fwd(const AffineLaunch &a);
cudaError_t launch_channel_swish_bwd(const AffineLaunch &a);

// One NCHW tensor of a grouped Swish launch with a per-channel alpha.
struct ChanSeg {
    const void *x;
    const void *dy;          // backward only
    void *out;               // y or dx
    const float *alpha;      // [C]
    float *dalpha;           // [C], backward only
    int64_t N, C, H, W;
    void *ws;                // backward: this segment's workspace (channel_swish_bwd_workspace_bytes)
};
// Segments whose planes take the row path run in one grid (up to 32 per
// launch, their d alpha sums in a second one); any other segment runs alone
// on its usual path (its workspace counter cleared first).
cudaError_t launch_channel_swish_fwd_grouped(int dtype, int nseg, const ChanSeg *segs, cudaStream_t stream);
cudaError_t launch_channel_swish_bwd_grouped(int dtype, int nseg, const ChanSeg *segs, cudaStream_t stream);

}  // namespace mea
