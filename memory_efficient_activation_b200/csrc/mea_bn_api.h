// mea_bn_api.h -- host-side interface of the concatenation + batch
// normalization + ReLU kernels (DenseNet-style shared-buffer recompute).
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace mea {

// The channel-concatenation of up to kBnMaxPieces NCHW pieces.  Piece i is a
// dense [N, k_i, H, W] tensor; its channel j is channel off_i + j of the
// concatenation.  off[npieces] = C.
constexpr int kBnMaxPieces = 128;

struct BnPieces {
    const void *ptr[kBnMaxPieces];
    int off[kBnMaxPieces + 1];
    int npieces;
};

struct BnOutPieces {
    void *ptr[kBnMaxPieces];
};

struct BnLaunch {
    int dtype;
    int64_t N, C, HW;
    BnPieces in;
    const float *gamma;
    const float *beta;
    float eps;
    float momentum;
    float *running_mean;     // nullable (with running_var)
    float *running_var;
    float *mean;             // [C]: written by the forward, read by apply / backward
    float *invstd;           // [C]
    void *y;                 // [N, C, HW]: forward / apply output
    const void *dy;          // [N, C, HW]: backward input
    BnOutPieces din;         // backward outputs, one per piece
    int accumulate;          // backward: add into din instead of overwriting
    float *dgamma;
    float *dbeta;
    void *workspace;
    cudaStream_t stream;
};

size_t bn_workspace_bytes(int64_t N, int64_t C);
cudaError_t launch_bn_fwd(const BnLaunch &a);     // statistics, then y
cudaError_t launch_bn_apply(const BnLaunch &a);   // y from saved statistics
cudaError_t launch_bn_bwd(const BnLaunch &a);

}  // namespace mea
