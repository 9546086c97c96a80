// mea_matmul_api.h -- host-side interface of the matmul + activation kernels
// (tcgen05 tensor cores, activation fused into the epilogue).
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace mea {

// Z = X W^T with X [M x K] and W [N x K] (row-major bf16, K contiguous).
//   mode 0 (forward):  out0 = Z (bf16, nullable), out1 = f(Z as stored)
//                      (bf16, nullable; at least one of the two).
//   mode 1 (backward): X is the upstream gradient G, zin the stored Z;
//                      out1 = (G W^T) f'(Z) (bf16).
struct MatmulLaunch {
    int act;
    int mode;
    int64_t M, N, K;
    const void *x;
    const void *w;
    const void *zin;
    void *out0;
    void *out1;
    float param;
    cudaStream_t stream;
};

cudaError_t launch_matmul_act(const MatmulLaunch &a);
cudaError_t matmul_error_word(int clear, unsigned int *word);   // synchronous

// Tile shape of the kernel (rows of X, rows of W, K per pipeline stage).
constexpr int kMatmulBM = 256;
constexpr int kMatmulBN = 256;
constexpr int kMatmulBK = 64;

}  // namespace mea
