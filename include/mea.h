/*
 * mea.h -- C ABI of the memory-efficient activation library (libmea.so).
 *
 * The library implements save-input-only elementwise activations on NVIDIA
 * B200 (sm_100a): the forward writes y = f(x) and keeps nothing else; the
 * backward recomputes what it needs from the saved input x in the same pass
 * and writes dx = dy * f'(x) (plus d alpha for a learnable Swish alpha,
 * scalar or one per channel, or d gamma / d beta for the fused per-channel
 * affine + activation).  The same recompute principle is applied beside two
 * neighbouring operations: a matrix multiply with the activation in its
 * epilogue (mea_matmul_act_*: only the product Z is kept, f'(Z) is applied
 * inside the backward matmul) and DenseNet's concatenation + batch
 * normalization + ReLU (mea_concat_bn_relu_*: the concatenation is never
 * formed, only the batch statistics are kept, the output is re-populated).
 *
 * Entry points: mea_act_fwd / mea_act_bwd (+ _workspace_bytes,
 * mea_act_bwd_dparam_noalloc); mea_act_fwd_grouped / mea_act_bwd_grouped
 * (+ _workspace_bytes: many independent tensors in one launch);
 * mea_affine_swish_* and mea_affine_act_*;
 * mea_swish_channel_*; mea_matmul_act_fwd / _bwd; mea_concat_bn_relu_fwd /
 * _apply / _bwd (+ _workspace_bytes); mea_status_string, mea_last_error,
 * mea_version.
 *
 * Sources, by page and section:
 *  - "Memory efficient Swish" (adeeplearner blog, 2021-05-17):
 *      "What is a Swish activation function?" / "How is Swish implemented?"
 *        Swish(x) = x * Sigmoid(alpha x), Sigmoid(v) = 1 / (1 + e^-v);
 *      "How is the memory efficient version Swish implemented?" and
 *      "What makes this implementation save GPU memory?"
 *        the forward saves only the input; the backward recomputes the
 *        sigmoid from it: dx = dy * s * (1 + x (1 - s)) at alpha = 1.
 *  - "What activations cost, in memory and in arithmetic" (asifuddin.com,
 *    problem B07), GIVEN: the family ReLU, LeakyReLU, sigmoid, tanh, GELU
 *    (erf) and GELU (tanh approximation); SOLUTION: elementwise work is bound
 *    by memory bandwidth (about c/4 FLOP per byte in bf16).
 *
 * Conventions shared by every entry point:
 *  - Pointers named x, dy, y, dx, gamma, beta, dgamma, dbeta, param_dev,
 *    dparam_dev and workspace are DEVICE pointers (memory the GPU can load
 *    and store, e.g. from cudaMalloc or a PyTorch CUDA tensor).  The shape
 *    array is a HOST pointer.  The caller owns every buffer; the library
 *    allocates nothing and keeps no pointer after the call returns.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream).  Argument validation is synchronous; a launch
 *    failure is reported as MEA_ERR_CUDA (from cudaGetLastError).  No kernel
 *    traps or asserts; no call synchronises the device.
 *  - Storage dtypes: MEA_F32 (IEEE binary32) and MEA_BF16 (bfloat16).  All
 *    arithmetic is fp32 on the widened values; bf16 results are rounded to
 *    nearest even.  Reductions accumulate in fp64 and return fp32.
 *  - Layout: tensors are dense and contiguous.  Pointers that are not
 *    16-byte aligned, and element counts that are not a multiple of the
 *    vector width, take a scalar path; that is never an error.
 *  - n = 0 (or a zero in shape) is a no-op that returns MEA_OK.
 *  - Results are bitwise deterministic for a given input, shape, dtype and
 *    pointer alignment class (16-byte aligned or not: it selects the kernel
 *    path): reductions run on a grid fixed by the shape and sum in a fixed
 *    order, independent of the stream, the run and the GPU's SM count.
 *  - Workspaces: the first 4 bytes are a completion counter (see
 *    mea_act_bwd); bytes 4..7 are an error word that the per-channel
 *    backward sets non-zero if one of its bounded waits on shared-memory
 *    barriers expires (which does not happen in correct operation); results
 *    are then undefined.  The matmul kernels, which take no workspace, record
 *    the same condition in a device word of the library.
 */
#ifndef MEA_H
#define MEA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MEA_API __attribute__((visibility("default")))
#else
#define MEA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (the runtime's and the driver's stream handle type). */
typedef struct CUstream_st *mea_stream_t;

/* Activation functions.  Definitions (problem B07 names them; the
 * definitions are the standard ones; Swish is from the Swish page):
 *   MEA_RELU        max(x, 0);            derivative: 1 if x > 0 else 0
 *   MEA_LEAKY_RELU  x > 0 ? x : slope x;  derivative: 1 if x > 0 else slope
 *   MEA_SIGMOID     1 / (1 + e^-x);       derivative: s (1 - s)
 *   MEA_TANH        tanh x;               derivative: 1 - tanh^2 x
 *   MEA_GELU_ERF    x Phi(x), Phi the standard normal CDF;
 *                   derivative: Phi(x) + x phi(x)
 *   MEA_GELU_TANH   x (1 + tanh u) / 2, u = sqrt(2/pi) (x + 0.044715 x^3)
 *   MEA_SWISH       x Sigmoid(alpha x);   derivative: s + alpha x s (1 - s),
 *                   s = Sigmoid(alpha x); d alpha = sum dy x^2 s (1 - s)   */
typedef enum {
    MEA_RELU = 0,
    MEA_LEAKY_RELU = 1,
    MEA_SIGMOID = 2,
    MEA_TANH = 3,
    MEA_GELU_ERF = 4,
    MEA_GELU_TANH = 5,
    MEA_SWISH = 6
} mea_act_t;

typedef enum { MEA_F32 = 0, MEA_BF16 = 1 } mea_dtype_t;

/* Memory order of a 4-D activation whose logical shape is {N, C, H, W}. */
typedef enum { MEA_NCHW = 0, MEA_NHWC = 1 } mea_layout_t;

typedef enum {
    MEA_OK = 0,
    MEA_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad enum, overlap */
    MEA_ERR_UNSUPPORTED = 2,   /* valid request this build does not serve */
    MEA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required */
    MEA_ERR_CUDA = 4           /* a CUDA runtime call or launch failed */
} mea_status_t;

/* Forward: y[i] = f(x[i]) for i < n.
 *   act, dtype   activation and storage dtype of x and y.
 *   x            device, n elements, read only.  This is the one tensor the
 *                caller keeps for the backward.
 *   y            device, n elements, written.  Must not overlap x (x is the
 *                saved tensor): any overlap returns MEA_ERR_INVALID_ARG.
 *   n            element count, >= 0.
 *   param        alpha for MEA_SWISH, slope for MEA_LEAKY_RELU, ignored
 *                otherwise.
 *   param_dev    optional device pointer to one float; when non-NULL it is
 *                read on the device and replaces `param` (a learnable alpha
 *                that lives on the GPU).
 *   stream       CUDA stream the kernel is queued on.
 * Source: the Swish page's forward (section "How is the memory efficient
 * version Swish implemented?"), generalised to the family of problem B07. */
MEA_API mea_status_t mea_act_fwd(mea_act_t act, mea_dtype_t dtype, const void *x, void *y,
                         int64_t n, float param, const float *param_dev,
                         mea_stream_t stream);

/* Bytes of device workspace mea_act_bwd needs: 0 unless want_dparam is
 * non-zero (d alpha of MEA_SWISH), in which case it is a small function of n
 * (at most 256 + 8 * 444 = 3,808 bytes).  Pure host arithmetic; no CUDA call. */
MEA_API size_t mea_act_bwd_workspace_bytes(mea_act_t act, int64_t n, int want_dparam);

/* Backward with recompute: dx[i] = dy[i] * f'(x[i]) for i < n, f' evaluated
 * from x alone (nothing but x was saved).
 *   x, dy        device, n elements each, read only.
 *   dx           device, n elements, written.  May be the same pointer as
 *                dy or as x (each element is read before it is written); a
 *                partial overlap returns MEA_ERR_INVALID_ARG.
 *   param,
 *   param_dev    as in mea_act_fwd.
 *   dparam_dev   optional device pointer to one float.  When non-NULL (only
 *                for MEA_SWISH, else MEA_ERR_UNSUPPORTED) it is OVERWRITTEN
 *                with d alpha = sum_i dy_i x_i^2 s_i (1 - s_i), fp64
 *                accumulation in a fixed order, rounded to fp32.
 *   workspace,
 *   ws_bytes     device scratch of at least mea_act_bwd_workspace_bytes()
 *                bytes, 16-byte aligned, when dparam_dev is non-NULL (else
 *                ignored).  Its first 4 bytes are a completion counter that
 *                must be zero before the first use (zero-fill the buffer
 *                once); every call returns the counter to zero when its
 *                kernel completes, so the buffer can be reused without
 *                clearing.  Calls that share a workspace must not run
 *                concurrently on the GPU.
 * Source: the Swish page, sections "How is the memory efficient version
 * Swish implemented?" and "What makes this implementation save GPU memory?";
 * d alpha is the derivative of sum(dy * Swish) in alpha. */
MEA_API mea_status_t mea_act_bwd(mea_act_t act, mea_dtype_t dtype, const void *x, const void *dy,
                         void *dx, int64_t n, float param, const float *param_dev,
                         float *dparam_dev, void *workspace, size_t ws_bytes,
                         mea_stream_t stream);

/* One tensor of a grouped call (mea_act_fwd_grouped / mea_act_bwd_grouped). */
typedef struct {
    const void *x;            /* device, n elements, read only (the saved tensor) */
    const void *dy;           /* backward: device, n elements; ignored by the forward */
    void *out;                /* device, n elements: y (forward) or dx (backward) */
    int64_t n;                /* element count, >= 0 */
    float param;              /* as in mea_act_fwd */
    const float *param_dev;   /* as in mea_act_fwd (nullable) */
    float *dparam_dev;        /* backward, MEA_SWISH: as in mea_act_bwd; set in every
                                 segment or in none; ignored by the forward */
} mea_act_segment_t;

/* Forward over several independent tensors in one launch: for every segment
 * s, out_s = f(x_s), with one activation and dtype for all.  Each segment's
 * result is bitwise the result of mea_act_fwd on that segment alone.  One
 * grid instead of nseg launches removes each small tensor's ramp-up, drain
 * and launch gap (the small feature maps of a network's branches or of
 * several micro-batches).
 *   segs         host array of nseg (>= 0) segments; read during the call only.
 *                Segments are launched up to 32 per kernel.
 *   Every segment is validated as mea_act_fwd validates its tensors, and no
 *   segment's output may overlap any other segment's input or output
 *   (MEA_ERR_INVALID_ARG, nothing launched).
 * Source: as mea_act_fwd; one launch for many tensors is this library's
 * (the pages call the activation once per layer). */
MEA_API mea_status_t mea_act_fwd_grouped(mea_act_t act, mea_dtype_t dtype, int nseg,
                                         const mea_act_segment_t *segs, mea_stream_t stream);

/* Bytes of device workspace mea_act_bwd_grouped needs for these segments:
 * 0 unless their dparam_dev are set; else the sum over segments of
 * mea_act_bwd_workspace_bytes rounded up to 256 bytes.  Pure host
 * arithmetic. */
MEA_API size_t mea_act_bwd_grouped_workspace_bytes(mea_act_t act, int nseg, const mea_act_segment_t *segs);

/* Backward over several independent tensors in one launch: for every
 * segment, dx_s = dy_s * f'(x_s), and with dparam_dev set (MEA_SWISH, every
 * segment) d alpha_s, each bitwise what mea_act_bwd gives for that segment
 * alone (same reduction grid and summation order).
 *   segs         as in mea_act_fwd_grouped; dx may alias that segment's dy
 *                or x exactly, no other overlap with any segment.
 *   workspace,
 *   ws_bytes     when d alpha is asked for: device scratch of at least
 *                mea_act_bwd_grouped_workspace_bytes(), 256-byte aligned,
 *                any contents (every call writes the partial sums it reads:
 *                no counter, no zero-fill).  The d alpha sums are formed by
 *                a second, small kernel (one block per segment) queued on
 *                the same stream.  Calls sharing a workspace must not run
 *                concurrently on the GPU.
 * Source: as mea_act_bwd. */
MEA_API mea_status_t mea_act_bwd_grouped(mea_act_t act, mea_dtype_t dtype, int nseg,
                                         const mea_act_segment_t *segs, void *workspace, size_t ws_bytes,
                                         mea_stream_t stream);

/* Bytes of device workspace mea_affine_swish_bwd needs for this dtype,
 * layout and logical shape {N, C, H, W} (host pointer).  Pure host
 * arithmetic; returns 0 for an invalid request. */
MEA_API size_t mea_affine_swish_bwd_workspace_bytes(mea_dtype_t dtype, mea_layout_t layout,
                                            const int64_t shape[4]);

/* Fused per-channel affine + Swish forward: z = gamma_c x + beta_c,
 * y = z Sigmoid(z).
 *   shape        host array {N, C, H, W} (logical dims, all >= 0).
 *   layout       MEA_NHWC: channel of flat index i is i mod C;
 *                MEA_NCHW: channel is (i / (H W)) mod C.
 *   x, y         device, N*C*H*W elements of `dtype`; y must not overlap x.
 *   gamma, beta  device fp32[C], read only.
 * Source: the save-input-only Swish of the Swish page applied after a
 * per-channel affine (the op that precedes Swish in EfficientNet blocks). */
MEA_API mea_status_t mea_affine_swish_fwd(mea_dtype_t dtype, mea_layout_t layout,
                                  const int64_t shape[4], const void *x,
                                  const float *gamma, const float *beta, void *y,
                                  mea_stream_t stream);

/* Fused per-channel affine + Swish backward: recomputes z from x and
 *   dz = dy (s + z s (1 - s)), s = Sigmoid(z);
 *   dx = gamma_c dz;  dgamma_c = sum dz x;  dbeta_c = sum dz
 * (sums over all N*H*W positions of channel c, fp64 accumulation in a fixed
 * order, rounded to fp32).
 *   x, dy        device, read only; dx device, written (may equal dy or x
 *                exactly, no partial overlap).
 *   gamma, beta  device fp32[C], read only.
 *   dgamma,
 *   dbeta        device fp32[C], OVERWRITTEN (not accumulated).
 *   workspace    device scratch of at least
 *                mea_affine_swish_bwd_workspace_bytes() bytes, 16-byte
 *                aligned, with the same completion-counter rule as the
 *                workspace of mea_act_bwd (zero-fill once; each call leaves
 *                the counter at zero; no concurrent sharing). */
MEA_API mea_status_t mea_affine_swish_bwd(mea_dtype_t dtype, mea_layout_t layout,
                                  const int64_t shape[4], const void *x, const void *dy,
                                  const float *gamma, const float *beta, void *dx,
                                  float *dgamma, float *dbeta, void *workspace,
                                  size_t ws_bytes, mea_stream_t stream);

/* Bytes of device workspace mea_affine_act_bwd needs (the same for every
 * activation; equal to mea_affine_swish_bwd_workspace_bytes).  Pure host
 * arithmetic; returns 0 for an invalid request. */
MEA_API size_t mea_affine_act_bwd_workspace_bytes(mea_dtype_t dtype, mea_layout_t layout,
                                                  const int64_t shape[4]);

/* Fused per-channel affine + any activation of the family, forward:
 * z = gamma_c x + beta_c, y = f(z), f as in mea_act_t with `param` (slope
 * of MEA_LEAKY_RELU, alpha of MEA_SWISH; ignored otherwise).
 *   Arguments otherwise as in mea_affine_swish_fwd; mea_affine_swish_fwd is
 *   this call with act = MEA_SWISH and param = 1.
 * Source: the save-input-only scheme of the Swish page ("What makes this
 * implementation save GPU memory?") applied to the per-channel affine that
 * precedes the activation, for the family of problem B07. */
MEA_API mea_status_t mea_affine_act_fwd(mea_act_t act, mea_dtype_t dtype, mea_layout_t layout,
                                        const int64_t shape[4], const void *x, const float *gamma,
                                        const float *beta, float param, void *y,
                                        mea_stream_t stream);

/* Fused per-channel affine + activation, backward: recomputes z from x and
 *   dz = dy f'(z);  dx = gamma_c dz;  dgamma_c = sum dz x;  dbeta_c = sum dz
 * (sums over all N*H*W positions of channel c, fp64 accumulation in a fixed
 * order, rounded to fp32; dgamma and dbeta are OVERWRITTEN).
 *   Arguments otherwise as in mea_affine_swish_bwd (workspace of at least
 *   mea_affine_act_bwd_workspace_bytes() bytes, same counter rule). */
MEA_API mea_status_t mea_affine_act_bwd(mea_act_t act, mea_dtype_t dtype, mea_layout_t layout,
                                        const int64_t shape[4], const void *x, const void *dy,
                                        const float *gamma, const float *beta, float param,
                                        void *dx, float *dgamma, float *dbeta, void *workspace,
                                        size_t ws_bytes, mea_stream_t stream);

/* Bytes of device workspace mea_swish_channel_bwd needs.  Pure host
 * arithmetic; returns 0 for an invalid request. */
MEA_API size_t mea_swish_channel_bwd_workspace_bytes(mea_dtype_t dtype, mea_layout_t layout,
                                                     const int64_t shape[4]);

/* Swish with one learnable alpha per channel, forward:
 * y = x Sigmoid(alpha_c x).
 *   shape, layout  as in mea_affine_swish_fwd (channel of each element).
 *   x, y           device, N*C*H*W elements of `dtype`; y must not overlap x.
 *   alpha          device fp32[C], read only.
 * Source: the Swish page's learnable alpha ("What is a Swish activation
 * function?"), one value per channel. */
MEA_API mea_status_t mea_swish_channel_fwd(mea_dtype_t dtype, mea_layout_t layout,
                                           const int64_t shape[4], const void *x,
                                           const float *alpha, void *y, mea_stream_t stream);

/* Swish with a per-channel alpha, backward (recompute from x alone):
 *   s = Sigmoid(alpha_c x);  dx = dy (s + alpha_c x s (1 - s));
 *   dalpha_c = sum dy x^2 s (1 - s)   (over the N*H*W positions of channel
 *   c, fp64 accumulation in a fixed order, rounded to fp32, OVERWRITTEN).
 *   x, dy     device, read only; dx device, written (may equal dy or x
 *             exactly, no partial overlap).
 *   alpha     device fp32[C]; dalpha device fp32[C].
 *   workspace device scratch of at least mea_swish_channel_bwd_workspace_bytes()
 *             bytes, 16-byte aligned, with the completion-counter rule of
 *             mea_act_bwd. */
MEA_API mea_status_t mea_swish_channel_bwd(mea_dtype_t dtype, mea_layout_t layout,
                                           const int64_t shape[4], const void *x, const void *dy,
                                           const float *alpha, void *dx, float *dalpha,
                                           void *workspace, size_t ws_bytes, mea_stream_t stream);

/* One NCHW tensor of a grouped per-channel Swish call
 * (mea_swish_channel_fwd_grouped / mea_swish_channel_bwd_grouped). */
typedef struct {
    const void *x;            /* device, [N, C, H, W] NCHW, read only (the saved tensor) */
    const void *dy;           /* backward: device, same shape; ignored by the forward */
    void *out;                /* device, same shape: y (forward) or dx (backward) */
    const float *alpha;       /* device fp32[C], read only */
    float *dalpha;            /* backward: device fp32[C], OVERWRITTEN; ignored by the forward */
    int64_t shape[4];         /* N, C, H, W (each >= 0) */
} mea_channel_segment_t;

/* Forward of Swish with a per-channel alpha over several independent NCHW
 * tensors: for every segment s, out_s = x_s Sigmoid(alpha_s,c x_s), each
 * bitwise what mea_swish_channel_fwd (MEA_NCHW) gives on that segment alone.
 * Segments whose planes take the library's row path (H W <= 1024 elements,
 * 16-byte aligned tensors: EfficientNet's 28 x 28 to 1 x 1 stages) run in
 * one grid, up to 32 per kernel; any other segment is launched alone.
 *   segs         host array of nseg (>= 0) segments; read during the call only.
 *   Every segment is validated as mea_swish_channel_fwd validates its
 *   tensors, and no segment's output may overlap any other segment's input
 *   or output (MEA_ERR_INVALID_ARG, nothing launched).
 * Source: as mea_swish_channel_fwd; one launch for many layers' tensors is
 * this library's (the pages call the activation once per layer). */
MEA_API mea_status_t mea_swish_channel_fwd_grouped(mea_dtype_t dtype, int nseg,
                                                   const mea_channel_segment_t *segs, mea_stream_t stream);

/* Bytes of device workspace mea_swish_channel_bwd_grouped needs: the sum over
 * segments of mea_swish_channel_bwd_workspace_bytes (MEA_NCHW) rounded up to
 * 256 bytes.  Pure host arithmetic; 0 for an invalid request. */
MEA_API size_t mea_swish_channel_bwd_grouped_workspace_bytes(mea_dtype_t dtype, int nseg,
                                                             const mea_channel_segment_t *segs);

/* Backward of Swish with a per-channel alpha over several independent NCHW
 * tensors: dx_s and dalpha_s for every segment, each bitwise what
 * mea_swish_channel_bwd (MEA_NCHW) gives on that segment alone (same blocks,
 * same summation order).  The row-path segments run in one grid and their
 * dalpha sums in a second, small kernel on the same stream.
 *   segs         as in mea_swish_channel_fwd_grouped; dx may alias that
 *                segment's dy or x exactly, no other overlap with any
 *                segment; dalpha of different segments must not overlap.
 *                A segment with C > 0 and no elements gets dalpha = 0.
 *   workspace,
 *   ws_bytes     device scratch of at least
 *                mea_swish_channel_bwd_grouped_workspace_bytes(), 256-byte
 *                aligned, any contents (the call clears what it needs).
 *                Calls sharing a workspace must not run concurrently on the
 *                GPU.
 * Source: as mea_swish_channel_bwd. */
MEA_API mea_status_t mea_swish_channel_bwd_grouped(mea_dtype_t dtype, int nseg,
                                                   const mea_channel_segment_t *segs, void *workspace,
                                                   size_t ws_bytes, mea_stream_t stream);

/* Matrix multiply with the activation fused into its epilogue, forward:
 *   Z = X W^T  (bf16 inputs, fp32 accumulation on the tensor cores),
 *   z = Z rounded to bf16 (written when z is non-NULL),
 *   y = f(Z as stored in bf16) (written when y is non-NULL).
 *   act, param  activation and its parameter, as in mea_act_fwd.
 *   M, N, K     X is [M x K], W is [N x K], Z, y are [M x N]; M or N of 0 is
 *               a no-op; K must be positive.  K and N must be multiples of 8
 *               (rows of 16-byte multiples), each below 2^31; otherwise
 *               MEA_ERR_UNSUPPORTED.
 *   x, w        device, bf16, row-major (K contiguous), read only, 16-byte
 *               aligned (else MEA_ERR_UNSUPPORTED).
 *   z, y        device, bf16, row-major [M x N], 16-byte aligned, written;
 *               at least one non-NULL; neither may overlap x, w or the other.
 * Only Z needs to be kept for the backward (the save-input-only scheme,
 * with the matmul output as the saved input); y feeds the next layer.
 * Source: problem B07 of "What activations cost, in memory and in
 * arithmetic", SOLUTION step 4 (the activation follows a d x d matrix
 * multiply on the same tensor; its arithmetic is free beside it, its memory
 * is not). */
MEA_API mea_status_t mea_matmul_act_fwd(mea_act_t act, int64_t M, int64_t N, int64_t K, const void *x,
                                        const void *w, float param, void *z, void *y, mea_stream_t stream);

/* Matrix multiply with the activation's derivative fused into its epilogue,
 * backward: dz = (G W^T) * f'(z), f' recomputed from the stored z.
 *   G           device bf16 [M x K] (the upstream gradient), read only.
 *   W           device bf16 [N x K]: for a following layer out = y W2^T
 *               with W2 [K x N], pass W = W2^T (N rows of K).
 *   z           device bf16 [M x N], the stored pre-activation, read only.
 *   dz          device bf16 [M x N], written; may be the same pointer as z
 *               (each element is read before it is written), no partial
 *               overlap with z, and no overlap with G or W.
 *   Other arguments and restrictions as in mea_matmul_act_fwd.
 * The product G W^T never reaches memory. */
MEA_API mea_status_t mea_matmul_act_bwd(mea_act_t act, int64_t M, int64_t N, int64_t K, const void *g,
                                        const void *w, const void *z, float param, void *dz,
                                        mea_stream_t stream);

/* Concatenation + batch normalization + ReLU without the concatenated
 * tensor (DenseNet's memory-efficient layer): the input is the channel
 * concatenation of `npieces` NCHW pieces, never formed in memory.
 *   pieces        HOST array of npieces DEVICE pointers; piece i is a dense
 *                 [N, channels[i], HW] tensor of `dtype`, 16-byte aligned for
 *                 the vector path (any alignment is served).
 *   channels      HOST array of npieces channel counts (each >= 1); C = their
 *                 sum (below 2^31); 1 <= npieces <= 128.
 *   N, HW         batch and plane size (H W); N HW >= 1.
 *   gamma, beta   device fp32 [C].
 *   mean, invstd  device fp32 [C], written: the batch mean and
 *                 1 / sqrt(var + eps), var the biased batch variance.  These
 *                 2 C floats are all the backward needs besides the pieces.
 *   running_mean,
 *   running_var   device fp32 [C] or both NULL: moved by `momentum` towards
 *                 the batch mean and the unbiased batch variance.
 *   y             device [N, C, HW] of `dtype`, written: max(gamma xhat +
 *                 beta, 0).  Meant to be a buffer shared by every layer: the
 *                 backward re-populates it (mea_concat_bn_relu_apply).  Must
 *                 not overlap a piece.
 *   workspace     device scratch of mea_concat_bn_relu_workspace_bytes(N, C)
 *                 bytes, 16-byte aligned (no counter: no zero-fill needed;
 *                 calls that share it must not run concurrently).
 * Source: "A memory-efficient implementation of DenseNets", section
 * "Motivation" (shared allocations for every concatenation and batch
 * normalization output, re-populated in the backward); batch normalization
 * in its standard training-mode definition. */
MEA_API size_t mea_concat_bn_relu_workspace_bytes(int64_t N, int64_t C);

MEA_API mea_status_t mea_concat_bn_relu_fwd(mea_dtype_t dtype, int npieces, const void *const *pieces,
                                            const int64_t *channels, int64_t N, int64_t HW,
                                            const float *gamma, const float *beta, float eps,
                                            float momentum, float *running_mean, float *running_var,
                                            float *mean, float *invstd, void *y, void *workspace,
                                            size_t ws_bytes, mea_stream_t stream);

/* Re-populates y = max(gamma (x - mean) invstd + beta, 0) from the pieces
 * and saved statistics (no reduction): the backward's recompute of the
 * forward output, bitwise equal to what mea_concat_bn_relu_fwd wrote.
 * Arguments as in mea_concat_bn_relu_fwd. */
MEA_API mea_status_t mea_concat_bn_relu_apply(mea_dtype_t dtype, int npieces, const void *const *pieces,
                                              const int64_t *channels, int64_t N, int64_t HW,
                                              const float *gamma, const float *beta,
                                              const float *mean, const float *invstd, void *y,
                                              mea_stream_t stream);

/* Backward from the pieces, dy and the saved statistics (the ReLU mask and
 * xhat are recomputed):
 *   dz = dy [gamma' x + beta' > 0] (the forward's own test);
 *   dbeta = sum dz, dgamma = sum dz xhat (fp64 sums in a fixed order,
 *   OVERWRITTEN, fp32); dx = gamma invstd (dz - dbeta / n - xhat dgamma / n).
 *   dy            device [N, C, HW] of `dtype`, read only.
 *   dpieces       HOST array of npieces DEVICE pointers, the gradients of the
 *                 pieces (same shapes); overwritten, or added to when
 *                 `accumulate` is non-zero (a piece feeds several layers).
 *                 dpieces[i] may be pieces[i] itself (no partial overlap).
 *   workspace     as in mea_concat_bn_relu_fwd. */
MEA_API mea_status_t mea_concat_bn_relu_bwd(mea_dtype_t dtype, int npieces, const void *const *pieces,
                                            const int64_t *channels, int64_t N, int64_t HW,
                                            const void *dy, const float *gamma, const float *beta,
                                            const float *mean, const float *invstd,
                                            void *const *dpieces, int accumulate, float *dgamma,
                                            float *dbeta, void *workspace, size_t ws_bytes,
                                            mea_stream_t stream);

/* Backward with d alpha that allocates nothing and takes no workspace.
 * No counterpart on the pages: this is a library convenience, not part of
 * the method.  It computes exactly what mea_act_bwd computes (same kernel,
 * same fixed reduction order, bitwise the same dx and d alpha) for callers
 * that cannot allocate device memory for the reduction scratch -- code whose
 * device memory is handed out entirely by another allocator (a framework's
 * caching allocator or a fixed memory plan), and latency-sensitive paths
 * that cannot accept the synchronisation cudaFree (and possibly cudaMalloc)
 * brings.  The scratch is a fixed 3,808-byte array in the library's device
 * code, present on every GPU that loads the library until the process exits.
 *   Arguments as for mea_act_bwd, without workspace / ws_bytes.  With
 *   dparam_dev NULL it is a plain backward (no scratch is used).
 *   Every element count is served (the reduction grid is capped so that its
 *   scratch fits the array); a request needing more scratch than the array
 *   holds would be refused with MEA_ERR_WORKSPACE.
 *   Every call looks up the array's device address on the current device
 *   with cudaGetSymbolAddress (so the address stays right after a device
 *   reset); the first call on a device may load the library's device code,
 *   so make it before any stream capture.  Every call clears the array's
 *   completion counter with cudaMemsetAsync on `stream` and then launches
 *   the kernel; it calls no cudaMalloc, cudaFree or other allocating
 *   routine.
 *   All calls on a device share the one array: calls whose kernels may run
 *   at the same time on the GPU (unordered streams) race and must not be
 *   issued; calls ordered on one stream are safe. */
MEA_API mea_status_t mea_act_bwd_dparam_noalloc(mea_act_t act, mea_dtype_t dtype, const void *x,
                                                const void *dy, void *dx, int64_t n, float param,
                                                const float *param_dev, float *dparam_dev,
                                                mea_stream_t stream);

/* Self-test of the bounded waits (failure detection without a GPU fault).
 * No counterpart on the pages.  Runs the pipelined NHWC backward of the
 * fused affine + Swish on the caller's tensors (arguments as for
 * mea_affine_swish_bwd with layout MEA_NHWC; dx, dgamma, dbeta are not
 * written) with the shared-memory copies of its producer withheld, so that
 * no stage barrier ever completes.  Every wait then gives up after a few
 * milliseconds, records the workspace's error word and lets its warp
 * finish, exactly the path a wait takes if a copy never lands.  The call
 * synchronises `stream`, stores the error word in *expired (1: the waits
 * expired and the kernel returned; the context stays usable) and clears the
 * word.  MEA_ERR_UNSUPPORTED when the shape or alignment does not take the
 * pipelined path (C a multiple of 4, x and dy 16-byte aligned, enough
 * tiles). */
MEA_API mea_status_t mea_affine_bwd_wait_selftest(mea_dtype_t dtype, const int64_t shape[4], const void *x,
                                                  const void *dy, const float *gamma, const float *beta, void *dx,
                                                  void *workspace, size_t ws_bytes, int *expired,
                                                  mea_stream_t stream);

/* Reads (and with clear non-zero, resets) the matmul kernels' device error
 * word on the current device: non-zero if a bounded barrier wait in a
 * mea_matmul_act_* kernel expired since the last clear (which does not
 * happen in correct operation).  Synchronises the current device.  Returns
 * -1 if the word cannot be read (a CUDA error; see mea_last_error). */
MEA_API int mea_matmul_error_word(int clear);

/* Static description of a status code. */
MEA_API const char *mea_status_string(mea_status_t status);

/* Detail of the most recent failing call on this host thread (which
 * argument, which CUDA error); "" if none.  Valid until the next call. */
MEA_API const char *mea_last_error(void);

/* Library version: major * 10000 + minor * 100 + patch. */
MEA_API int mea_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MEA_H */
