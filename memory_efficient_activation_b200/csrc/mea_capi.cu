// mea_capi.cu -- the C ABI of include/mea.h: argument validation, error
// reporting and dispatch to the kernel launchers.  Host code only.
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <vector>

#include "../../include/mea.h"
#include "mea_bn_api.h"
#include "mea_channel_api.h"
#include "mea_internal.h"
#include "mea_matmul_api.h"

namespace {

thread_local char g_err[512];

// One NVTX range per C-ABI call, named for the entry point, so that a
// profiler's timeline shows which call issued which kernels.  With no tool
// attached the NVTX calls return at once.
struct Range {
    explicit Range(const char *name) { nvtxRangePushA(name); }
    ~Range() { nvtxRangePop(); }
    Range(const Range &) = delete;
    Range &operator=(const Range &) = delete;
};

void clear_error() { g_err[0] = '\0'; }

mea_status_t fail(mea_status_t st, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return st;
}

bool valid_act(int a) { return a >= MEA_RELU && a <= MEA_SWISH; }
bool valid_dtype(int d) { return d == MEA_F32 || d == MEA_BF16; }
size_t dtype_bytes(int d) { return d == MEA_BF16 ? 2 : 4; }

// Largest element count whose byte size and index arithmetic stay in range.
constexpr int64_t kMaxElems = (int64_t)1 << 60;

// [a, a + na) and [b, b + nb) share at least one byte.
bool overlaps(const void *a, size_t na, const void *b, size_t nb)
{
    const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
    return pa < pb + nb && pb < pa + na;
}

// Identical ranges are allowed (each element is read before it is written);
// any other overlap is not.
bool partial_overlap(const void *a, const void *b, size_t bytes)
{
    return a != b && overlaps(a, bytes, b, bytes);
}

mea_status_t cuda_fail(cudaError_t e, const char *what)
{
    return fail(MEA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

mea_status_t check_shape(const int64_t *shape, int64_t *n)
{
    if (!shape) return fail(MEA_ERR_INVALID_ARG, "shape is NULL");
    int64_t prod = 1;
    for (int i = 0; i < 4; ++i) {
        if (shape[i] < 0) return fail(MEA_ERR_INVALID_ARG, "shape[%d] = %lld is negative", i, (long long)shape[i]);
        if (shape[i] > 0 && prod > kMaxElems / shape[i])
            return fail(MEA_ERR_INVALID_ARG, "shape has more than 2^60 elements");
        prod *= shape[i];
    }
    *n = prod;
    return MEA_OK;
}

// Shared by the per-channel entry points.
size_t chan_ws_bytes(int kind, int dtype, int layout, const int64_t *shape)
{
    int64_t n = 0;
    if (!valid_dtype(dtype) || (layout != MEA_NCHW && layout != MEA_NHWC)) return 0;
    char saved[sizeof(g_err)];
    __builtin_memcpy(saved, g_err, sizeof(g_err));
    const bool ok = check_shape(shape, &n) == MEA_OK;
    __builtin_memcpy(g_err, saved, sizeof(g_err));
    if (!ok) return 0;
    return kind == 0 ? mea::affine_bwd_workspace_bytes(dtype, layout, shape[0], shape[1], shape[2], shape[3])
                     : mea::channel_swish_bwd_workspace_bytes(dtype, layout, shape[0], shape[1], shape[2], shape[3]);
}

// kind 0: affine + activation (p0 = gamma, p1 = beta); kind 1: Swish with a
// per-channel alpha (p0 = alpha).
mea_status_t chan_fwd(int kind, const char *name, int act, int dtype, int layout, const int64_t *shape,
                      const void *x, const float *p0, const float *p1, float param, void *y, mea_stream_t stream)
{
    clear_error();
    if (kind == 0 && !valid_act(act)) return fail(MEA_ERR_INVALID_ARG, "act = %d is not a mea_act_t", act);
    if (!valid_dtype(dtype)) return fail(MEA_ERR_INVALID_ARG, "dtype = %d is not a mea_dtype_t", dtype);
    if (layout != MEA_NCHW && layout != MEA_NHWC)
        return fail(MEA_ERR_INVALID_ARG, "layout = %d is not a mea_layout_t", layout);
    int64_t n = 0;
    mea_status_t st = check_shape(shape, &n);
    if (st != MEA_OK) return st;
    if (n == 0) return MEA_OK;
    if (!x || !y || !p0 || (kind == 0 && !p1))
        return fail(MEA_ERR_INVALID_ARG, kind == 0 ? "x, y, gamma or beta is NULL" : "x, y or alpha is NULL");
    const size_t bytes = (size_t)n * dtype_bytes(dtype);
    if (overlaps(x, bytes, y, bytes))
        return fail(MEA_ERR_INVALID_ARG, "y overlaps x (x is the saved tensor; the forward keeps it intact)");
    mea::AffineLaunch l{};
    l.act = act;
    l.param = param;
    l.dtype = dtype;
    l.layout = layout;
    l.N = shape[0];
    l.C = shape[1];
    l.H = shape[2];
    l.W = shape[3];
    l.x = x;
    l.gamma = p0;
    l.beta = p1;
    l.out = y;
    l.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = kind == 0 ? mea::launch_affine_fwd(l) : mea::launch_channel_swish_fwd(l);
    return e == cudaSuccess ? MEA_OK : cuda_fail(e, name);
}

mea_status_t chan_bwd(int kind, const char *name, int act, int dtype, int layout, const int64_t *shape,
                      const void *x, const void *dy, const float *p0, const float *p1, float param, void *dx,
                      float *d0, float *d1, void *workspace, size_t ws_bytes, mea_stream_t stream)
{
    clear_error();
    if (kind == 0 && !valid_act(act)) return fail(MEA_ERR_INVALID_ARG, "act = %d is not a mea_act_t", act);
    if (!valid_dtype(dtype)) return fail(MEA_ERR_INVALID_ARG, "dtype = %d is not a mea_dtype_t", dtype);
    if (layout != MEA_NCHW && layout != MEA_NHWC)
        return fail(MEA_ERR_INVALID_ARG, "layout = %d is not a mea_layout_t", layout);
    int64_t n = 0;
    mea_status_t st = check_shape(shape, &n);
    if (st != MEA_OK) return st;
    if (shape[1] == 0) return MEA_OK;                 // no channels: nothing to write
    if (kind == 0 && (!d0 || !d1 || !p0 || !p1))
        return fail(MEA_ERR_INVALID_ARG, "gamma, beta, dgamma or dbeta is NULL");
    if (kind == 1 && (!d0 || !p0)) return fail(MEA_ERR_INVALID_ARG, "alpha or dalpha is NULL");
    if (n > 0 && (!x || !dy || !dx)) return fail(MEA_ERR_INVALID_ARG, "x, dy or dx is NULL");
    const size_t need = chan_ws_bytes(kind, dtype, layout, shape);
    if (!workspace || ws_bytes < need)
        return fail(MEA_ERR_WORKSPACE, "%s needs %zu bytes of workspace, got %zu%s", name, need, ws_bytes,
                    workspace ? "" : " (NULL)");
    if (reinterpret_cast<uintptr_t>(workspace) & 15u)
        return fail(MEA_ERR_WORKSPACE, "workspace must be 16-byte aligned");
    const size_t bytes = (size_t)n * dtype_bytes(dtype);
    if (n > 0 && (partial_overlap(dx, dy, bytes) || partial_overlap(dx, x, bytes)))
        return fail(MEA_ERR_INVALID_ARG, "dx partially overlaps x or dy (only exact aliasing is allowed)");
    const size_t cbytes = (size_t)shape[1] * sizeof(float);
    if (kind == 0 && overlaps(d0, cbytes, d1, cbytes)) return fail(MEA_ERR_INVALID_ARG, "dgamma overlaps dbeta");
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (n == 0) {
        // An empty batch still defines the parameter gradients: zero.
        cudaError_t e = cudaMemsetAsync(d0, 0, cbytes, s);
        if (e == cudaSuccess && kind == 0) e = cudaMemsetAsync(d1, 0, cbytes, s);
        return e == cudaSuccess ? MEA_OK : cuda_fail(e, name);
    }
    mea::AffineLaunch l{};
    l.act = act;
    l.param = param;
    l.dtype = dtype;
    l.layout = layout;
    l.N = shape[0];
    l.C = shape[1];
    l.H = shape[2];
    l.W = shape[3];
    l.x = x;
    l.dy = dy;
    l.gamma = p0;
    l.beta = p1;
    l.out = dx;
    l.dgamma = d0;
    l.dbeta = d1;
    l.workspace = workspace;
    l.stream = s;
    cudaError_t e = kind == 0 ? mea::launch_affine_bwd(l) : mea::launch_channel_swish_bwd(l);
    return e == cudaSuccess ? MEA_OK : cuda_fail(e, name);
}

}  // namespace

namespace mea {
void set_last_error_detail(const char *detail) { snprintf(g_err, sizeof(g_err), "%s", detail); }
}  // namespace mea

extern "C" {

const char *mea_status_string(mea_status_t status)
{
    switch (status) {
    case MEA_OK: return "success";
    case MEA_ERR_INVALID_ARG: return "invalid argument";
    case MEA_ERR_UNSUPPORTED: return "unsupported request";
    case MEA_ERR_WORKSPACE: return "workspace missing or too small";
    case MEA_ERR_CUDA: return "CUDA error";
    }
    return "unknown status";
}

const char *mea_last_error(void) { return g_err; }

int mea_version(void) { return 1 * 10000 + 3 * 100 + 0; }

mea_status_t mea_act_fwd(mea_act_t act, mea_dtype_t dtype, const void *x, void *y, int64_t n, float param,
                         const float *param_dev, mea_stream_t stream)
{
    Range range_("mea_act_fwd");
    clear_error();
    if (!valid_act(act)) return fail(MEA_ERR_INVALID_ARG, "act = %d is not a mea_act_t", (int)act);
    if (!valid_dtype(dtype)) return fail(MEA_ERR_INVALID_ARG, "dtype = %d is not a mea_dtype_t", (int)dtype);
    if (n < 0 || n > kMaxElems) return fail(MEA_ERR_INVALID_ARG, "n = %lld out of range", (long long)n);
    if (n == 0) return MEA_OK;
    if (!x || !y) return fail(MEA_ERR_INVALID_ARG, "x or y is NULL");
    const size_t bytes = (size_t)n * dtype_bytes(dtype);
    if (overlaps(x, bytes, y, bytes))
        return fail(MEA_ERR_INVALID_ARG, "y overlaps x (x is the saved tensor; the forward keeps it intact)");
    mea::ActLaunch l{};
    l.act = act;
    l.dtype = dtype;
    l.x = x;
    l.out = y;
    l.n = n;
    l.param = param;
    l.param_dev = param_dev;
    l.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = mea::launch_act_fwd(l);
    return e == cudaSuccess ? MEA_OK : cuda_fail(e, "mea_act_fwd launch");
}

size_t mea_act_bwd_workspace_bytes(mea_act_t act, int64_t n, int want_dparam)
{
    (void)act;
    if (!want_dparam || n < 0) return 0;
    return mea::kWsHeader + sizeof(double) * (size_t)mea::red_grid(n);
}

mea_status_t mea_act_bwd(mea_act_t act, mea_dtype_t dtype, const void *x, const void *dy, void *dx, int64_t n,
                         float param, const float *param_dev, float *dparam_dev, void *workspace,
                         size_t ws_bytes, mea_stream_t stream)
{
    Range range_("mea_act_bwd");
    clear_error();
    if (!valid_act(act)) return fail(MEA_ERR_INVALID_ARG, "act = %d is not a mea_act_t", (int)act);
    if (!valid_dtype(dtype)) return fail(MEA_ERR_INVALID_ARG, "dtype = %d is not a mea_dtype_t", (int)dtype);
    if (n < 0 || n > kMaxElems) return fail(MEA_ERR_INVALID_ARG, "n = %lld out of range", (long long)n);
    if (dparam_dev && act != MEA_SWISH)
        return fail(MEA_ERR_UNSUPPORTED, "a parameter gradient exists only for MEA_SWISH (d alpha)");
    if (dparam_dev) {
        const size_t need = mea_act_bwd_workspace_bytes(act, n, 1);
        if (!workspace || ws_bytes < need)
            return fail(MEA_ERR_WORKSPACE, "d alpha needs %zu bytes of workspace, got %zu%s", need, ws_bytes,
                        workspace ? "" : " (NULL)");
        if (reinterpret_cast<uintptr_t>(workspace) & 15u)
            return fail(MEA_ERR_WORKSPACE, "workspace must be 16-byte aligned");
    }
    if (n == 0 && !dparam_dev) return MEA_OK;
    if (n > 0 && (!x || !dy || !dx)) return fail(MEA_ERR_INVALID_ARG, "x, dy or dx is NULL");
    const size_t bytes = (size_t)n * dtype_bytes(dtype);
    if (n > 0 && (partial_overlap(dx, dy, bytes) || partial_overlap(dx, x, bytes)))
        return fail(MEA_ERR_INVALID_ARG, "dx partially overlaps x or dy (only exact aliasing is allowed)");
    mea::ActLaunch l{};
    l.act = act;
    l.dtype = dtype;
    l.x = x;
    l.dy = dy;
    l.out = dx;
    l.n = n;
    l.param = param;
    l.param_dev = param_dev;
    l.dparam = dparam_dev;
    l.workspace = workspace;
    l.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = mea::launch_act_bwd(l);
    return e == cudaSuccess ? MEA_OK : cuda_fail(e, "mea_act_bwd launch");
}

static size_t round256(size_t b) { return (b + 255) & ~(size_t)255; }

// Validates the segments of a grouped call (each as the single-tensor call
// validates its tensors; no output overlapping another segment's tensors)
// and fills the launch table.  bwd: dy is read and dx may alias dy or x.
static mea_status_t grouped_segments(const char *name, int nseg, const mea_act_segment_t *segs, int dtype,
                                     bool bwd, std::vector<mea::ActSeg> &out)
{
    if (nseg < 0) return fail(MEA_ERR_INVALID_ARG, "%s: nseg = %d", name, nseg);
    if (nseg > 0 && !segs) return fail(MEA_ERR_INVALID_ARG, "%s: segs is NULL", name);
    const size_t es = dtype_bytes(dtype);
    for (int i = 0; i < nseg; ++i) {
        const mea_act_segment_t &g = segs[i];
        if (g.n < 0 || g.n > kMaxElems)
            return fail(MEA_ERR_INVALID_ARG, "%s: segment %d: n = %lld out of range", name, i, (long long)g.n);
        if (g.n == 0) continue;
        if (!g.x || !g.out || (bwd && !g.dy))
            return fail(MEA_ERR_INVALID_ARG, "%s: segment %d: a tensor pointer is NULL", name, i);
        const size_t b = (size_t)g.n * es;
        if (!bwd && overlaps(g.x, b, g.out, b))
            return fail(MEA_ERR_INVALID_ARG, "%s: segment %d: y overlaps x", name, i);
        if (bwd && (partial_overlap(g.out, g.dy, b) || partial_overlap(g.out, g.x, b)))
            return fail(MEA_ERR_INVALID_ARG, "%s: segment %d: dx partially overlaps x or dy", name, i);
    }
    for (int i = 0; i < nseg; ++i) {
        if (segs[i].n == 0) continue;
        const size_t bi = (size_t)segs[i].n * es;
        for (int j = 0; j < nseg; ++j) {
            if (j == i || segs[j].n == 0) continue;
            const size_t bj = (size_t)segs[j].n * es;
            if (overlaps(segs[i].out, bi, segs[j].x, bj) || overlaps(segs[i].out, bi, segs[j].out, bj) ||
                (bwd && overlaps(segs[i].out, bi, segs[j].dy, bj)))
                return fail(MEA_ERR_INVALID_ARG, "%s: the output of segment %d overlaps a tensor of segment %d",
                            name, i, j);
        }
    }
    out.resize((size_t)nseg);
    for (int i = 0; i < nseg; ++i) {
        mea::ActSeg a{};
        a.x = segs[i].x;
        a.dy = bwd ? segs[i].dy : nullptr;
        a.out = segs[i].out;
        a.n = segs[i].n;
        a.param = segs[i].param;
        a.param_dev = segs[i].param_dev;
        a.dparam = bwd ? segs[i].dparam_dev : nullptr;
        out[(size_t)i] = a;
    }
    return MEA_OK;
}

mea_status_t mea_act_fwd_grouped(mea_act_t act, mea_dtype_t dtype, int nseg, const mea_act_segment_t *segs,
                                 mea_stream_t stream)
{
    Range range_("mea_act_fwd_grouped");
    clear_error();
    if (!valid_act(act)) return fail(MEA_ERR_INVALID_ARG, "act = %d is not a mea_act_t", (int)act);
    if (!valid_dtype(dtype)) return fail(MEA_ERR_INVALID_ARG, "dtype = %d is not a mea_dtype_t", (int)dtype);
    std::vector<mea::ActSeg> tab;
    mea_status_t st = grouped_segments("mea_act_fwd_grouped", nseg, segs, dtype, false, tab);
    if (st != MEA_OK) return st;
    if (nseg == 0) return MEA_OK;
    mea::ActGroupLaunch l{act, dtype, nseg, tab.data(), reinterpret_cast<cudaStream_t>(stream)};
    cudaError_t e = mea::launch_act_fwd_grouped(l);
    return e == cudaSuccess ? MEA_OK : cuda_fail(e, "mea_act_fwd_grouped launch");
}

size_t mea_act_bwd_grouped_workspace_bytes(mea_act_t act, int nseg, const mea_act_segment_t *segs)
{
    if (nseg <= 0 || !segs || !segs[0].dparam_dev) return 0;
    size_t total = 0;
    for (int i = 0; i < nseg; ++i) total += round256(mea_act_bwd_workspace_bytes(act, segs[i].n, 1));
    return total;
}

mea_status_t mea_act_bwd_grouped(mea_act_t act, mea_dtype_t dtype, int nseg, const mea_act_segment_t *segs,
                                 void *workspace, size_t ws_bytes, mea_stream_t stream)
{
    Range range_("mea_act_bwd_grouped");
    clear_error();
    if (!valid_act(act)) return fail(MEA_ERR_INVALID_ARG, "act = %d is not a mea_act_t", (int)act);
    if (!valid_dtype(dtype)) return fail(MEA_ERR_INVALID_ARG, "dtype = %d is not a mea_dtype_t", (int)dtype);
    std::vector<mea::ActSeg> tab;
    mea_status_t st = grouped_segments("mea_act_bwd_grouped", nseg, segs, dtype, true, tab);
    if (st != MEA_OK) return st;
    if (nseg == 0) return MEA_OK;
    const bool da = segs[0].dparam_dev != nullptr;
    for (int i = 1; i < nseg; ++i)
        if ((segs[i].dparam_dev != nullptr) != da)
            return fail(MEA_ERR_INVALID_ARG, "mea_act_bwd_grouped: dparam_dev must be set in every segment or "
                                             "in none (segment %d differs)", i);
    if (da) {
        if (act != MEA_SWISH)
            return fail(MEA_ERR_UNSUPPORTED, "a parameter gradient exists only for MEA_SWISH (d alpha)");
        const size_t need = mea_act_bwd_grouped_workspace_bytes(act, nseg, segs);
        if (!workspace || ws_bytes < need)
            return fail(MEA_ERR_WORKSPACE, "grouped d alpha needs %zu bytes of workspace, got %zu%s", need, ws_bytes,
                        workspace ? "" : " (NULL)");
        if (reinterpret_cast<uintptr_t>(workspace) & 255u)
            return fail(MEA_ERR_WORKSPACE, "grouped workspace must be 256-byte aligned");
        size_t off = 0;
        for (int i = 0; i < nseg; ++i) {
            tab[(size_t)i].ws = static_cast<char *>(workspace) + off;
            off += round256(mea_act_bwd_workspace_bytes(act, segs[i].n, 1));
        }
    } else {
        bool any = false;
        for (int i = 0; i < nseg; ++i) any |= segs[i].n > 0;
        if (!any) return MEA_OK;
    }
    mea::ActGroupLaunch l{act, dtype, nseg, tab.data(), reinterpret_cast<cudaStream_t>(stream)};
    cudaError_t e = mea::launch_act_bwd_grouped(l);
    return e == cudaSuccess ? MEA_OK : cuda_fail(e, "mea_act_bwd_grouped launch");
}

mea_status_t mea_affine_bwd_wait_selftest(mea_dtype_t dtype, const int64_t shape[4], const void *x, const void *dy,
                                          const float *gamma, const float *beta, void *dx, void *workspace,
                                          size_t ws_bytes, int *expired, mea_stream_t stream)
{
    Range range_("mea_affine_bwd_wait_selftest");
    clear_error();
    if (!expired) return fail(MEA_ERR_INVALID_ARG, "expired is NULL");
    *expired = 0;
    if (!valid_dtype(dtype)) return fail(MEA_ERR_INVALID_ARG, "dtype = %d is not a mea_dtype_t", (int)dtype);
    int64_t n = 0;
    mea_status_t st = check_shape(shape, &n);
    if (st != MEA_OK) return st;
    if (n == 0 || !x || !dy || !dx || !gamma || !beta)
        return fail(MEA_ERR_INVALID_ARG, "the self-test needs a non-empty NHWC problem and every tensor pointer");
    const size_t need = chan_ws_bytes(0, dtype, MEA_NHWC, shape);
    if (!workspace || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 15u))
        return fail(MEA_ERR_WORKSPACE, "the self-test needs %zu bytes of 16-byte aligned workspace", need);
    mea::AffineLaunch l{};
    l.act = MEA_SWISH;
    l.param = 1.f;
    l.dtype = dtype;
    l.layout = MEA_NHWC;
    l.N = shape[0];
    l.C = shape[1];
    l.H = shape[2];
    l.W = shape[3];
    l.x = x;
    l.dy = dy;
    l.gamma = gamma;
    l.beta = beta;
    l.out = dx;
    l.workspace = workspace;
    l.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = mea::launch_affine_bwd_wait_selftest(l);
    if (e == cudaErrorNotSupported)
        return fail(MEA_ERR_UNSUPPORTED, "this shape or alignment does not take the pipelined NHWC backward");
    if (e == cudaSuccess) e = cudaStreamSynchronize(l.stream);
    unsigned int word = 0;
    unsigned int *err = reinterpret_cast<unsigned int *>(static_cast<char *>(workspace) + 4);
    if (e == cudaSuccess) e = cudaMemcpy(&word, err, sizeof(word), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemset(err, 0, sizeof(word));
    if (e != cudaSuccess) return cuda_fail(e, "mea_affine_bwd_wait_selftest");
    *expired = (int)word;
    return MEA_OK;
}

size_t mea_affine_swish_bwd_workspace_bytes(mea_dtype_t dtype, mea_layout_t layout, const int64_t shape[4])
{
    return chan_ws_bytes(0, dtype, layout, shape);
}

mea_status_t mea_affine_swish_fwd(mea_dtype_t dtype, mea_layout_t layout, const int64_t shape[4], const void *x,
                                  const float *gamma, const float *beta, void *y, mea_stream_t stream)
{
    Range range_("mea_affine_swish_fwd");
    return chan_fwd(0, "mea_affine_swish_fwd", MEA_SWISH, dtype, layout, shape, x, gamma, beta, 1.f, y, stream);
}

mea_status_t mea_affine_swish_bwd(mea_dtype_t dtype, mea_layout_t layout, const int64_t shape[4], const void *x,
                                  const void *dy, const float *gamma, const float *beta, void *dx, float *dgamma,
                                  float *dbeta, void *workspace, size_t ws_bytes, mea_stream_t stream)
{
    Range range_("mea_affine_swish_bwd");
    return chan_bwd(0, "mea_affine_swish_bwd", MEA_SWISH, dtype, layout, shape, x, dy, gamma, beta, 1.f, dx, dgamma,
                    dbeta, workspace, ws_bytes, stream);
}

size_t mea_affine_act_bwd_workspace_bytes(mea_dtype_t dtype, mea_layout_t layout, const int64_t shape[4])
{
    return chan_ws_bytes(0, dtype, layout, shape);
}

mea_status_t mea_affine_act_fwd(mea_act_t act, mea_dtype_t dtype, mea_layout_t layout, const int64_t shape[4],
                                const void *x, const float *gamma, const float *beta, float param, void *y,
                                mea_stream_t stream)
{
    Range range_("mea_affine_act_fwd");
    return chan_fwd(0, "mea_affine_act_fwd", act, dtype, layout, shape, x, gamma, beta, param, y, stream);
}

mea_status_t mea_affine_act_bwd(mea_act_t act, mea_dtype_t dtype, mea_layout_t layout, const int64_t shape[4],
                                const void *x, const void *dy, const float *gamma, const float *beta, float param,
                                void *dx, float *dgamma, float *dbeta, void *workspace, size_t ws_bytes,
                                mea_stream_t stream)
{
    Range range_("mea_affine_act_bwd");
    return chan_bwd(0, "mea_affine_act_bwd", act, dtype, layout, shape, x, dy, gamma, beta, param, dx, dgamma, dbeta,
                    workspace, ws_bytes, stream);
}

size_t mea_swish_channel_bwd_workspace_bytes(mea_dtype_t dtype, mea_layout_t layout, const int64_t shape[4])
{
    return chan_ws_bytes(1, dtype, layout, shape);
}

mea_status_t mea_swish_channel_fwd(mea_dtype_t dtype, mea_layout_t layout, const int64_t shape[4], const void *x,
                                   const float *alpha, void *y, mea_stream_t stream)
{
    Range range_("mea_swish_channel_fwd");
    return chan_fwd(1, "mea_swish_channel_fwd", MEA_SWISH, dtype, layout, shape, x, alpha, nullptr, 1.f, y, stream);
}

mea_status_t mea_swish_channel_bwd(mea_dtype_t dtype, mea_layout_t layout, const int64_t shape[4], const void *x,
                                   const void *dy, const float *alpha, void *dx, float *dalpha, void *workspace,
                                   size_t ws_bytes, mea_stream_t stream)
{
    Range range_("mea_swish_channel_bwd");
    return chan_bwd(1, "mea_swish_channel_bwd", MEA_SWISH, dtype, layout, shape, x, dy, alpha, nullptr, 1.f, dx,
                    dalpha, nullptr, workspace, ws_bytes, stream);
}

// Validates a grouped per-channel Swish call and converts its segments.
static mea_status_t channel_segments(const char *name, int nseg, const mea_channel_segment_t *segs, int dtype,
                                     bool bwd, std::vector<mea::ChanSeg> &out)
{
    if (!valid_dtype(dtype)) return fail(MEA_ERR_INVALID_ARG, "dtype = %d is not a mea_dtype_t", dtype);
    if (nseg < 0) return fail(MEA_ERR_INVALID_ARG, "%s: nseg = %d", name, nseg);
    if (nseg > 0 && !segs) return fail(MEA_ERR_INVALID_ARG, "%s: segs is NULL", name);
    const size_t es = dtype_bytes(dtype);
    std::vector<size_t> bytes((size_t)nseg, 0);
    for (int i = 0; i < nseg; ++i) {
        const mea_channel_segment_t &g = segs[i];
        int64_t n = 0;
        mea_status_t st = check_shape(g.shape, &n);
        if (st != MEA_OK) {
            char why[256];
            snprintf(why, sizeof(why), "%s", mea_last_error());
            return fail(st, "%s: segment %d: %s", name, i, why);
        }
        bytes[(size_t)i] = (size_t)n * es;
        const int64_t C = g.shape[1];
        if (C > 0 && (!g.alpha || (bwd && !g.dalpha)))
            return fail(MEA_ERR_INVALID_ARG, "%s: segment %d: alpha%s is NULL", name, i, bwd ? " or dalpha" : "");
        if (n == 0) continue;
        if (!g.x || !g.out || (bwd && !g.dy))
            return fail(MEA_ERR_INVALID_ARG, "%s: segment %d: a tensor pointer is NULL", name, i);
        const size_t b = bytes[(size_t)i];
        if (!bwd && overlaps(g.x, b, g.out, b))
            return fail(MEA_ERR_INVALID_ARG, "%s: segment %d: y overlaps x", name, i);
        if (bwd && (partial_overlap(g.out, g.dy, b) || partial_overlap(g.out, g.x, b)))
            return fail(MEA_ERR_INVALID_ARG, "%s: segment %d: dx partially overlaps x or dy", name, i);
    }
    for (int i = 0; i < nseg; ++i) {
        const size_t bi = bytes[(size_t)i], ci = (size_t)segs[i].shape[1] * sizeof(float);
        for (int j = 0; j < nseg; ++j) {
            if (j == i) continue;
            const size_t bj = bytes[(size_t)j], cj = (size_t)segs[j].shape[1] * sizeof(float);
            if (bi > 0 && bj > 0 &&
                (overlaps(segs[i].out, bi, segs[j].x, bj) || overlaps(segs[i].out, bi, segs[j].out, bj) ||
                 (bwd && overlaps(segs[i].out, bi, segs[j].dy, bj))))
                return fail(MEA_ERR_INVALID_ARG, "%s: the output of segment %d overlaps a tensor of segment %d",
                            name, i, j);
            if (bwd && ci > 0 && cj > 0 && overlaps(segs[i].dalpha, ci, segs[j].dalpha, cj))
                return fail(MEA_ERR_INVALID_ARG, "%s: dalpha of segments %d and %d overlap", name, i, j);
        }
    }
    out.resize((size_t)nseg);
    for (int i = 0; i < nseg; ++i) {
        const mea_channel_segment_t &g = segs[i];
        mea::ChanSeg c{};
        c.x = g.x;
        c.dy = bwd ? g.dy : nullptr;
        c.out = g.out;
        c.alpha = g.alpha;
        c.dalpha = bwd ? g.dalpha : nullptr;
        c.N = g.shape[0];
        c.C = g.shape[1];
        c.H = g.shape[2];
        c.W = g.shape[3];
        out[(size_t)i] = c;
    }
    return MEA_OK;
}

mea_status_t mea_swish_channel_fwd_grouped(mea_dtype_t dtype, int nseg, const mea_channel_segment_t *segs,
                                           mea_stream_t stream)
{
    Range range_("mea_swish_channel_fwd_grouped");
    clear_error();
    std::vector<mea::ChanSeg> tab;
    mea_status_t st = channel_segments("mea_swish_channel_fwd_grouped", nseg, segs, dtype, false, tab);
    if (st != MEA_OK) return st;
    if (nseg == 0) return MEA_OK;
    cudaError_t e = mea::launch_channel_swish_fwd_grouped(dtype, nseg, tab.data(), reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MEA_OK : cuda_fail(e, "mea_swish_channel_fwd_grouped launch");
}

size_t mea_swish_channel_bwd_grouped_workspace_bytes(mea_dtype_t dtype, int nseg, const mea_channel_segment_t *segs)
{
    if (nseg <= 0 || !segs) return 0;
    size_t total = 0;
    for (int i = 0; i < nseg; ++i) {
        const size_t b = chan_ws_bytes(1, dtype, MEA_NCHW, segs[i].shape);
        if (b == 0) return 0;
        total += round256(b);
    }
    return total;
}

mea_status_t mea_swish_channel_bwd_grouped(mea_dtype_t dtype, int nseg, const mea_channel_segment_t *segs,
                                           void *workspace, size_t ws_bytes, mea_stream_t stream)
{
    Range range_("mea_swish_channel_bwd_grouped");
    clear_error();
    std::vector<mea::ChanSeg> tab;
    mea_status_t st = channel_segments("mea_swish_channel_bwd_grouped", nseg, segs, dtype, true, tab);
    if (st != MEA_OK) return st;
    if (nseg == 0) return MEA_OK;
    const size_t need = mea_swish_channel_bwd_grouped_workspace_bytes(dtype, nseg, segs);
    if (!workspace || ws_bytes < need)
        return fail(MEA_ERR_WORKSPACE, "mea_swish_channel_bwd_grouped needs %zu bytes of workspace, got %zu%s", need,
                    ws_bytes, workspace ? "" : " (NULL)");
    if (reinterpret_cast<uintptr_t>(workspace) & 255u)
        return fail(MEA_ERR_WORKSPACE, "grouped workspace must be 256-byte aligned");
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    size_t off = 0;
    for (int i = 0; i < nseg; ++i) {
        tab[(size_t)i].ws = static_cast<char *>(workspace) + off;
        off += round256(chan_ws_bytes(1, dtype, MEA_NCHW, segs[i].shape));
        // An empty batch still defines d alpha: zero.
        const mea::ChanSeg &g = tab[(size_t)i];
        if (g.C > 0 && g.N * g.H * g.W == 0) {
            cudaError_t e = cudaMemsetAsync(g.dalpha, 0, (size_t)g.C * sizeof(float), s);
            if (e != cudaSuccess) return cuda_fail(e, "mea_swish_channel_bwd_grouped");
        }
    }
    cudaError_t e = mea::launch_channel_swish_bwd_grouped(dtype, nseg, tab.data(), s);
    return e == cudaSuccess ? MEA_OK : cuda_fail(e, "mea_swish_channel_bwd_grouped launch");
}

static mea_status_t check_matmul(const char *name, int act, int64_t M, int64_t N, int64_t K)
{
    (void)name;
    if (!valid_act(act)) return fail(MEA_ERR_INVALID_ARG, "act = %d is not a mea_act_t", act);
    if (M < 0 || N < 0 || K < 0) return fail(MEA_ERR_INVALID_ARG, "M, N and K must be non-negative");
    const int64_t lim = (int64_t)1 << 31;
    if (M >= lim || N >= lim || K >= lim) return fail(MEA_ERR_UNSUPPORTED, "M, N and K must be below 2^31");
    return MEA_OK;
}

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

mea_status_t mea_matmul_act_fwd(mea_act_t act, int64_t M, int64_t N, int64_t K, const void *x, const void *w,
                                float param, void *z, void *y, mea_stream_t stream)
{
    Range range_("mea_matmul_act_fwd");
    clear_error();
    mea_status_t st = check_matmul("mea_matmul_act_fwd", act, M, N, K);
    if (st != MEA_OK) return st;
    if (M == 0 || N == 0) return MEA_OK;
    if (K == 0) return fail(MEA_ERR_UNSUPPORTED, "K = 0 (an empty product) is not served");
    if (K % 8 || N % 8) return fail(MEA_ERR_UNSUPPORTED, "K and N must be multiples of 8");
    if (!x || !w) return fail(MEA_ERR_INVALID_ARG, "x or w is NULL");
    if (!z && !y) return fail(MEA_ERR_INVALID_ARG, "z and y are both NULL");
    if (!aligned16(x) || !aligned16(w) || (z && !aligned16(z)) || (y && !aligned16(y)))
        return fail(MEA_ERR_UNSUPPORTED, "x, w, z and y must be 16-byte aligned");
    const size_t bx = (size_t)M * K * 2, bw = (size_t)N * K * 2, bo = (size_t)M * N * 2;
    for (void *o : {z, y}) {
        if (!o) continue;
        if (overlaps(o, bo, x, bx) || overlaps(o, bo, w, bw))
            return fail(MEA_ERR_INVALID_ARG, "an output overlaps x or w");
    }
    if (z && y && overlaps(z, bo, y, bo)) return fail(MEA_ERR_INVALID_ARG, "z overlaps y");
    mea::MatmulLaunch l{};
    l.act = act;
    l.mode = 0;
    l.M = M;
    l.N = N;
    l.K = K;
    l.x = x;
    l.w = w;
    l.out0 = z;
    l.out1 = y;
    l.param = param;
    l.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = mea::launch_matmul_act(l);
    return e == cudaSuccess ? MEA_OK : cuda_fail(e, "mea_matmul_act_fwd launch");
}

mea_status_t mea_matmul_act_bwd(mea_act_t act, int64_t M, int64_t N, int64_t K, const void *g, const void *w,
                                const void *z, float param, void *dz, mea_stream_t stream)
{
    Range range_("mea_matmul_act_bwd");
    clear_error();
    mea_status_t st = check_matmul("mea_matmul_act_bwd", act, M, N, K);
    if (st != MEA_OK) return st;
    if (M == 0 || N == 0) return MEA_OK;
    if (K == 0) return fail(MEA_ERR_UNSUPPORTED, "K = 0 (an empty product) is not served");
    if (K % 8 || N % 8) return fail(MEA_ERR_UNSUPPORTED, "K and N must be multiples of 8");
    if (!g || !w || !z || !dz) return fail(MEA_ERR_INVALID_ARG, "g, w, z or dz is NULL");
    if (!aligned16(g) || !aligned16(w) || !aligned16(z) || !aligned16(dz))
        return fail(MEA_ERR_UNSUPPORTED, "g, w, z and dz must be 16-byte aligned");
    const size_t bg = (size_t)M * K * 2, bw = (size_t)N * K * 2, bo = (size_t)M * N * 2;
    if (overlaps(dz, bo, g, bg) || overlaps(dz, bo, w, bw))
        return fail(MEA_ERR_INVALID_ARG, "dz overlaps g or w");
    if (partial_overlap(dz, z, bo)) return fail(MEA_ERR_INVALID_ARG, "dz partially overlaps z");
    mea::MatmulLaunch l{};
    l.act = act;
    l.mode = 1;
    l.M = M;
    l.N = N;
    l.K = K;
    l.x = g;
    l.w = w;
    l.zin = z;
    l.out1 = dz;
    l.param = param;
    l.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = mea::launch_matmul_act(l);
    return e == cudaSuccess ? MEA_OK : cuda_fail(e, "mea_matmul_act_bwd launch");
}

int mea_matmul_error_word(int clear)
{
    clear_error();
    unsigned int w = 0;
    cudaError_t e = mea::matmul_error_word(clear, &w);
    if (e != cudaSuccess) {
        cuda_fail(e, "mea_matmul_error_word");
        return -1;
    }
    return (int)w;
}

static mea_status_t bn_common(const char *name, int dtype, int npieces, const void *const *pieces,
                              const int64_t *channels, int64_t N, int64_t HW, mea::BnLaunch *l, size_t *plane_bytes)
{
    (void)name;
    if (!valid_dtype(dtype)) return fail(MEA_ERR_INVALID_ARG, "dtype = %d is not a mea_dtype_t", dtype);
    if (npieces < 1 || npieces > mea::kBnMaxPieces)
        return fail(MEA_ERR_UNSUPPORTED, "npieces = %d is outside 1..%d", npieces, mea::kBnMaxPieces);
    if (!pieces || !channels) return fail(MEA_ERR_INVALID_ARG, "pieces or channels is NULL");
    if (N < 0 || HW < 0) return fail(MEA_ERR_INVALID_ARG, "N and HW must be non-negative");
    if (N == 0 || HW == 0) return fail(MEA_ERR_INVALID_ARG, "batch statistics need N HW >= 1");
    int64_t C = 0;
    l->in.npieces = npieces;
    for (int i = 0; i < npieces; ++i) {
        if (channels[i] < 1) return fail(MEA_ERR_INVALID_ARG, "channels[%d] = %lld", i, (long long)channels[i]);
        if (!pieces[i]) return fail(MEA_ERR_INVALID_ARG, "pieces[%d] is NULL", i);
        l->in.ptr[i] = pieces[i];
        l->in.off[i] = (int)C;
        C += channels[i];
        if (C >= ((int64_t)1 << 31)) return fail(MEA_ERR_UNSUPPORTED, "more than 2^31 channels");
    }
    l->in.off[npieces] = (int)C;
    if (N > kMaxElems / HW || N * HW > kMaxElems / C) return fail(MEA_ERR_INVALID_ARG, "tensor too large");
    if (N * HW >= ((int64_t)1 << 31)) return fail(MEA_ERR_UNSUPPORTED, "N HW must be below 2^31");
    l->dtype = dtype;
    l->N = N;
    l->C = C;
    l->HW = HW;
    *plane_bytes = (size_t)N * HW * dtype_bytes(dtype);
    return MEA_OK;
}

size_t mea_concat_bn_relu_workspace_bytes(int64_t N, int64_t C)
{
    if (N < 1 || C < 1) return 0;
    return mea::bn_workspace_bytes(N, C);
}

mea_status_t mea_concat_bn_relu_fwd(mea_dtype_t dtype, int npieces, const void *const *pieces, const int64_t *channels,
                                    int64_t N, int64_t HW, const float *gamma, const float *beta, float eps,
                                    float momentum, float *running_mean, float *running_var, float *mean,
                                    float *invstd, void *y, void *workspace, size_t ws_bytes, mea_stream_t stream)
{
    Range range_("mea_concat_bn_relu_fwd");
    clear_error();
    mea::BnLaunch l{};
    size_t pb = 0;
    mea_status_t st = bn_common("mea_concat_bn_relu_fwd", dtype, npieces, pieces, channels, N, HW, &l, &pb);
    if (st != MEA_OK) return st;
    if (!gamma || !beta || !mean || !invstd || !y) return fail(MEA_ERR_INVALID_ARG, "gamma, beta, mean, invstd or y is NULL");
    if (!running_mean != !running_var) return fail(MEA_ERR_INVALID_ARG, "running_mean and running_var go together");
    if (!(eps >= 0.f)) return fail(MEA_ERR_INVALID_ARG, "eps must be >= 0");
    const size_t need = mea::bn_workspace_bytes(N, l.C);
    if (!workspace || ws_bytes < need)
        return fail(MEA_ERR_WORKSPACE, "needs %zu bytes of workspace, got %zu%s", need, ws_bytes, workspace ? "" : " (NULL)");
    if (reinterpret_cast<uintptr_t>(workspace) & 15u) return fail(MEA_ERR_WORKSPACE, "workspace must be 16-byte aligned");
    for (int i = 0; i < npieces; ++i)
        if (overlaps(y, pb * l.C, pieces[i], pb * channels[i])) return fail(MEA_ERR_INVALID_ARG, "y overlaps piece %d", i);
    l.gamma = gamma;
    l.beta = beta;
    l.eps = eps;
    l.momentum = momentum;
    l.running_mean = running_mean;
    l.running_var = running_var;
    l.mean = mean;
    l.invstd = invstd;
    l.y = y;
    l.workspace = workspace;
    l.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = mea::launch_bn_fwd(l);
    return e == cudaSuccess ? MEA_OK : cuda_fail(e, "mea_concat_bn_relu_fwd launch");
}

mea_status_t mea_concat_bn_relu_apply(mea_dtype_t dtype, int npieces, const void *const *pieces,
                                      const int64_t *channels, int64_t N, int64_t HW, const float *gamma,
                                      const float *beta, const float *mean, const float *invstd, void *y,
                                      mea_stream_t stream)
{
    Range range_("mea_concat_bn_relu_apply");
    clear_error();
    mea::BnLaunch l{};
    size_t pb = 0;
    mea_status_t st = bn_common("mea_concat_bn_relu_apply", dtype, npieces, pieces, channels, N, HW, &l, &pb);
    if (st != MEA_OK) return st;
    if (!gamma || !beta || !mean || !invstd || !y) return fail(MEA_ERR_INVALID_ARG, "gamma, beta, mean, invstd or y is NULL");
    for (int i = 0; i < npieces; ++i)
        if (overlaps(y, pb * l.C, pieces[i], pb * channels[i])) return fail(MEA_ERR_INVALID_ARG, "y overlaps piece %d", i);
    l.gamma = gamma;
    l.beta = beta;
    l.mean = const_cast<float *>(mean);
    l.invstd = const_cast<float *>(invstd);
    l.y = y;
    l.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = mea::launch_bn_apply(l);
    return e == cudaSuccess ? MEA_OK : cuda_fail(e, "mea_concat_bn_relu_apply launch");
}

mea_status_t mea_concat_bn_relu_bwd(mea_dtype_t dtype, int npieces, const void *const *pieces, const int64_t *channels,
                                    int64_t N, int64_t HW, const void *dy, const float *gamma, const float *beta,
                                    const float *mean, const float *invstd, void *const *dpieces, int accumulate,
                                    float *dgamma, float *dbeta, void *workspace, size_t ws_bytes,
                                    mea_stream_t stream)
{
    Range range_("mea_concat_bn_relu_bwd");
    clear_error();
    mea::BnLaunch l{};
    size_t pb = 0;
    mea_status_t st = bn_common("mea_concat_bn_relu_bwd", dtype, npieces, pieces, channels, N, HW, &l, &pb);
    if (st != MEA_OK) return st;
    if (!dy || !gamma || !beta || !mean || !invstd || !dgamma || !dbeta || !dpieces)
        return fail(MEA_ERR_INVALID_ARG, "dy, gamma, beta, mean, invstd, dgamma, dbeta or dpieces is NULL");
    const size_t need = mea::bn_workspace_bytes(N, l.C);
    if (!workspace || ws_bytes < need)
        return fail(MEA_ERR_WORKSPACE, "needs %zu bytes of workspace, got %zu%s", need, ws_bytes, workspace ? "" : " (NULL)");
    if (reinterpret_cast<uintptr_t>(workspace) & 15u) return fail(MEA_ERR_WORKSPACE, "workspace must be 16-byte aligned");
    const size_t cb = (size_t)l.C * sizeof(float);
    if (overlaps(dgamma, cb, dbeta, cb)) return fail(MEA_ERR_INVALID_ARG, "dgamma overlaps dbeta");
    for (int i = 0; i < npieces; ++i) {
        if (!dpieces[i]) return fail(MEA_ERR_INVALID_ARG, "dpieces[%d] is NULL", i);
        const size_t bi = pb * channels[i];
        if (overlaps(dpieces[i], bi, dy, pb * l.C)) return fail(MEA_ERR_INVALID_ARG, "dpieces[%d] overlaps dy", i);
        for (int j = 0; j < npieces; ++j) {
            const size_t bj = pb * channels[j];
            if (j == i ? partial_overlap(dpieces[i], pieces[j], bi) : overlaps(dpieces[i], bi, pieces[j], bj))
                return fail(MEA_ERR_INVALID_ARG, "dpieces[%d] overlaps piece %d", i, j);
            if (j != i && overlaps(dpieces[i], bi, dpieces[j], bj))
                return fail(MEA_ERR_INVALID_ARG, "dpieces[%d] overlaps dpieces[%d]", i, j);
        }
        l.din.ptr[i] = dpieces[i];
    }
    l.dy = dy;
    l.gamma = gamma;
    l.beta = beta;
    l.mean = const_cast<float *>(mean);
    l.invstd = const_cast<float *>(invstd);
    l.accumulate = accumulate;
    l.dgamma = dgamma;
    l.dbeta = dbeta;
    l.workspace = workspace;
    l.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = mea::launch_bn_bwd(l);
    return e == cudaSuccess ? MEA_OK : cuda_fail(e, "mea_concat_bn_relu_bwd launch");
}

}  // extern "C"
