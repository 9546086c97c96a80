// mea_channel_alpha.cu -- Swish with one learnable alpha per channel:
//
//   y = x Sigmoid(alpha_c x)
//   dx = dy (s + alpha_c x s Sigmoid(-alpha_c x)),  s = Sigmoid(alpha_c x)
//   dalpha_c = sum dy x^2 s Sigmoid(-alpha_c x)   (over all N H W positions)
//
// The per-channel generalisation of the scalar learnable alpha (the Swish
// page's module carries alpha; its gradient in alpha is the derivative of
// sum(dy Swish) in alpha).  Data movement and the deterministic reductions
// are the per-channel kernels of mea_channel.cuh; this file supplies the
// arithmetic (ChannelSwishOp) and the dispatch over storage dtype.
#include "mea_channel.cuh"

namespace mea {

struct ChannelSwishOp {
    static constexpr int NR = 1;   // dalpha
    struct K {
    };
    using Ch = Coef;               // Swish constants of the channel's alpha
    static __device__ __forceinline__ K kcoef(const ChanArgs &) { return K{}; }
    static __device__ __forceinline__ Ch load(const ChanArgs &a, int c) { return Swish::coef(__ldg(a.p0 + c)); }

    template <bool P>
    static __device__ __forceinline__ float f(float x, const K &, const Ch &h, bool &tail)
    {
        return Swish::f<P>(x, h, tail);
    }
    template <bool P>
    static __device__ __forceinline__ float f_tail(float x, const K &, const Ch &h)
    {
        return Swish::f_tail<P>(x, h);
    }
    static __device__ __forceinline__ bool is_tail(float x, const K &, const Ch &h) { return Swish::is_tail(x, h); }
    // Every element the backward main path may flag (deep tail; with bf16
    // storage the neighbourhood of the zero of f').
    template <bool P>
    static __device__ __forceinline__ bool flag_bwd(float x, const K &, const Ch &h)
    {
        return Swish::bwd_flagged<P>(x, h);
    }
    // o = dx, t = d alpha term
    template <bool P>
    static __device__ __forceinline__ void bwd(float x, float dy, const K &, const Ch &h, bool &tail, float &o,
                                               float &t)
    {
        o = Swish::df_da<P>(x, dy, h, tail, t);
    }
    // A flagged element: the near-zero or deep-tail recompute, else the main
    // form.
    template <bool P>
    static __device__ __forceinline__ void bwd_tail(float x, float dy, const K &, const Ch &h, float &o, float &t)
    {
        if (Swish::is_tail_bwd<P>(x, h)) {
            o = Swish::df_da_tail<P>(x, dy, h, t);
            return;
        }
        bool unused = false;
        o = Swish::df_da<P>(x, dy, h, unused, t);
    }
    static __device__ __forceinline__ float finish(float, float o, float t, const Ch &, float (&acc)[NR])
    {
        acc[0] += t;
        return o;
    }

    // Two channels at once (each with its own alpha, so f' stays per element).
    struct Ch2 {
        Ch a, b;
    };
    static __device__ __forceinline__ Ch2 pair(const Ch &a, const Ch &b) { return Ch2{a, b}; }
    template <bool P>
    static __device__ __forceinline__ F2 f2(F2 x, const K &, const Ch2 &h, bool &tail)
    {
        float x0, x1;
        upk(x, x0, x1);
        return pk(Swish::f<P>(x0, h.a, tail), Swish::f<P>(x1, h.b, tail));
    }
    template <bool P>
    static __device__ __forceinline__ void bwd2(F2 x, F2 dy, const K &, const Ch2 &h, bool &tail, F2 &o, F2 &t)
    {
        float x0, x1, d0, d1, t0, t1;
        upk(x, x0, x1);
        upk(dy, d0, d1);
        const float o0 = Swish::df_da<P>(x0, d0, h.a, tail, t0);
        const float o1 = Swish::df_da<P>(x1, d1, h.b, tail, t1);
        o = pk(o0, o1);
        t = pk(t0, t1);
    }
    static __device__ __forceinline__ F2 finish2(F2, F2 o, F2 t, const Ch2 &, F2 (&acc)[NR])
    {
        acc[0] = add2(acc[0], t);
        return o;
    }
};

size_t channel_swish_bwd_workspace_bytes(int dtype, int layout, int64_t N, int64_t C, int64_t H, int64_t W)
{
    return chan_bwd_workspace_bytes(ChannelSwishOp::NR, dtype, layout, N, C, H, W);
}

cudaError_t launch_channel_swish_fwd(const AffineLaunch &a)
{
    const ChanArgs ca{a.gamma, nullptr, 1.f};
    return a.dtype == kBF16 ? launch_channel<ChannelSwishOp, Bf16, 0>(a, ca, nullptr, nullptr)
                            : launch_channel<ChannelSwishOp, float, 0>(a, ca, nullptr, nullptr);
}

cudaError_t launch_channel_swish_bwd(const AffineLaunch &a)
{
    const ChanArgs ca{a.gamma, nullptr, 1.f};
    return a.dtype == kBF16 ? launch_channel<ChannelSwishOp, Bf16, 1>(a, ca, a.dgamma, nullptr)
                            : launch_channel<ChannelSwishOp, float, 1>(a, ca, a.dgamma, nullptr);
}

namespace {

// Segments the row path takes go into one grid (kMaxRowSegs at a time),
// each with the block partition and partials of its single-tensor launch;
// any other segment is launched alone on its usual path.
template <typename T, int MODE>
cudaError_t launch_grouped(int dtype, int nseg, const ChanSeg *segs, cudaStream_t stream)
{
    constexpr int NR = ChannelSwishOp::NR, V = Store<T>::V;
    RowSegTable tab{};
    tab.scalar = 1.f;
    int k = 0;
    int64_t blocks = 0, outs = 0;
    size_t smem = 0;
    auto flush = [&]() -> cudaError_t {
        if (k == 0) return cudaSuccess;
        tab.nseg = k;
        tab.start[k] = (int)blocks;
        tab.ostart[k] = (int)outs;
        cudaError_t e = launch_pdl(chan_row_group_kernel<ChannelSwishOp, T, MODE>, dim3((unsigned)blocks),
                                   dim3(kRowThreads), smem, stream, tab);
        if (e == cudaSuccess && MODE == 1) {
            const int64_t cb = (outs + kRowThreads / 32 - 1) / (kRowThreads / 32);
            e = launch_pdl(chan_row_group_colsum_kernel<NR>, dim3((unsigned)cb), dim3(kRowThreads), 0, stream, tab);
        }
        k = 0;
        blocks = outs = 0;
        smem = 0;
        return e;
    };
    for (int i = 0; i < nseg; ++i) {
        const ChanSeg &g = segs[i];
        const int64_t HW = g.H * g.W;
        if (g.N * g.C * HW == 0) continue;
        uintptr_t al = reinterpret_cast<uintptr_t>(g.x) | reinterpret_cast<uintptr_t>(g.out);
        if (MODE == 1) al |= reinterpret_cast<uintptr_t>(g.dy);
        const RowShape rs = row_shape(NR, V, g.N, g.C, HW);
        cudaError_t e = cudaSuccess;
        if (rs.planes == 0 || (al & 15u) || rs.grid > 0x7fffffff || NR * g.C > 0x7fffffff) {
            AffineLaunch a{};
            a.act = 6;
            a.param = 1.f;
            a.dtype = dtype;
            a.layout = 0;
            a.N = g.N;
            a.C = g.C;
            a.H = g.H;
            a.W = g.W;
            a.x = g.x;
            a.dy = g.dy;
            a.gamma = g.alpha;
            a.out = g.out;
            a.dgamma = g.dalpha;
            a.workspace = g.ws;
            a.stream = stream;
            if (MODE == 1) e = cudaMemsetAsync(g.ws, 0, kWsHeader, stream);
            if (e == cudaSuccess)
                e = launch_channel<ChannelSwishOp, T, MODE>(a, ChanArgs{g.alpha, nullptr, 1.f},
                                                            MODE == 1 ? g.dalpha : nullptr, nullptr);
            if (e != cudaSuccess) return e;
            continue;
        }
        if (k == kMaxRowSegs || blocks + rs.grid > 0x7fffffff || outs + NR * g.C > 0x7fffffff) {
            e = flush();
            if (e != cudaSuccess) return e;
        }
        RowSeg &r = tab.seg[k];
        r.x = g.x;
        r.dy = MODE == 1 ? g.dy : nullptr;
        r.out = g.out;
        r.p0 = g.alpha;
        r.p1 = nullptr;
        r.partials = MODE == 1 ? reinterpret_cast<double *>(static_cast<char *>(g.ws) + kWsHeader) : nullptr;
        r.out0 = MODE == 1 ? g.dalpha : nullptr;
        r.out1 = nullptr;
        r.N = g.N;
        r.C = g.C;
        r.HW = HW;
        r.P = rs.planes;
        tab.start[k] = (int)blocks;
        tab.ostart[k] = (int)outs;
        blocks += rs.grid;
        outs += NR * g.C;
        if (MODE == 1) {
            const size_t b = sizeof(float) * NR * (size_t)rs.planes * (size_t)HW;
            if (b > smem) smem = b;
        }
        ++k;
    }
    return flush();
}

}  // namespace

cudaError_t launch_channel_swish_fwd_grouped(int dtype, int nseg, const ChanSeg *segs, cudaStream_t stream)
{
    return dtype == kBF16 ? launch_grouped<Bf16, 0>(dtype, nseg, segs, stream)
                          : launch_grouped<float, 0>(dtype, nseg, segs, stream);
}

cudaError_t launch_channel_swish_bwd_grouped(int dtype, int nseg, const ChanSeg *segs, cudaStream_t stream)
{
    return dtype == kBF16 ? launch_grouped<Bf16, 1>(dtype, nseg, segs, stream)
                          : launch_grouped<float, 1>(dtype, nseg, segs, stream);
}

}  // namespace mea
