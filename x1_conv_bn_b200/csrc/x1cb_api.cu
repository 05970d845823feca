// The C ABI of include/x1cb.h: argument checks, launch plans (cached per
// shape), and the three-stage bottleneck chain.  All compute is in the
// kernels of x1cb_conv.cu and x1cb_pack.cu.
#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <initializer_list>
#include <mutex>

#include "x1cb_internal.h"

namespace x1cb {
namespace {

std::atomic<unsigned long long> g_wait_limit_ns{0};
std::atomic<int> g_inject{0};
std::atomic<int> g_block_fusion{0};
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;

struct DevInfo {
    int ok = 0;  // 1 = sm_100, -1 = not
    int sms = 0;
};

int device_info(int &sms)
{
    static std::mutex mu;
    static DevInfo info[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return X1CB_ERR_CUDA;
    std::lock_guard<std::mutex> lk(mu);
    if (info[dev].ok == 0) {
        int major = 0, n = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return X1CB_ERR_CUDA;
        info[dev].ok = (major == 10) ? 1 : -1;
        info[dev].sms = n;
    }
    if (info[dev].ok != 1)
        return X1CB_ERR_ARCH;
    sms = info[dev].sms;
    return X1CB_OK;
}

// Small cache of launch plans keyed by shape (the tile search is not free and
// a B=1 call is latency-bound).
struct PlanKey {
    int B, H, W, Ic, Oc, R, has_res, sms;
    int stride, Hin, Win, Ic2, stride2, Hin2, Win2, pool, Rw, stride_w;
    bool operator==(const PlanKey &o) const { return std::memcmp(this, &o, sizeof(*this)) == 0; }
};

int get_plan(ConvPlan &p, int B, int H, int W, int Ic, int Oc, int R, int has_res, int S,
             int m_r, int sms, const ConvGeom &g = ConvGeom{})
{
    static std::mutex mu;
    static PlanKey keys[32];
    static ConvPlan plans[32];
    static int used = 0, next = 0;
    PlanKey k;
    std::memset(&k, 0, sizeof(k));
    k = PlanKey{B, H, W, Ic, Oc, R, has_res, sms,
                g.stride, g.Hin, g.Win, g.Ic2, g.stride2, g.Hin2, g.Win2, g.pool, g.Rw,
                g.stride_w};
    {
        std::lock_guard<std::mutex> lk(mu);
        for (int i = 0; i < used; ++i)
            if (keys[i] == k) {
                p = plans[i];
                goto found;
            }
    }
    if (int e = plan_conv_ex(p, B, H, W, Ic, Oc, R, has_res, S, m_r, sms, g))
        return e;
    {
        std::lock_guard<std::mutex> lk(mu);
        keys[next] = k;
        plans[next] = p;
        next = (next + 1) % 32;
        if (used < 32)
            ++used;
    }
found:
    p.S = S;
    p.m_r = m_r;
    p.inject = g_inject.load();
    const unsigned long long lim = g_wait_limit_ns.load();
    p.wait_limit_ns = lim ? lim : kDefaultWaitNs;
    return X1CB_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Every operand must be memory of the current device: the kernels launch on
// the current device, and a pointer into another GPU (or into host memory)
// would be read through a peer or host mapping, or fault.  NULL entries are
// skipped (optional operands).
int check_resident(std::initializer_list<const void *> ptrs)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return X1CB_ERR_CUDA;
    for (const void *q : ptrs) {
        if (!q)
            continue;
        cudaPointerAttributes a;
        if (cudaPointerGetAttributes(&a, q) != cudaSuccess) {
            cudaGetLastError();  // not sticky: clear it for later calls
            return X1CB_ERR_DEVICE;
        }
        if ((a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged) || a.device != dev)
            return X1CB_ERR_DEVICE;
    }
    return X1CB_OK;
}

bool overlap(const void *a, size_t na, const void *b, size_t nb)
{
    if (!a || !b || na == 0 || nb == 0)
        return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}

// Checks shared by the convolution entry points.
int check_conv_shape(int B, int H, int W, int Ic, int Oc, int S)
{
    if (B < 0 || H < 0 || W < 0)
        return X1CB_ERR_SHAPE;
    if (Ic < 32 || Ic % 32 || Ic > 4096 || Oc < 128 || Oc % 128 || Oc > 65536)
        return X1CB_ERR_SHAPE;
    if (S < 1 || S > 60)
        return X1CB_ERR_SHAPE;
    if (static_cast<long long>(H) * W > INT_MAX / 2)
        return X1CB_ERR_SHAPE;
    // every tensor byte offset must stay far below 2^40 (TMA stride limit)
    const long long px = static_cast<long long>(B) * H * W;
    if (px * (Ic > Oc ? Ic : Oc) >= (1LL << 40))
        return X1CB_ERR_SHAPE;
    return X1CB_OK;
}

int conv_common(const int8_t *x, const int8_t *w, const int32_t *bias, const int32_t *m,
                int32_t m_r, int32_t S, const int8_t *r, int8_t *out, int B, int H, int W, int Ic,
                int Oc, int R, void *stream, bool check_ptrs = true)
{
    if (int e = check_conv_shape(B, H, W, Ic, Oc, S))
        return e;
    const size_t px = static_cast<size_t>(B) * H * W;
    if (px == 0)
        return X1CB_OK;  // empty batch or image: nothing to do (pointers may be NULL)
    if (!x || !w || !bias || !m || !out)
        return X1CB_ERR_NULL;
    if (!aligned16(x) || !aligned16(w) || !aligned16(out) || (r && !aligned16(r)) ||
        (reinterpret_cast<uintptr_t>(bias) & 3u) || (reinterpret_cast<uintptr_t>(m) & 3u))
        return X1CB_ERR_ALIGN;
    const size_t out_bytes = px * Oc;
    if (overlap(out, out_bytes, x, px * Ic) || overlap(out, out_bytes, r, r ? px * Oc : 0) ||
        overlap(out, out_bytes, w, static_cast<size_t>(Oc) * Ic * R * R) ||
        overlap(out, out_bytes, bias, Oc * 4u) || overlap(out, out_bytes, m, Oc * 4u))
        return X1CB_ERR_OVERLAP;
    int sms = 0;
    if (int e = device_info(sms))
        return e;
    if (check_ptrs)
        if (int e = check_resident({x, w, bias, m, r, out}))
            return e;
    // The 128 -> 128 3x3 (the bottleneck's Conv2) runs on CTA pairs that
    // share each MMA and hold half the weights each: a deeper halo ring than
    // one SM can keep beside all 144 KB of them.
    if (R == 3 && !r && Ic == 128 && Oc == 128 && g_inject.load() == 0) {
        ChainPlan cp;
        if (plan_conv2_pair(cp, B, H, W, S) == X1CB_OK) {
            const unsigned long long lim = g_wait_limit_ns.load();
            cp.wait_limit_ns = lim ? lim : kDefaultWaitNs;
            return launch_chain(cp, x, w, bias, m, nullptr, nullptr, nullptr, nullptr, out,
                                static_cast<cudaStream_t>(stream));
        }
    }
    ConvPlan p;
    if (int e = get_plan(p, B, H, W, Ic, Oc, R, r != nullptr, S, m_r, sms))
        return e;
    return launch_conv(p, x, w, bias, m, r, out, static_cast<cudaStream_t>(stream));
}

// Convolutions whose input differs from their output grid: stride > 1, and
// optionally a second 1x1 source (the projection shortcut) accumulated into
// the same outputs.  x is [B, Ic/32, Hin, Win, 32]; out is [B, Oc/32, H, W,
// 32] with H, W the convolution's output extent; x2 is [B, Ic2/32, Hin2,
// Win2, 32] read at (stride2*h, stride2*w).
int conv_geom_common(const int8_t *x, const int8_t *w, const int32_t *bias, const int32_t *m,
                     int32_t S, int8_t *out, int B, int Hin, int Win, int Ic, int Oc, int R,
                     int stride, const int8_t *x2, const int8_t *w2, int Ic2, int Hin2,
                     int Win2, int stride2, void *stream, bool check_ptrs = true,
                     bool pool = false, int Rw = 0, int stride_w = 0)
{
    const int pad = (R - 1) / 2;
    const int Rw_ = Rw > 0 ? Rw : R, padw = (Rw_ - 1) / 2;
    const int sw = stride_w > 0 ? stride_w : stride;
    if (Hin < 0 || Win < 0 || stride < 1 || stride > 8 || stride2 < 1 || stride2 > 8)
        return X1CB_ERR_SHAPE;
    const int H = Hin + 2 * pad >= R ? (Hin + 2 * pad - R) / stride + 1 : 0;
    const int W = Win + 2 * padw >= Rw_ ? (Win + 2 * padw - Rw_) / sw + 1 : 0;
    // (a pooled layer has 64 output channels: checked as 128 here, exactly below)
    if (int e = check_conv_shape(B, Hin, Win, Ic, pool ? 128 : Oc, S))
        return e;
    if (pool && Oc != 64)
        return X1CB_ERR_SHAPE;
    if (Ic2) {
        if (Ic2 < 32 || Ic2 % 32 || Ic2 > 4096 || Hin2 < 0 || Win2 < 0)
            return X1CB_ERR_SHAPE;
        if (int e = check_conv_shape(B, Hin2, Win2, Ic2, Oc, S))
            return e;
    }
    const size_t px = static_cast<size_t>(B) * H * W;
    if (px == 0)
        return X1CB_OK;
    // the written output: the pooled image when pooling
    const size_t px_out =
        pool ? static_cast<size_t>(B) * ((H - 1) / 2 + 1) * ((W - 1) / 2 + 1) : px;
    if (Ic2 && ((H - 1) * static_cast<long long>(stride2) >= Hin2 ||
                (W - 1) * static_cast<long long>(stride2) >= Win2))
        return X1CB_ERR_SHAPE;
    if (!x || !w || !bias || !m || !out || (Ic2 && (!x2 || !w2)))
        return X1CB_ERR_NULL;
    if (!aligned16(x) || !aligned16(w) || !aligned16(out) || (x2 && !aligned16(x2)) ||
        (w2 && !aligned16(w2)) || (reinterpret_cast<uintptr_t>(bias) & 3u) ||
        (reinterpret_cast<uintptr_t>(m) & 3u))
        return X1CB_ERR_ALIGN;
    const size_t out_bytes = px_out * Oc;
    const size_t in_bytes = static_cast<size_t>(B) * Hin * Win * Ic;
    const size_t in2_bytes = static_cast<size_t>(B) * Hin2 * Win2 * Ic2;
    if (overlap(out, out_bytes, x, in_bytes) || overlap(out, out_bytes, x2, in2_bytes) ||
        overlap(out, out_bytes, w, static_cast<size_t>(Oc) * Ic * R * Rw_) ||
        overlap(out, out_bytes, w2, static_cast<size_t>(Oc) * Ic2) ||
        overlap(out, out_bytes, bias, Oc * 4u) || overlap(out, out_bytes, m, Oc * 4u))
        return X1CB_ERR_OVERLAP;
    int sms = 0;
    if (int e = device_info(sms))
        return e;
    if (check_ptrs)
        if (int e = check_resident({x, w, bias, m, out, x2, w2}))
            return e;
    // The 128 -> 128 3x3 at stride 2 (the projection block's Conv2) runs on
    // CTA pairs, as at stride 1 (see conv_common).
    if (R == 3 && Rw_ == 3 && stride == 2 && sw == 2 && Ic == 128 && Oc == 128 && !pool &&
        !Ic2 && g_inject.load() == 0) {
        ChainPlan cp;
        if (plan_conv2_pair(cp, B, H, W, S, 2, Hin, Win) == X1CB_OK) {
            const unsigned long long lim = g_wait_limit_ns.load();
            cp.wait_limit_ns = lim ? lim : kDefaultWaitNs;
            return launch_chain(cp, x, w, bias, m, nullptr, nullptr, nullptr, nullptr, out,
                                static_cast<cudaStream_t>(stream));
        }
    }
    ConvGeom g;
    g.stride = stride;
    g.Hin = Hin;
    g.Win = Win;
    g.Ic2 = Ic2;
    g.stride2 = stride2;
    g.Hin2 = Hin2;
    g.Win2 = Win2;
    g.pool = pool ? 1 : 0;
    g.Rw = Rw;
    g.stride_w = stride_w;
    ConvPlan p;
    if (int e = get_plan(p, B, H, W, Ic, Oc, R, 0, S, 0, sms, g))
        return e;
    return launch_conv(p, x, w, bias, m, nullptr, out, static_cast<cudaStream_t>(stream), x2, w2);
}

int device_info_check()
{
    int sms = 0;
    return device_info(sms);
}

}  // namespace

int bottleneck_chain(const int8_t *x, const int8_t *w1, const int32_t *b1, const int32_t *m1,
                     const int8_t *w2, const int32_t *b2, const int32_t *m2, const int8_t *w3,
                     const int32_t *b3, const int32_t *m3, int32_t m_r, int32_t S, int8_t *out,
                     void *workspace, size_t ws_bytes, int B, int H, int W, int Cin, int Cmid,
                     void *stream, bool ws_trusted)
{
    if (int e = check_conv_shape(B, H, W, Cin, Cmid, S))
        return e;
    if (int e = check_conv_shape(B, H, W, Cmid, Cin, S))
        return e;
    if (static_cast<size_t>(B) * H * W == 0)
        return X1CB_OK;
    if (!x || !w1 || !b1 || !m1 || !w2 || !b2 || !m2 || !w3 || !b3 || !m3 || !out)
        return X1CB_ERR_NULL;
    const size_t need = bottleneck_i8_workspace_size(B, H, W, Cmid);
    if (need > 0 && (!workspace || ws_bytes < need))
        return X1CB_ERR_WORKSPACE;
    if (workspace && !aligned16(workspace))
        return X1CB_ERR_ALIGN;
    const size_t px = static_cast<size_t>(B) * H * W;
    if (overlap(out, px * Cin, x, px * Cin) || overlap(workspace, need, x, px * Cin) ||
        overlap(workspace, need, out, px * Cin))
        return X1CB_ERR_OVERLAP;
    if (px == 0)
        return X1CB_OK;
    if (int e = device_info_check())
        return e;
    if (int e = check_resident({x, w1, b1, m1, w2, b2, m2, w3, b3, m3, out}))
        return e;
    if (!ws_trusted)
        if (int e = check_resident({workspace}))
            return e;
    int8_t *y1 = static_cast<int8_t *>(workspace);
    int8_t *y2 = y1 + need / 2;
    // Conv2 -> Conv3 in one kernel where the shape has the fused form: Conv2's
    // output stays on chip and only Conv1's output goes through the workspace.
    ChainPlan cp;
    if (g_block_fusion.load() && plan_chain(cp, B, H, W, Cmid, Cin, S, m_r) == X1CB_OK) {
        if (int e = conv_common(x, w1, b1, m1, 0, S, nullptr, y1, B, H, W, Cin, Cmid, 1, stream,
                                false))
            return e;
        cp.wait_limit_ns = g_wait_limit_ns.load() ? g_wait_limit_ns.load() : kDefaultWaitNs;
        return launch_chain(cp, y1, w2, b2, m2, w3, b3, m3, x, out,
                            static_cast<cudaStream_t>(stream));
    }
    // Operands were checked above; the intermediates are the workspace.
    if (int e = conv_common(x, w1, b1, m1, 0, S, nullptr, y1, B, H, W, Cin, Cmid, 1, stream,
                            false))
        return e;
    if (int e = conv_common(y1, w2, b2, m2, 0, S, nullptr, y2, B, H, W, Cmid, Cmid, 3, stream,
                            false))
        return e;
    return conv_common(y2, w3, b3, m3, m_r, S, x, out, B, H, W, Cmid, Cin, 1, stream, false);
}

}  // namespace x1cb

using namespace x1cb;

extern "C" {

int conv1x1_bn_add_relu_i8(const int8_t *x, const int8_t *w, const int32_t *bias,
                           const int32_t *m, int32_t m_r, int32_t S, const int8_t *r,
                           int8_t *out, int B, int H, int W, int Ic, int Oc, void *stream)
{
    return conv_common(x, w, bias, m, m_r, S, r, out, B, H, W, Ic, Oc, 1, stream);
}

int conv3x3_bn_relu_i8(const int8_t *x, const int8_t *w, const int32_t *bias, const int32_t *m,
                       int32_t S, int8_t *out, int B, int H, int W, int Ic, int Oc, int pad,
                       void *stream)
{
    if (pad != 1)
        return X1CB_ERR_SHAPE;
    return conv_common(x, w, bias, m, 0, S, nullptr, out, B, H, W, Ic, Oc, 3, stream);
}

int conv3x3_conv1x1_bn_add_relu_i8(const int8_t *y1, const int8_t *w2, const int32_t *b2,
                                   const int32_t *m2, const int8_t *w3, const int32_t *b3,
                                   const int32_t *m3, int32_t m_r, int32_t S, const int8_t *r,
                                   int8_t *out, int B, int H, int W, int Cmid, int Cout,
                                   void *stream)
{
    if (int e = check_conv_shape(B, H, W, Cmid, Cout, S))
        return e;
    const size_t px = static_cast<size_t>(B) * H * W;
    if (px == 0)
        return X1CB_OK;
    if (!y1 || !w2 || !b2 || !m2 || !w3 || !b3 || !m3 || !r || !out)
        return X1CB_ERR_NULL;
    if (!aligned16(y1) || !aligned16(w2) || !aligned16(w3) || !aligned16(r) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(b2) & 3u) || (reinterpret_cast<uintptr_t>(m2) & 3u) ||
        (reinterpret_cast<uintptr_t>(b3) & 3u) || (reinterpret_cast<uintptr_t>(m3) & 3u))
        return X1CB_ERR_ALIGN;
    const size_t ob = px * Cout;
    if (overlap(out, ob, y1, px * Cmid) || overlap(out, ob, r, ob) ||
        overlap(out, ob, w2, static_cast<size_t>(Cmid) * Cmid * 9) ||
        overlap(out, ob, w3, static_cast<size_t>(Cout) * Cmid))
        return X1CB_ERR_OVERLAP;
    ChainPlan cp;
    if (int e = plan_chain(cp, B, H, W, Cmid, Cout, S, m_r))
        return e;
    if (int e = device_info_check())
        return e;
    if (int e = check_resident({y1, w2, b2, m2, w3, b3, m3, r, out}))
        return e;
    cp.wait_limit_ns = g_wait_limit_ns.load() ? g_wait_limit_ns.load() : kDefaultWaitNs;
    return launch_chain(cp, y1, w2, b2, m2, w3, b3, m3, r, out, static_cast<cudaStream_t>(stream));
}

int conv3x3s2_bn_relu_i8(const int8_t *x, const int8_t *w, const int32_t *bias,
                         const int32_t *m, int32_t S, int8_t *out, int B, int H, int W, int Ic,
                         int Oc, void *stream)
{
    return conv_geom_common(x, w, bias, m, S, out, B, H, W, Ic, Oc, 3, 2, nullptr, nullptr, 0, 0,
                            0, 1, stream);
}

int conv1x1_proj_bn_relu_i8(const int8_t *y, const int8_t *w3, const int8_t *x,
                            const int8_t *wp, const int32_t *bias, const int32_t *m, int32_t S,
                            int8_t *out, int B, int H, int W, int Cy, int Hx, int Wx, int Cx,
                            int Oc, void *stream)
{
    if (Cx <= 0)
        return X1CB_ERR_SHAPE;
    return conv_geom_common(y, w3, bias, m, S, out, B, H, W, Cy, Oc, 1, 1, x, wp, Cx, Hx, Wx, 2,
                            stream);
}

int conv_bn_relu_maxpool_i8(const int8_t *x, const int8_t *w, const int32_t *bias,
                            const int32_t *m, int32_t S, int8_t *out, int B, int H, int W, int Ic,
                            int Oc, int R, int stride, void *stream)
{
    if ((R != 1 && R != 3 && R != 5 && R != 7) || (stride != 1 && stride != 2))
        return X1CB_ERR_SHAPE;
    return conv_geom_common(x, w, bias, m, S, out, B, H, W, Ic, Oc, R, stride, nullptr, nullptr,
                            0, 0, 0, 1, stream, true, true);
}

int stem_conv_bn_relu_maxpool_i8(const int8_t *folded, const int8_t *wf, const int32_t *bias,
                                 const int32_t *m, int32_t S, int8_t *out, int B, int H, int W,
                                 int R, void *stream)
{
    // R x R stride-2 convolution of the image as an R x 1 convolution of its
    // width-folded form (one 32-channel block per output column: the fold
    // applied the column stride), then pooling.
    if ((R != 1 && R != 3 && R != 5 && R != 7) || W < 0)
        return X1CB_ERR_SHAPE;
    const int pad = (R - 1) / 2;
    const int Wc = W + 2 * pad >= R ? (W + 2 * pad - R) / 2 + 1 : 0;
    return conv_geom_common(folded, wf, bias, m, S, out, B, H, Wc, 32, 64, R, 2, nullptr, nullptr,
                            0, 0, 0, 1, stream, true, true, 1, 1);
}

size_t bottleneck_proj_i8_workspace_size(int B, int H, int W, int Cmid)
{
    if (B < 0 || H < 0 || W < 0 || Cmid < 0)
        return 0;
    const size_t Ho = H > 0 ? (H - 1) / 2 + 1 : 0, Wo = W > 0 ? (W - 1) / 2 + 1 : 0;
    const size_t y1 = static_cast<size_t>(B) * H * W * Cmid;
    const size_t y2 = static_cast<size_t>(B) * Ho * Wo * Cmid;
    return ((y1 + 255) & ~static_cast<size_t>(255)) + ((y2 + 255) & ~static_cast<size_t>(255));
}

int bottleneck_proj_i8(const int8_t *x, const int8_t *w1, const int32_t *b1, const int32_t *m1,
                       const int8_t *w2, const int32_t *b2, const int32_t *m2, const int8_t *w3,
                       const int8_t *wp, const int32_t *b3, const int32_t *m3, int32_t S,
                       int8_t *out, void *workspace, size_t ws_bytes, int B, int H, int W,
                       int Cin, int Cmid, int Cout, void *stream)
{
    if (int e = check_conv_shape(B, H, W, Cin, Cmid, S))
        return e;
    if (int e = check_conv_shape(B, H, W, Cmid, Cout, S))
        return e;
    const int Ho = H > 0 ? (H - 1) / 2 + 1 : 0, Wo = W > 0 ? (W - 1) / 2 + 1 : 0;
    const size_t px_in = static_cast<size_t>(B) * H * W;
    const size_t px_out = static_cast<size_t>(B) * Ho * Wo;
    if (px_in == 0)
        return X1CB_OK;
    if (!x || !w1 || !b1 || !m1 || !w2 || !b2 || !m2 || !w3 || !wp || !b3 || !m3 || !out)
        return X1CB_ERR_NULL;
    const size_t need = bottleneck_proj_i8_workspace_size(B, H, W, Cmid);
    if (!workspace || ws_bytes < need)
        return X1CB_ERR_WORKSPACE;
    if (!aligned16(workspace))
        return X1CB_ERR_ALIGN;
    if (overlap(out, px_out * Cout, x, px_in * Cin) || overlap(workspace, need, x, px_in * Cin) ||
        overlap(workspace, need, out, px_out * Cout))
        return X1CB_ERR_OVERLAP;
    if (int e = device_info_check())
        return e;
    if (int e = check_resident({x, w1, b1, m1, w2, b2, m2, w3, wp, b3, m3, out, workspace}))
        return e;
    int8_t *y1 = static_cast<int8_t *>(workspace);
    int8_t *y2 = y1 + ((px_in * Cmid + 255) & ~static_cast<size_t>(255));
    if (int e = conv_common(x, w1, b1, m1, 0, S, nullptr, y1, B, H, W, Cin, Cmid, 1, stream,
                            false))
        return e;
    if (int e = conv_geom_common(y1, w2, b2, m2, S, y2, B, H, W, Cmid, Cmid, 3, 2, nullptr,
                                 nullptr, 0, 0, 0, 1, stream, false))
        return e;
    return conv_geom_common(y2, w3, b3, m3, S, out, B, Ho, Wo, Cmid, Cout, 1, 1, x, wp, Cin, H, W,
                            2, stream, false);
}

size_t bottleneck_i8_workspace_size(int B, int H, int W, int Cmid)
{
    if (B < 0 || H < 0 || W < 0 || Cmid < 0)
        return 0;
    const size_t mid = static_cast<size_t>(B) * H * W * Cmid;
    return 2 * ((mid + 255) & ~static_cast<size_t>(255));
}

int bottleneck_i8(const int8_t *x, const int8_t *w1, const int32_t *b1, const int32_t *m1,
                  const int8_t *w2, const int32_t *b2, const int32_t *m2, const int8_t *w3,
                  const int32_t *b3, const int32_t *m3, int32_t m_r, int32_t S, int8_t *out,
                  void *workspace, size_t ws_bytes, int B, int H, int W, int Cin, int Cmid,
                  void *stream)
{
    return bottleneck_chain(x, w1, b1, m1, w2, b2, m2, w3, b3, m3, m_r, S, out, workspace,
                            ws_bytes, B, H, W, Cin, Cmid, stream, false);
}
int x1cb_pack_act(const int8_t *nhwc, int8_t *nc32, int B, int H, int W, int C, void *stream)
{
    if (B < 0 || H < 0 || W < 0 || C < 32 || C % 32)
        return X1CB_ERR_SHAPE;
    if (static_cast<size_t>(B) * H * W == 0)
        return X1CB_OK;
    if (!nhwc || !nc32)
        return X1CB_ERR_NULL;
    if (!aligned16(nhwc) || !aligned16(nc32))
        return X1CB_ERR_ALIGN;
    const size_t n = static_cast<size_t>(B) * H * W * C;
    if (overlap(nhwc, n, nc32, n))
        return X1CB_ERR_OVERLAP;
    if (int e = check_resident({nhwc, nc32}))
        return e;
    return launch_pack_act(nhwc, nc32, B, H, W, C, static_cast<cudaStream_t>(stream));
}

int x1cb_unpack_act(const int8_t *nc32, int8_t *nhwc, int B, int H, int W, int C, void *stream)
{
    if (B < 0 || H < 0 || W < 0 || C < 32 || C % 32)
        return X1CB_ERR_SHAPE;
    if (static_cast<size_t>(B) * H * W == 0)
        return X1CB_OK;
    if (!nhwc || !nc32)
        return X1CB_ERR_NULL;
    if (!aligned16(nhwc) || !aligned16(nc32))
        return X1CB_ERR_ALIGN;
    const size_t n = static_cast<size_t>(B) * H * W * C;
    if (overlap(nhwc, n, nc32, n))
        return X1CB_ERR_OVERLAP;
    if (int e = check_resident({nhwc, nc32}))
        return e;
    return launch_unpack_act(nc32, nhwc, B, H, W, C, static_cast<cudaStream_t>(stream));
}

int x1cb_pack_weight(const int8_t *oihw, int8_t *blocked, int Oc, int Ic, int R, void *stream)
{
    if (!oihw || !blocked)
        return X1CB_ERR_NULL;
    if ((Oc != 64 && (Oc < 128 || Oc % 128)) || Ic < 32 || Ic % 32 ||
        (R != 1 && R != 3 && R != 5 && R != 7))
        return X1CB_ERR_SHAPE;
    const size_t n = static_cast<size_t>(Oc) * Ic * R * R;
    if (overlap(oihw, n, blocked, n))
        return X1CB_ERR_OVERLAP;
    if (int e = check_resident({oihw, blocked}))
        return e;
    return launch_pack_weight(oihw, blocked, Oc, Ic, R, static_cast<cudaStream_t>(stream));
}

int x1cb_pack_stem(const int8_t *nhwc, int8_t *folded, int B, int H, int W, int Cin, int R,
                   void *stream)
{
    if (B < 0 || H < 0 || W < 0 || Cin < 1 || (R != 1 && R != 3 && R != 5 && R != 7) ||
        R * Cin > 32)
        return X1CB_ERR_SHAPE;
    const int pad = (R - 1) / 2;
    const int Wc = W + 2 * pad >= R ? (W + 2 * pad - R) / 2 + 1 : 0;
    if (static_cast<size_t>(B) * H * Wc == 0)
        return X1CB_OK;
    if (!nhwc || !folded)
        return X1CB_ERR_NULL;
    if (!aligned16(folded))
        return X1CB_ERR_ALIGN;
    const size_t px = static_cast<size_t>(B) * H * W;
    if (overlap(nhwc, px * Cin, folded, static_cast<size_t>(B) * H * Wc * 32))
        return X1CB_ERR_OVERLAP;
    if (int e = check_resident({nhwc, folded}))
        return e;
    return launch_pack_stem(nhwc, folded, B, H, W, Cin, R, static_cast<cudaStream_t>(stream));
}

int x1cb_pack_stem_weight(const int8_t *oihw, int8_t *blocked, int Oc, int Cin, int R,
                          void *stream)
{
    if (!oihw || !blocked)
        return X1CB_ERR_NULL;
    if (Oc != 64 || Cin < 1 || (R != 1 && R != 3 && R != 5 && R != 7) || R * Cin > 32)
        return X1CB_ERR_SHAPE;
    if (overlap(oihw, static_cast<size_t>(Oc) * Cin * R * R, blocked,
                static_cast<size_t>(R) * Oc * 32))
        return X1CB_ERR_OVERLAP;
    if (int e = check_resident({oihw, blocked}))
        return e;
    return launch_pack_stem_weight(oihw, blocked, Oc, Cin, R, static_cast<cudaStream_t>(stream));
}

const char *x1cb_status_string(int s)
{
    switch (s) {
    case X1CB_OK: return "ok";
    case X1CB_ERR_NULL: return "null pointer";
    case X1CB_ERR_SHAPE: return "unsupported shape or parameter";
    case X1CB_ERR_ALIGN: return "pointer not 16-byte aligned";
    case X1CB_ERR_ARCH: return "no sm_100 device";
    case X1CB_ERR_CUDA: return "CUDA call failed";
    case X1CB_ERR_TIMEOUT: return "kernel wait timed out";
    case X1CB_ERR_WORKSPACE: return "workspace missing or too small";
    case X1CB_ERR_OVERLAP: return "output overlaps an input";
    case X1CB_ERR_DEVICE: return "operand is not memory of the current device";
    default: return "unknown status";
    }
}

int x1cb_last_device_error(unsigned int *bits, int clear)
{
    if (cudaDeviceSynchronize() != cudaSuccess)
        return X1CB_ERR_CUDA;
    const unsigned int v = read_and_clear_dev_status(clear != 0);
    if (cudaGetLastError() != cudaSuccess)
        return X1CB_ERR_CUDA;
    if (bits)
        *bits = v;
    return v ? X1CB_ERR_TIMEOUT : X1CB_OK;
}

int x1cb_last_epilogue_forms(unsigned int *bits, int clear)
{
    if (!bits)
        return X1CB_ERR_NULL;
    if (cudaDeviceSynchronize() != cudaSuccess)
        return X1CB_ERR_CUDA;
    *bits = read_and_clear_dev_forms(clear != 0);
    return cudaGetLastError() == cudaSuccess ? X1CB_OK : X1CB_ERR_CUDA;
}

long long x1cb_trace_copy(unsigned long long *host, long long words, int clear)
{
    if (!host && words > 0)
        return X1CB_ERR_NULL;
    if (cudaDeviceSynchronize() != cudaSuccess)
        return X1CB_ERR_CUDA;
    const long long n = copy_trace(host, words, clear != 0);
    return n < 0 ? X1CB_ERR_CUDA : n;
}

void x1cb_set_block_fusion(int enable) { g_block_fusion.store(enable ? 1 : 0); }

void x1cb_set_wait_limit_ns(unsigned long long ns) { g_wait_limit_ns.store(ns); }

void x1cb_debug_inject(int mode) { g_inject.store(mode); }

int x1cb_describe_plan(int B, int H, int W, int Ic, int Oc, int R, int has_res, char *buf,
                       size_t len)
{
    if (!buf || len == 0)
        return X1CB_ERR_NULL;
    if (int e = check_conv_shape(B, H, W, Ic, Oc, 24))
        return e;
    if (R != 1 && R != 3)
        return X1CB_ERR_SHAPE;
    if (static_cast<long long>(B) * H * W == 0)
        return X1CB_ERR_SHAPE;
    int sms = 148;
    if (device_info(sms) != X1CB_OK)
        sms = 148;  // describe for a B200 when no device is present
    ConvPlan p;
    if (int e = plan_conv(p, B, H, W, Ic, Oc, R, has_res, 24, 0, sms))
        return e;
    std::snprintf(buf, len,
                  "tile=%dx%dx%d rows=%d m_tiles=%d NC=%d groups=%d nmma=%d subs=%d kb=%d "
                  "kc=%d a_stages=%d r_stages=%d fold=%d smem=%d grid=%d halo=%d swz=%d "
                  "wstream=%d mwarps=%d stage_ch=%d cta_pair=%d",
                  p.tw, p.th, p.tg, p.rows, p.num_m_tiles, p.NC, p.n_groups, p.nmma, p.n_subs,
                  p.kb_per_tile, p.a_kc, p.a_stages, p.r_stages, p.fold_room, p.smem_bytes, p.grid,
                  p.halo, p.io_swz, p.wstream, p.n_mma_warps, p.stage_ch, p.pair);
    // The 128 -> 128 3x3 runs on CTA pairs instead (see conv_common): its
    // plan follows the single-CTA one.
    ChainPlan cp;
    if (R == 3 && !has_res && Ic == 128 && Oc == 128 && plan_conv2_pair(cp, B, H, W, 24) == X1CB_OK) {
        const size_t n = std::strlen(buf);
        std::snprintf(buf + n, len - n, " pair=1 pair_tile=%dx%dx%d pair_a_stages=%d "
                      "pair_r_stages=%d pair_smem=%d", cp.tw, cp.th, cp.tg, cp.a_stages,
                      cp.r_stages, cp.smem_bytes);
    }
    return X1CB_OK;
}

int x1cb_describe_plan_ex(int B, int Hin, int Win, int Ic, int Oc, int R, int stride, int Ic2,
                          int has_res, int pool, char *buf, size_t len)
{
    if (!buf || len == 0)
        return X1CB_ERR_NULL;
    if (R != 1 && R != 3 && R != 5 && R != 7)
        return X1CB_ERR_SHAPE;
    if (int e = check_conv_shape(B, Hin, Win, Ic, pool ? 128 : Oc, 24))
        return e;
    const int pad = (R - 1) / 2;
    if (stride < 1 || stride > 8 || Hin + 2 * pad < R || Win + 2 * pad < R || Ic2 < 0 ||
        Ic2 % 32 || (Ic2 && (R != 1 || stride != 1)))
        return X1CB_ERR_SHAPE;
    const int H = (Hin + 2 * pad - R) / stride + 1, W = (Win + 2 * pad - R) / stride + 1;
    if (static_cast<long long>(B) * H * W == 0)
        return X1CB_ERR_SHAPE;
    int sms = 148;
    if (device_info(sms) != X1CB_OK)
        sms = 148;
    ConvGeom g;
    g.stride = stride;
    g.Hin = Hin;
    g.Win = Win;
    if (Ic2) {  // the projection source: the stride-2 1x1 over a 2H x 2W image
        g.Ic2 = Ic2;
        g.stride2 = 2;
        g.Hin2 = 2 * H;
        g.Win2 = 2 * W;
    }
    g.pool = pool ? 1 : 0;
    ConvPlan p;
    if (int e = plan_conv_ex(p, B, H, W, Ic, Oc, R, has_res, 24, 0, sms, g))
        return e;
    std::snprintf(buf, len,
                  "tile=%dx%dx%d rows=%d m_tiles=%d NC=%d groups=%d nmma=%d subs=%d kb=%d "
                  "kc=%d a_stages=%d r_stages=%d fold=%d smem=%d grid=%d halo=%d swz=%d "
                  "out=%dx%d stride=%d kb2=%d wstream=%d pool=%dx%d mwarps=%d stage_ch=%d",
                  p.tw, p.th, p.tg, p.rows, p.num_m_tiles, p.NC, p.n_groups, p.nmma, p.n_subs,
                  p.kb_per_tile, p.a_kc, p.a_stages, p.r_stages, p.fold_room, p.smem_bytes, p.grid,
                  p.halo, p.io_swz, H, W, p.stride, p.C1b, p.wstream, p.pw, p.ph, p.n_mma_warps,
                  p.stage_ch);
    // The 128 -> 128 3x3 at stride 1 or 2 runs on CTA pairs instead.
    ChainPlan cp;
    if (R == 3 && Ic == 128 && Oc == 128 && !Ic2 && !has_res && !pool && stride <= 2 &&
        plan_conv2_pair(cp, B, H, W, 24, stride, Hin, Win) == X1CB_OK) {
        const size_t n = std::strlen(buf);
        std::snprintf(buf + n, len - n, " pair=1 pair_tile=%dx%dx%d pair_a_stages=%d "
                      "pair_r_stages=%d pair_smem=%d", cp.tw, cp.th, cp.tg, cp.a_stages,
                      cp.r_stages, cp.smem_bytes);
    }
    return X1CB_OK;
}

int x1cb_describe_chain(int B, int H, int W, int Cmid, int Cout, char *buf, size_t len)
{
    if (!buf || len == 0)
        return X1CB_ERR_NULL;
    ChainPlan p;
    if (int e = plan_chain(p, B, H, W, Cmid, Cout, 24, 1 << 23))
        return e;
    int clusters = 0;
    if (resident_clusters(p.smem_bytes, clusters) != X1CB_OK)
        clusters = 0;  // no device: the plan alone
    std::snprintf(buf, len,
                  "tile=%dx%dx%d rows=%d m_tiles=%d pairs=%d a_stages=%d r_stages=%d smem=%d "
                  "resident_clusters=%d swz=%d",
                  p.tw, p.th, p.tg, p.rows, p.num_m_tiles, p.n_pairs, p.a_stages, p.r_stages,
                  p.smem_bytes, clusters, p.io_swz);
    return X1CB_OK;
}

const char *x1cb_version(void) { return "x1cb 0.2.0 sm_100a"; }

}  // extern "C"
