// Fused INT8 implicit-GEMM convolution + folded BN (+ shortcut Sum) + ReLU +
// requantisation for sm_100a.
//
// What it computes follows the Inspur MLPerf v2.0 ResNet50 convolution-merge
// article (news.cnblogs.com/n/719672): section 2.2 (Conv3 + Bn + Sum + Relu of
// the Res3.x block, and Conv + Bn + Relu for Conv1/Conv2), section 3.1 (int8
// data in NC/32HW32, blocked weights [O1, I1, O2, I2]), section 3.3 (the 1x1
// convolution is the GEMM out[M,N] = data[M,K] . weight[N,K]^T with M = B*H*W,
// N = Oc, K = Ic), section 3.4 (the shortcut tile is fetched asynchronously
// early and Bn+Sum+Relu runs on the accumulator before the write-back).
//
// How it computes it is designed for B200 rather than taken from the
// article's A100 kernel:
//  * one persistent CTA per SM, 20 warps, warp-specialised:
//      warp 0      TMA producer: weights (once, resident in shared memory) and
//                  the activation slots (a_kc K blocks of 128 rows x 32 bytes,
//                  or for the 3x3 one framed "halo" tile per channel block
//                  that all nine filter taps read at row offsets)
//      warp 1      MMA issuer: tcgen05.mma.kind::i8 into TMEM (int32), owner
//                  of the TMEM allocation; the whole warp runs the loop and
//                  one elected lane issues
//      warp 2      TMA producer of the I/O stages: each 16 KB stage receives a
//                  shortcut tile (128 pixels x 128 channels) long before use
//      warp 3      TMA store of finished I/O stages
//      warps 4-19  epilogue: tcgen05.ld, exact requantisation; each result
//                  byte overwrites the shortcut byte of the same (pixel,
//                  channel) in the stage, which warp 3 then stores whole.
//                  The four warps of a TMEM lane quarter take turns on stages.
//  * a tile is 128 GEMM rows = tw x th pixels of tg images, chosen per shape
//    so that whole TMA boxes cover the image (16 px x 8 images for 28x28 1x1)
//  * I/O stages use the TMA's 128-byte swizzle where the shape allows, so the
//    epilogue's per-pixel 32-byte accesses are free of bank conflicts
//  * TMEM holds 512 int32 columns; the accumulator ring lets the MMA of the
//    next tile run while the epilogue drains the previous one
//  * every wait is bounded (waiting threads sleep on the barrier); on timeout
//    the CTA raises an abort flag, records a status bit, lets in-flight copies
//    and MMAs land, frees TMEM, and exits.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <climits>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "x1cb_internal.h"
#include "x1cb_plan.h"
#include "x1cb_epi.cuh"
#include "x1cb_ptx.cuh"
#include "x1cb_trace.cuh"

namespace x1cb {

// Sticky device status word (timeouts).  Read and cleared by the API.
__device__ unsigned int g_dev_status;
// Epilogue forms chosen since the last clear: bit f set when a CTA ran form f
// (0 generic, 1 64-bit high word, 2 all-32-bit, 3 all-32-bit with the bias in
// the MMA).  Observability for tests and benchmarks; one atomic per CTA.
__device__ unsigned int g_dev_forms;
#ifdef X1CB_TRACE
__device__ unsigned long long g_trace[kTraceWords];
#endif

namespace {

struct Bars {
    uint32_t base;
    int a_stages, r_stages;
    __device__ uint32_t at(int i) const { return base + 8u * static_cast<uint32_t>(i); }
    __device__ uint32_t w_full() const { return at(0); }
    __device__ uint32_t mma_done() const { return at(1); }
    __device__ uint32_t never() const { return at(2); }
    __device__ uint32_t a_full(int s) const { return at(3 + s); }
    __device__ uint32_t a_empty(int s) const { return at(3 + a_stages + s); }
    // I/O stage s: io_full = shortcut landed (or stage free when there is no
    // shortcut), out_ready = every epilogue warp wrote its results,
    // io_empty = the store of the stage has read it.
    __device__ uint32_t io_full(int s) const { return at(3 + 2 * a_stages + s); }
    __device__ uint32_t out_ready(int s) const { return at(3 + 2 * a_stages + r_stages + s); }
    __device__ uint32_t io_empty(int s) const { return at(3 + 2 * a_stages + 2 * r_stages + s); }
    // Accumulator slots: up to 8 (64-column accumulators of a 64-channel layer).
    __device__ uint32_t acc_full(int s) const { return at(3 + 2 * a_stages + 3 * r_stages + s); }
    __device__ uint32_t acc_empty(int s) const
    {
        return at(3 + 2 * a_stages + 3 * r_stages + 8 + s);
    }
    // Pool mode: the four warps of a turn meet here before pooling their tile.
    __device__ uint32_t pool_bar(int turn) const
    {
        return at(3 + 2 * a_stages + 3 * r_stages + 16 + turn);
    }
    // CTA pairs: each CTA arrives on the other's before leaving.
    __device__ uint32_t exit_bar() const { return at(3 + 2 * a_stages + 3 * r_stages + 20); }
    static int count(int a, int r) { return 3 + 2 * a + 3 * r + 16 + 4 + 1; }
};

// A layer with a shortcut is always a plain stride-1 1x1 (the planner and the
// API admit no other): its instantiations (kRes = 1: I/O stages of four
// 32-channel chunks; kRes = 2: of two, for layers whose resident weights leave
// little room for the rings; kRes = 3: four, on pairs of CTAs that share each
// MMA and hold half the weights each) read these plan fields as constants, so
// they carry none of the halo, pooling or second-source code (which cost the
// shortcut layers up to 4 % when it was compiled into them).  kRes = 0: no
// shortcut, every form.
template <int kRes> __device__ __forceinline__ int plan_halo(const ConvPlan &p)
{
    return kRes ? 0 : p.halo;
}
template <int kRes> __device__ __forceinline__ bool plan_pool(const ConvPlan &p)
{
    return !kRes && p.pool;
}
template <int kRes> __device__ __forceinline__ int plan_stage_ch(const ConvPlan &p)
{
    return kRes == 1 || kRes == 3 ? kRChunks : (kRes == 2 ? kRChunks / 2 : p.stage_ch);
}
template <int kRes> __device__ __forceinline__ int plan_c1b(const ConvPlan &p)
{
    return kRes ? 0 : p.C1b;
}
// Bytes between I/O ring slots: a shortcut layer's stages are packed at their
// own size; the others keep 16 KB slots (pooled tiles use the upper half).
template <int kRes> __device__ __forceinline__ int plan_r_slot(const ConvPlan &p)
{
    return kRes ? plan_stage_ch<kRes>(p) * kTileRows * 32 : kRSlotBytes;
}

template <int kRes>
__device__ __forceinline__ void tile_origin(const ConvPlan &p, int mt, int &w0, int &h0, int &b0)
{
    const int iw = mt % p.nTw;
    const int ih = (mt / p.nTw) % p.nTh;
    const int ig = mt / (p.nTw * p.nTh);
    if (plan_pool<kRes>(p)) {  // conv origin of pooled tile (iw, ih): one pixel before 2 * pooled origin
        w0 = 2 * iw * p.pw - 1;
        h0 = 2 * ih * p.ph - 1;
    } else {
        w0 = iw * p.tw;
        h0 = ih * p.th;
    }
    b0 = ig * p.tg;
}

// Ring position of activation box n (boxes counted over the CTA's tiles, bpt
// per tile).  One MMA warp: slot n % a_stages.  Two: the even tiles' boxes
// take the first half of the ring and the odd tiles' the second, each half in
// order, so each half has one consumer that takes its boxes in order (a
// parity wait on a slot is exact only then).
__device__ __forceinline__ void a_ring_pos(const ConvPlan &p, bool split, int n, int bpt,
                                           int &stage, uint32_t &phase)
{
    if (split) {
        const int half = p.a_stages / 2;
        const int t = n / bpt, b = n - t * bpt;
        const int li = (t >> 1) * bpt + b;  // the box's place in its half
        const int q = li / half;
        stage = (t & 1) * half + (li - q * half);
        phase = static_cast<uint32_t>(q & 1);
    } else {
        const int q = n / p.a_stages;
        stage = n - q * p.a_stages;
        phase = static_cast<uint32_t>(q & 1);
    }
}

// Epilogue of one warp.  For every tile of this CTA and every accumulator
// slot it reads its 32 TMEM lanes (= 32 pixels of the tile), two adjacent
// 32-channel chunks per I/O stage, requantises them (with the shortcut bytes
// of the stage) and writes the 32-byte results back into the stage in place.
struct EpiCtx {
    const ConvPlan *p;
    Bars bars;
    WaitCtl ctl;
    uint32_t tmem_base;
    uint8_t *io;
    volatile int *io_ticket;  // I/O stages before this one have been seen to arrive
    const int32_t *cm;
    const long long *cC;
    int group, mt_first, mt_step, mt_end;
};

// kMode: 3 = all-32-bit form with the bias folded into the MMA, 2 = all-32-bit
// form, 1 = 64-bit fast form, 0 = generic.  kK1 (modes 2-3 with a shortcut):
// the shortcut's scale in the all-32-bit form, k = m_r / 2^(S-1), is 1.
//
// The warps of one TMEM lane quarter take turns on the I/O stages: turn g
// handles stages g, g + kTurns, ... (counted over all of the CTA's tiles), all
// four 32-channel chunks of its 32 rows.  Turns drift apart in time, so while
// one warp waits for its stage or its TMEM load the others compute.
//
// A parity wait on an mbarrier is only meaningful when the phase before the
// awaited one is known to be complete.  Accumulator slots: the turns are as
// many as the I/O stages the TMEM holds, so each turn uses one slot and takes
// every phase of it.  I/O slots: before awaiting a stage's arrival a turn
// makes sure the slot's previous stage is complete (see below), so each
// slot's phases are observed in order whatever the ring depth.
template <int kRes, int kMode, bool kK1 = false>
__device__ __forceinline__ void epilogue_warp(const EpiCtx &cx, int warp, int lane)
{
    constexpr int kTurns = kEpiWarps / 4;                 // warps per TMEM lane quarter
    static_assert(kTurns == kTmemCols / (32 * kRChunks),
                  "one turn per I/O stage held in TMEM: each turn owns one accumulator slot");
    // (64-channel layers: stages of two chunks, eight 64-column slots; turn g
    // then owns slots g and g + 4, still seeing each slot's phases in order)
    const ConvPlan &p = *cx.p;
    const int q = warp & 3;                               // TMEM lane quarter this warp may access
    const int turn = (warp - kEpiWarp0) >> 2;
    const int row = q * 32 + lane;                        // GEMM row = pixel of the tile
    const int plane_t = p.tw * p.th;                      // pixels per image in the I/O box
    const int xi = row % p.row_pitch;
    const int yi = (row % p.plane_m) / p.row_pitch;
    const int gi = row / p.plane_m;
    // Rows past the tile, and the halo form's frame columns/rows, are not pixels.
    const bool in_box = xi < p.tw && yi < p.th && gi < p.tg;
    // This row's 32 bytes inside chunk 0 of an I/O stage ([tg][4][th][tw][32]);
    // rows outside the box read row 0's bytes and write nothing.
    const int row_off = in_box ? ((gi * plan_stage_ch<kRes>(p)) * plane_t + yi * p.tw + xi) * 32 : 0;
    const int chunk_stride = plane_t * 32;
    // (o >> 3) & 0x70 is bits 7-9 of o moved to bits 4-6: the 128-byte swizzle.
    const int swz_mask = p.io_swz ? 0x70 : 0;
    const int n_slots = p.n_slots;
    const int chunks_per_sub = p.nmma / 32;
    const int stages_per_sub = chunks_per_sub / plan_stage_ch<kRes>(p);
    const long long my_tiles =
        cx.mt_first < cx.mt_end ? (cx.mt_end - cx.mt_first + cx.mt_step - 1) / cx.mt_step
                                    : 0;
    const long long total = my_tiles * p.n_subs * stages_per_sub;
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    // Shortcut operands.  64-bit fast form: r*2^(8*k8) by one byte permute and
    // m_r*2^(s-8*k8).  All-32-bit form: the sign-extended byte (k8 = 0) and
    // k = m_r / 2^(S-1).
    const int sh = 32 - p.S;
    const int k8 = kMode >= 2 ? 0 : (sh < 0 ? 0 : (sh / 8 < 3 ? sh / 8 : 3));
    const int mr2 =
        kMode == 1 ? static_cast<int>(static_cast<long long>(p.m_r) * (1ll << (sh - 8 * k8)))
                   : (kMode >= 2 ? static_cast<int>(static_cast<long long>(p.m_r) /
                                                    (1ll << (p.S - 1)))
                                 : 0);
    uint32_t rsel[4];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        uint32_t sel = 0;
        for (int i = 0; i < 4; ++i) {
            const uint32_t nib = i < k8 ? 4u : (i == k8 ? static_cast<uint32_t>(b) : 8u | b);
            sel |= nib << (4 * i);
        }
        rsel[b] = sel;
    }
    // Pool mode (64 channels: one stage per tile, so turn g takes tiles g,
    // g + kTurns, ...): the tile coordinates (iw, ih) of this turn's next
    // tile and their step, tracked with carries (image index unused).
    int pool_iw = 0, pool_ih = 0, pool_dw = 0, pool_dh = 0;
    if (plan_pool<kRes>(p)) {
        const int mt0 = cx.mt_first + turn * cx.mt_step;
        pool_iw = mt0 % p.nTw;
        pool_ih = (mt0 / p.nTw) % p.nTh;
        const int d = kTurns * cx.mt_step;
        pool_dw = d % p.nTw;
        pool_dh = (d / p.nTw) % p.nTh;
    }
    // Pool mode: this thread's 16-byte piece of the pooled stage -- piece k
    // (pooled pixel k/2 mod np of chunk k/2/np, K half k&1) of the tile's
    // np * stage_ch * 2, all within the turn's 128 threads (the planner
    // checks) -- as offsets into the stage, the same for every tile.
    int pool_src = -1, pool_dst = 0;
    const int pool_row = p.tw * 32;
    if (plan_pool<kRes>(p)) {
        const int k = q * 32 + lane, np = p.pw * p.ph;
        if (k < np * plan_stage_ch<kRes>(p) * 2) {
            const int half = k & 1, c = (k >> 1) / np, pix = (k >> 1) % np;
            const int pi = pix / p.pw, pj = pix % p.pw;
            pool_src = c * chunk_stride + half * 16 + (2 * pi * p.tw + 2 * pj) * 32;
            pool_dst = kRSlotBytes / 2 + (c * np + pix) * 32 + half * 16;
        }
    }
    // Position of stage n = turn: I/O ring slot and phase, stage within its
    // accumulator slot (rl), N slice (j), accumulator slot and phase.
    int st = turn % p.r_stages;
    uint32_t st_phase = static_cast<uint32_t>((turn / p.r_stages) & 1);
    int rl = turn % stages_per_sub;
    const int sub_n = turn / stages_per_sub;
    int j = sub_n % p.n_subs;
    int acc = sub_n % n_slots;
    uint32_t acc_phase = static_cast<uint32_t>((sub_n / n_slots) & 1);
    uint32_t pool_phase = 0;
    for (long long n = turn; n < total; n += kTurns) {
        // Every lane waits; the vote keeps the decision warp-uniform so the
        // .sync.aligned TMEM loads below always run converged.
        if (!__all_sync(0xffffffffu, mbar_wait(cx.bars.acc_full(acc), acc_phase, cx.ctl,
                                               kDevTimeoutEpilogue)))
            return;
        const bool tr = q == 0 && lane == 0;  // one trace writer per turn
        if (tr)
            X1CB_TRACE_AT(p.trace, 4, n);
        tc_fence_after();
        // Before the parity wait on the slot's arrival, make sure its previous
        // phase (stage n - r_stages, another turn's) is complete.  Ring of at
        // least kTurns stages: wait, as the producer does, until that stage has
        // been stored (exact: stage n - 2*r_stages was stored before this
        // turn's previous stage could be loaded).  Shallower ring: take the
        // arrivals in stage order with the ticket.
        const bool deep = p.r_stages >= kTurns;
        if (deep ? !__all_sync(0xffffffffu, mbar_wait(cx.bars.io_empty(st), st_phase ^ 1u,
                                                      cx.ctl, kDevTimeoutEpilogue))
                 : !__all_sync(0xffffffffu, ticket_wait(cx.io_ticket, static_cast<int>(n),
                                                        cx.ctl, kDevTimeoutEpilogue)))
            return;
        if (!__all_sync(0xffffffffu, mbar_wait(cx.bars.io_full(st), st_phase, cx.ctl,
                                               kDevTimeoutEpilogue)))
            return;
        if (tr)
            X1CB_TRACE_AT(p.trace, 5, n);
        // The four warps of a turn each pass the ticket on; it only moves forward.
        if (!deep && lane == 0)
            atomicMax(const_cast<int *>(cx.io_ticket), static_cast<int>(n + 1));
        const uint32_t tbase = cx.tmem_base + lane_addr + static_cast<uint32_t>(acc * p.nmma);
        uint8_t *stage = cx.io + st * plan_r_slot<kRes>(p);
        bool conv_px = true;  // pool mode: this row is a pixel of the conv output
        if (plan_pool<kRes>(p)) {
            // the tile's conv origin: one pixel before twice its pooled origin
            const int w0 = 2 * pool_iw * p.pw - 1, h0 = 2 * pool_ih * p.ph - 1;
            conv_px = w0 + xi >= 0 && w0 + xi < p.W && h0 + yi >= 0 && h0 + yi < p.H;
            // next stage of this turn: kTurns tiles on (one stage per pooled
            // tile), tile coordinates advanced with carries, no divisions
            pool_iw += pool_dw;
            if (pool_iw >= p.nTw) {
                pool_iw -= p.nTw;
                ++pool_ih;
            }
            pool_ih += pool_dh;
            if (pool_ih >= p.nTh)
                pool_ih -= p.nTh;
        }
#pragma unroll 1
        for (int c = 0; c < plan_stage_ch<kRes>(p); ++c) {
            const int cs = rl * plan_stage_ch<kRes>(p) + c;        // chunk within the TMEM slot
            const int gch = j * chunks_per_sub + cs;   // chunk within the CTA's channels
            uint32_t v[32];
            __syncwarp();
            tmem_ld_32x32b_x32_sync(tbase + static_cast<uint32_t>(cs * 32), v);
            // This pixel's two 16-byte halves (swizzled stages: the 16-byte unit
            // index within each 128-byte row is XORed with the row index).
            const int o = row_off + c * chunk_stride;
            const int sw = swz_mask & (o >> 3);
            uint4 *pa = reinterpret_cast<uint4 *>(stage + (o ^ sw));
            uint4 *pb = reinterpret_cast<uint4 *>(stage + ((o + 16) ^ sw));
            uint32_t rw[8];
            if (kRes) {
                const uint4 ra = *pa, rb = *pb;
                rw[0] = ra.x; rw[1] = ra.y; rw[2] = ra.z; rw[3] = ra.w;
                rw[4] = rb.x; rw[5] = rb.y; rw[6] = rb.z; rw[7] = rb.w;
            }
            uint32_t ow[8];
            if (kMode >= 2) {
                requant_hi32<(kRes != 0), kMode == 2, kK1, 8>(
                    v, cx.cm + gch * 32, reinterpret_cast<const int32_t *>(cx.cC) + gch * 32, rw,
                    mr2, rsel, ow);
            } else if (kMode == 1) {
                requant_fast<(kRes != 0), 8>(v, cx.cm + gch * 32, cx.cC + gch * 32, rw, mr2, rsel, ow);
            } else {
                requant32<(kRes != 0)>(v, cx.cm + gch * 32, cx.cC + gch * 32, rw, p.m_r, p.S, ow);
            }
            if (in_box) {
                if (plan_pool<kRes>(p) && !conv_px)  // outside the conv output: never the maximum
                    ow[0] = ow[1] = ow[2] = ow[3] = ow[4] = ow[5] = ow[6] = ow[7] = 0u;
                *pa = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                *pb = make_uint4(ow[4], ow[5], ow[6], ow[7]);
            }
        }
        if (plan_pool<kRes>(p)) {
            // Every conv pixel of the tile is in the stage once the turn's four
            // warps are here; then each thread pools 16-byte pieces (16 channels)
            // of pooled pixels into the upper half of the stage.
            // (an mbarrier, so that a turn whose wait ran out cannot strand the
            // others: this wait is bounded like every other)
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(cx.bars.pool_bar(turn));
            if (!__all_sync(0xffffffffu, mbar_wait(cx.bars.pool_bar(turn), pool_phase, cx.ctl,
                                                   kDevTimeoutEpilogue)))
                return;
            if (tr)
                X1CB_TRACE_AT(p.trace, 10, n);
            pool_phase ^= 1u;
            if (pool_src >= 0) {  // this thread's piece (offsets fixed per layer)
                const uint8_t *src = stage + pool_src;
                uint4 mx = make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int r = 0; r < 3; ++r)
#pragma unroll
                    for (int t = 0; t < 3; ++t) {
                        const uint4 v =
                            *reinterpret_cast<const uint4 *>(src + r * pool_row + t * 32);
                        mx.x = __vmaxu4(mx.x, v.x);
                        mx.y = __vmaxu4(mx.y, v.y);
                        mx.z = __vmaxu4(mx.z, v.z);
                        mx.w = __vmaxu4(mx.w, v.w);
                    }
                *reinterpret_cast<uint4 *>(stage + pool_dst) = mx;
            }
        }
        // Results must be visible to the TMA store (async proxy).
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (tr)
            X1CB_TRACE_AT(p.trace, 6, n);
        if (lane == 0) {
            mbar_arrive(cx.bars.out_ready(st));
            // one arrival per stage of the slot (CTA pairs: from both CTAs, on
            // rank 0's barrier, which its MMA warp waits on)
            if (kRes == 3)
                mbar_arrive_cluster(mapa_shared(cx.bars.acc_empty(acc), 0));
            else
                mbar_arrive(cx.bars.acc_empty(acc));
        }
        st += kTurns;
        while (st >= p.r_stages) {
            st -= p.r_stages;
            st_phase ^= 1u;
        }
        rl += kTurns;
        while (rl >= stages_per_sub) {
            rl -= stages_per_sub;
            if (++j == p.n_subs)
                j = 0;
            if (++acc == n_slots) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    }
}

// MMA-side operations of one CTA or of a CTA pair (rank 0 issues M = 256
// MMAs over both CTAs' operands; its waits see the other CTA's arrivals with
// cluster scope, its commits arrive on both CTAs' barriers).
template <bool kPair>
__device__ __forceinline__ bool mma_wait(uint32_t bar, uint32_t parity, const WaitCtl &ctl,
                                         unsigned int code)
{
    return kPair ? mbar_wait_cl(bar, parity, ctl, code) : mbar_wait(bar, parity, ctl, code);
}
template <bool kPair>
__device__ __forceinline__ void mma_issue(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                          uint32_t accumulate)
{
    if (kPair)
        mma_i8_pair(d, a, b, idesc, accumulate);
    else
        mma_i8(d, a, b, idesc, accumulate);
}
template <bool kPair> __device__ __forceinline__ void mma_commit_to(uint32_t bar)
{
    if (kPair)
        mma_commit_pair(bar);
    else
        mma_commit(bar);
}

// kSplit: two MMA warps (warp 2 issues MMAs; no shortcut), a separate
// instantiation so that the one-issuer kernels keep their code as it was.
template <int kRes, bool kSplit>
__global__ void __launch_bounds__(kThreads, 1)
    conv_bn_act_kernel(const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmW,
                       const __grid_constant__ CUtensorMap tmR,
                       const __grid_constant__ CUtensorMap tmO,
                       const __grid_constant__ CUtensorMap tmA2,
                       const __grid_constant__ CUtensorMap tmW2,
                       const int32_t *__restrict__ bias, const int32_t *__restrict__ mult,
                       const ConvPlan p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    long long *cC = reinterpret_cast<long long *>(smem + p.off_cc);
    int32_t *cm = reinterpret_cast<int32_t *>(smem + p.off_cm);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + p.off_misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + p.off_misc + 4);
    volatile int *io_ticket = reinterpret_cast<volatile int *>(smem + p.off_misc + 8);
    Bars bars{sbase + static_cast<uint32_t>(p.off_bar), p.a_stages, p.r_stages};
    // With the test hook armed, the MMA warp's planted wait has the limit and
    // every other wait four times it, so the planted one is the wait that runs
    // out and the others leave on the abort flag.
    const WaitCtl ctl{abort_flag, &g_dev_status,
                      p.inject == 1 ? 4 * p.wait_limit_ns : p.wait_limit_ns};
    const uint64_t drain_ns = 200000000ull;  // 0.2 s for copies/MMAs already issued

    // CTA pairs (kRes = 3): cluster c = blockIdx.x / 2 takes channel group
    // c % n_groups and pair tiles pt = c / n_groups + k * (clusters per group);
    // rank r of the pair takes m-tile 2 pt + r (past the last tile: zeros
    // loaded, nothing stored), so both ranks run the same number of tiles.
    constexpr bool kPair = kRes == 3;
    const uint32_t rank = kPair ? cluster_ctarank() : 0u;
    const bool leader = rank == 0;
    const int unit = kPair ? static_cast<int>(blockIdx.x / 2) : static_cast<int>(blockIdx.x);
    const int units = kPair ? static_cast<int>(gridDim.x / 2) : static_cast<int>(gridDim.x);
    const int group = unit % p.n_groups;
    const int mt_first = kPair ? 2 * (unit / p.n_groups) + static_cast<int>(rank)
                               : unit / p.n_groups;
    const int mt_step = kPair ? 2 * (units / p.n_groups) : units / p.n_groups;
    const int mt_end = kPair ? (p.num_m_tiles + 1) & ~1 : p.num_m_tiles;
    const int stages_per_tile = p.NC / (32 * plan_stage_ch<kRes>(p));

    // ---- set-up ---------------------------------------------------------------
    // Trace events (trace builds): 0 producer box n may load; 1 MMA sees box n;
    // 2 MMA has slot for sub-tile n; 3 MMA committed sub-tile n; 4 epilogue
    // sees the accumulator of I/O stage n; 5 ... its shortcut; 6 ... is done;
    // 7 store warp sees stage n; 8 stage n's store has read it; 9 I/O
    // producer issues stage n; 10 pool turn met for stage n; 15: start, end.
    if (threadIdx.x == 0)
        X1CB_TRACE_AT(p.trace, 15, 0);
    if (threadIdx.x == 0) {
        *abort_flag = 0;
        *io_ticket = 0;
        mbar_init(bars.w_full(), 1);
        mbar_init(bars.mma_done(), kSplit ? 2 : 1);  // each MMA warp's final commit
        mbar_init(bars.never(), 1);
        for (int s = 0; s < p.a_stages; ++s) {
            mbar_init(bars.a_full(s), 1);
            mbar_init(bars.a_empty(s), 1);
        }
        for (int s = 0; s < p.r_stages; ++s) {
            mbar_init(bars.io_full(s), 1);
            mbar_init(bars.out_ready(s), 4);  // one warp per TMEM lane quarter
            mbar_init(bars.io_empty(s), 1);
        }
        for (int t = 0; t < 4; ++t)
            mbar_init(bars.pool_bar(t), 4);
        for (int s = 0; s < 8; ++s) {
            mbar_init(bars.acc_full(s), 1);
            // every stage of the slot, each from one warp per lane quarter (of
            // both CTAs of a pair)
            mbar_init(bars.acc_empty(s),
                      (kPair ? 8 : 4) * (p.nmma / (32 * plan_stage_ch<kRes>(p))));
        }
        mbar_init(bars.exit_bar(), 1);
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmW);
        tma_prefetch_desc(&tmO);
        if (kRes)
            tma_prefetch_desc(&tmR);
        if (plan_c1b<kRes>(p)) {
            tma_prefetch_desc(&tmA2);
            tma_prefetch_desc(&tmW2);
        }
    }
    // Launched as a dependent of the preceding kernel (programmatic dependent
    // launch), this CTA may start while that kernel drains: everything above
    // touches only shared memory and the kernel parameters; from here on the
    // kernel reads and writes global memory, so it waits for the preceding
    // grid to complete.
    griddep_wait();
    // Folded-BN constants of this CTA's channels.  Generic form:
    // C = bias*m + 2^(S-1), so that t = acc*m + C (+ r*m_r) is one wide
    // multiply-add per term.  Fast form (when exact for every channel of the
    // CTA): m' = m*2^(32-S), C' = bias*m' + 2^31 (see requant_fast).
    // All-32-bit form (see requant_hi32): m'' = m*2^(33-S) and bias as int32.
    const int K = p.kb_per_tile * kKBlock;
    bool my_fast = true, my_hi = true;
    for (int n = threadIdx.x; n < p.NC; n += blockDim.x) {
        const int o = group * p.NC + n;
        my_fast = my_fast && fast_form_ok(mult[o], bias[o], p.m_r, p.S, K, kRes);
        my_hi = my_hi && hi32_ok(mult[o], bias[o], p.S, K);
    }
    bool my_fold = p.fold_room != 0;
    for (int n = threadIdx.x; n < p.NC; n += blockDim.x) {
        const int b = bias[group * p.NC + n];
        my_fold = my_fold && b <= kBiasFoldMax && b >= -kBiasFoldMax;
    }
    const bool all_fast = __syncthreads_and(my_fast ? 1 : 0) != 0;
    const bool all_hi = __syncthreads_and(my_hi ? 1 : 0) != 0 && hi32_layer_ok(p.m_r, p.S, kRes);
    const bool fold = __syncthreads_and(my_fold ? 1 : 0) != 0 && all_hi;
    const int mode = all_hi ? (fold ? 3 : 2) : (all_fast ? 1 : 0);
    if (threadIdx.x == 0)
        atomicOr(&g_dev_forms, 1u << mode);
    if (fold) {
        // constant A tile (every row [1, 127 x 15, 1, 127 x 15]) and digit rows
        uint4 *ta = reinterpret_cast<uint4 *>(smem + p.off_ba);
        for (int i = threadIdx.x; i < kTileRows * 2; i += blockDim.x)
            ta[i] = make_uint4(0x7F7F7F01u, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
        // (CTA pairs: this CTA's half of the B rows, channels rank * NC/2 on)
        const int nb = kPair ? p.NC / 2 : p.NC;
        for (int n = threadIdx.x; n < nb; n += blockDim.x) {
            uint32_t w[8];
            bias_digits(bias[group * p.NC + static_cast<int>(rank) * nb + n], w);
            uint4 *tb = reinterpret_cast<uint4 *>(smem + p.off_bb + n * 32);
            tb[0] = make_uint4(w[0], w[1], w[2], w[3]);
            tb[1] = make_uint4(w[4], w[5], w[6], w[7]);
        }
        fence_proxy_async_smem();  // the MMA reads these through the async proxy
    }
    int32_t *cb = reinterpret_cast<int32_t *>(cC);  // bias, in the all-32-bit form
    for (int n = threadIdx.x; n < p.NC; n += blockDim.x) {
        const int o = group * p.NC + n;
        const long long mm = mult[o];
        if (mode == 3) {
            cm[n] = static_cast<int32_t>(mm * (1ll << (33 - p.S)));  // bias is in the MMA
        } else if (mode == 2) {
            cm[n] = static_cast<int32_t>(mm * (1ll << (33 - p.S)));
            cb[n] = bias[o];
        } else if (mode == 1) {
            const long long mp = mm * (1ll << (32 - p.S));
            cm[n] = static_cast<int32_t>(mp);
            cC[n] = static_cast<long long>(bias[o]) * mp + (1ll << 31);
        } else {
            cm[n] = static_cast<int32_t>(mm);
            cC[n] = static_cast<long long>(bias[o]) * mm + (1ll << (p.S - 1));
        }
    }
    if (warp == 1) {
        if (kPair) {
            tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_u32(tmem_slot), kTmemCols);
            tmem_relinquish();
        }
        tc_fence_before();
    }
    __syncthreads();
    if (kPair)  // both CTAs' barriers and TMEM exist before traffic crosses
        cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ---- producer: resident weights, then activation K blocks ---------------
        // One thread issues a tensor copy only every several hundred cycles, so
        // n_iss lanes issue in rounds: in round j lane l takes box
        // n = j*n_iss + l (boxes counted over the CTA's tiles); the lanes wait
        // for their slots together (mbar_wait_lanes) and issue as one.  A
        // round waits for n_iss consecutive slots, so n_iss is at most half
        // the ring; and each slot barrier's parity stays unambiguous because
        // a lane's wait for box n follows the round that saw box n - 1 - S
        // consumed, with the MMA consuming in order.
        const int n_iss = max(1, min(kAIssuers, p.a_stages / 2));
        if (lane == 0) {
            const uint32_t sw = sbase + p.off_w;
            const int o1 = group * (p.NC / p.O2);  // weight block of this CTA's channels
            if (kPair) {
                // this CTA's half of each K block (output channels rank * NC/2
                // on), both halves completing on rank 0's barrier
                const int half_nc = p.NC / 2;
                const uint32_t wbytes = static_cast<uint32_t>(p.kb_per_tile * half_nc * 32);
                if (leader)
                    mbar_arrive_expect_tx(bars.w_full(), 2 * wbytes);
                const uint32_t wfull0 = mapa_shared(bars.w_full(), 0);
                for (int kb = 0; kb < p.kb_per_tile; ++kb)
                    tma2_load_4d(sw + kb * half_nc * 32, &tmW, wfull0, 0, 0, kb,
                                 o1 + static_cast<int>(rank));
            } else if (!p.wstream) {
                const uint32_t wbytes = static_cast<uint32_t>(p.kb_per_tile * p.NC * 32);
                mbar_arrive_expect_tx(bars.w_full(), wbytes);
                // The second source's weights (if any) follow the first's K blocks.
                for (int kb = 0; kb < p.kb_per_tile; ++kb) {
                    if (kb < p.kb_a)
                        tma_load_4d(sw + kb * p.NC * 32, &tmW, bars.w_full(), 0, 0, kb, o1);
                    else
                        tma_load_4d(sw + kb * p.NC * 32, &tmW2, bars.w_full(), 0, 0,
                                    kb - p.kb_a, o1);
                }
            } else {
                mbar_arrive(bars.w_full());  // weights travel with the activation stages
            }
        }
        __syncwarp();
        const unsigned iss_mask = (1u << n_iss) - 1;  // the issuing lanes
        if (lane < n_iss) {
            const int o1 = group * (p.NC / p.O2);
            // Streamed weights: bytes per stage, each K block NC rows x 32 bytes.
            const uint32_t wpart = static_cast<uint32_t>(p.w_part);
            const uint32_t wkb = static_cast<uint32_t>(p.NC * 32);
            // One box = a_kc consecutive K blocks (channel blocks c1..c1+a_kc-1 of
            // one filter tap), each a 128-row x 32-byte tile, back to back.
            const uint32_t abytes =
                plan_halo<kRes>(p) == 3 ? static_cast<uint32_t>((2 * p.th + p.R - 2) * p.tw * 32)
                : plan_halo<kRes>(p)    ? static_cast<uint32_t>((plan_halo<kRes>(p) == 2 ? 8 : 2) * 16 * p.plane_m * p.tg)
                            : static_cast<uint32_t>(p.a_kc * p.rows * 32);  // K halves / blocks
            const uint32_t sa = sbase + p.off_a;
            const uint64_t pol = policy_evict_first();
            // Boxes per tile: halo form one per channel block; else K blocks run
            // channel block fastest, then filter column, then filter row, then
            // (if present) the second source's channel blocks.
            const int cb = p.C1 / p.a_kc;
            const int first_boxes = plan_halo<kRes>(p) ? p.C1 : p.R * p.Rw * cb;
            const int bpt = plan_halo<kRes>(p) ? p.C1 : p.kb_per_tile / p.a_kc;
            const long long my_tiles =
                mt_first < mt_end ? (mt_end - mt_first + mt_step - 1) / mt_step : 0;
            const long long total = my_tiles * bpt;
            long long issued = 0;
            // This lane's box n = base + lane as ring stage/phase and as (tile i,
            // box b of the tile), advanced by counters (n_iss <= a_stages / 2:
            // at most one wrap of the ring per round).
            // This lane's box n = base + lane: tile i, box b of the tile, and the
            // ring position of the next box of each half (one half: the whole
            // ring), all advanced by counters over the n_iss boxes of a round
            // (see a_ring_pos; no divisions on the issue path).
            constexpr bool split = kSplit;
            const int half = split ? p.a_stages / 2 : p.a_stages;
            int i = 0, b = 0, pos0 = 0, pos1 = 0;
            uint32_t ph0 = 0u, ph1 = 0u;
            if (!split) {
                pos0 = lane < n_iss ? lane : 0;
                i = lane / bpt;
                b = lane % bpt;
            } else {
                for (int k = 0; k < lane && k < n_iss; ++k) {  // past box (i, b)
                    if (i & 1) {
                        if (++pos1 == half) {
                            pos1 = 0;
                            ph1 ^= 1u;
                        }
                    } else if (++pos0 == half) {
                        pos0 = 0;
                        ph0 ^= 1u;
                    }
                    if (++b == bpt) {
                        b = 0;
                        ++i;
                    }
                }
            }
            for (long long base = 0; base < total; base += n_iss) {
                const long long n = base + lane;
                const bool have = lane < n_iss && n < total;
                const bool odd = split && (i & 1);
                const int stage = odd ? half + pos1 : pos0;
                const uint32_t phase = odd ? ph1 : ph0;
                if (!mbar_wait_lanes(iss_mask, have, bars.a_empty(stage), phase ^ 1u, ctl,
                                     kDevTimeoutProducer))
                    break;
                if (have) {
                    X1CB_TRACE_AT(p.trace, 0, n);
                    const int mt = mt_first + i * mt_step;
                    int w0, h0, b0;
                    tile_origin<kRes>(p, mt, w0, h0, b0);
                    const uint32_t slot = sa + static_cast<uint32_t>(stage) * p.a_slot;
                    if (kPair) {
                        // this CTA's tile, completing on rank 0's barrier (which
                        // expects both CTAs' boxes)
                        if (leader)
                            mbar_arrive_expect_tx(bars.a_full(stage), 2 * abytes);
                        tma2_load_5d_hint(slot, &tmA, mapa_shared(bars.a_full(stage), 0), 0, w0,
                                          h0, b0, b * p.a_kc, pol);
                    } else {
                    mbar_arrive_expect_tx(bars.a_full(stage), abytes + wpart);
                    if (plan_halo<kRes>(p) == 2) {
                        // one slot per channel block c1 = b: plane (pr, pc) from
                        // input (pc - 1, 2*h0 - 1 + pr), step 2
                        for (int pl = 0; pl < 4; ++pl)
                            for (int hf = 0; hf < 2; ++hf)
                                tma_load_5d_hint(
                                    slot + static_cast<uint32_t>((2 * pl + hf) * p.a_half), &tmA,
                                    bars.a_full(stage), 16 * hf, (pl & 1) - 1,
                                    2 * h0 - 1 + (pl >> 1), b, b0, pol);
                    } else if (plan_halo<kRes>(p) == 3) {
                        // the tile's columns, input rows from 2*h0 - pad on (output
                        // row y, tap dr reads input row 2y - pad + dr)
                        tma_load_5d_hint(slot, &tmA, bars.a_full(stage), 0, w0, 2 * h0 - p.pad,
                                         b0, 0, pol);
                    } else if (plan_halo<kRes>(p)) {
                        // the tile's pixels plus a one-pixel frame (zeros outside the
                        // image), each K half as one box
                        tma_load_5d_hint(slot, &tmA, bars.a_full(stage), 0, w0 - p.pad,
                                         h0 - p.pad, b, b0, pol);
                        tma_load_5d_hint(slot + static_cast<uint32_t>(p.a_half), &tmA,
                                         bars.a_full(stage), 16, w0 - p.pad, h0 - p.pad, b, b0,
                                         pol);
                    } else if (b < first_boxes) {
                        // output pixel (w0, h0) reads input (w0*stride + ds - pad, ...);
                        // a strided map steps `stride` input pixels per loaded pixel
                        const int c1 = (b % cb) * p.a_kc;
                        const int tap = b / cb;
                        const int ds = tap % p.Rw, dr = tap / p.Rw;
                        tma_load_5d_hint(slot, &tmA, bars.a_full(stage), 0,
                                         w0 * p.stride - p.padw + ds, h0 * p.stride - p.pad + dr,
                                         b0, c1, pol);
                    } else {
                        tma_load_5d_hint(slot, &tmA2, bars.a_full(stage), 0, w0 * p.stride2,
                                         h0 * p.stride2, b0, (b - first_boxes) * p.a_kc, pol);
                    }
                    if (wpart) {  // the box's K blocks' weights
                        const uint32_t wdst = slot + static_cast<uint32_t>(p.a_part);
                        if (plan_halo<kRes>(p)) {  // the nine taps of channel block b
                            for (int t = 0; t < 9; ++t)
                                tma_load_4d(wdst + t * wkb, &tmW, bars.a_full(stage), 0, 0,
                                            t * p.C1 + b, o1);
                        } else if (b < first_boxes) {
                            const int kb0 = (b / cb) * p.C1 + (b % cb) * p.a_kc;
                            for (int i = 0; i < p.a_kc; ++i)
                                tma_load_4d(wdst + i * wkb, &tmW, bars.a_full(stage), 0, 0,
                                            kb0 + i, o1);
                        } else {
                            const int kb0 = (b - first_boxes) * p.a_kc;
                            for (int i = 0; i < p.a_kc; ++i)
                                tma_load_4d(wdst + i * wkb, &tmW2, bars.a_full(stage), 0, 0,
                                            kb0 + i, o1);
                        }
                    }
                    }  // (not a pair)
                }
                issued = base + n_iss < total ? base + n_iss : total;
                if (!split) {  // (n_iss <= a_stages / 2: at most one wrap)
                    pos0 += n_iss;
                    if (pos0 >= half) {
                        pos0 -= half;
                        ph0 ^= 1u;
                    }
                    for (b += n_iss; b >= bpt; b -= bpt)
                        ++i;
                } else {
                    for (int k = 0; k < n_iss; ++k) {  // past box (i, b)
                        if (i & 1) {
                            if (++pos1 == half) {
                                pos1 = 0;
                                ph1 ^= 1u;
                            }
                        } else if (++pos0 == half) {
                            pos0 = 0;
                            ph0 ^= 1u;
                        }
                        if (++b == bpt) {
                            b = 0;
                            ++i;
                        }
                    }
                }
            }
            // Let every copy still in flight land before shared memory goes away.
            // (CTA pairs: both CTAs' copies complete on rank 0's barriers, and the
            // exit handshake holds rank 1 until rank 0 has drained them.)
            __syncwarp(iss_mask);
            if (lane == 0 && leader) {
                if (!mbar_drain(bars.w_full(), 0, drain_ns))
                    atomicOr(&g_dev_status, kDevDrainFailed);
                // The latest box of every slot: the last a_stages boxes of one
                // ring; for a split ring, walking back until every slot was seen
                // (the walk and its divisions run once, on the way out).
                const unsigned long long all_slots = (1ull << p.a_stages) - 1;
                unsigned long long seen = 0;
                const int n_issued = static_cast<int>(issued);
                const int stop = split ? 0 : (n_issued > p.a_stages ? n_issued - p.a_stages : 0);
                for (int i = n_issued - 1; i >= stop && seen != all_slots; --i) {
                    int s;
                    uint32_t ph;
                    a_ring_pos(p, split, i, bpt, s, ph);
                    if (seen >> s & 1ull)
                        continue;
                    seen |= 1ull << s;
                    if (!mbar_drain(bars.a_full(s), ph, drain_ns))
                        atomicOr(&g_dev_status, kDevDrainFailed);
                }
            }
        }
        __syncwarp();
    } else if (warp == 2 && !kSplit) {
        // ---- producer of I/O stages: shortcut tiles, issued as early as the ring
        // allows; without a shortcut it only hands out free stages ----------------
        if (lane == 0) {
            const uint32_t rbytes = static_cast<uint32_t>(plan_stage_ch<kRes>(p) * p.rows * 32);
            const uint32_t sio = sbase + p.off_r;
            const uint64_t pol = policy_evict_first();
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            [[maybe_unused]] long long n_io = 0;  // stages handed out (trace index)
            bool ok = true;
            for (int mt = mt_first; ok && mt < mt_end; mt += mt_step) {
                int w0, h0, b0;
                tile_origin<kRes>(p, mt, w0, h0, b0);
                for (int rs = 0; rs < stages_per_tile; ++rs) {
                    if (!mbar_wait(bars.io_empty(stage), phase ^ 1u, ctl, kDevTimeoutProducer)) {
                        ok = false;
                        break;
                    }
                    X1CB_TRACE_AT(p.trace, 9, n_io);
                    ++n_io;
                    if (kRes) {
                        mbar_arrive_expect_tx(bars.io_full(stage), rbytes);
                        const int o1 = group * (p.NC / 32) + rs * plan_stage_ch<kRes>(p);
                        if (p.io_swz)
                            tma_load_5d_hint(sio + stage * plan_r_slot<kRes>(p), &tmR, bars.io_full(stage),
                                             0, w0 / 4, h0, o1, b0, pol);
                        else if (p.io_wide)
                            tma_load_4d_hint(sio + stage * plan_r_slot<kRes>(p), &tmR, bars.io_full(stage),
                                             w0 * 4, h0, o1, b0, pol);
                        else
                            tma_load_5d_hint(sio + stage * plan_r_slot<kRes>(p), &tmR, bars.io_full(stage),
                                             0, w0, h0, o1, b0, pol);
                        ++issued;
                    } else {
                        mbar_arrive(bars.io_full(stage));
                    }
                    if (++stage == p.r_stages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            const long long last = issued < p.r_stages ? issued : p.r_stages;
            for (long long i = issued - last; i < issued; ++i) {
                const int s = static_cast<int>(i % p.r_stages);
                const uint32_t ph = static_cast<uint32_t>((i / p.r_stages) & 1);
                if (!mbar_drain(bars.io_full(s), ph, drain_ns))
                    atomicOr(&g_dev_status, kDevDrainFailed);
            }
        }
        __syncwarp();
    } else if (warp == 3) {
        // ---- TMA store of finished I/O stages ----------------------------------------
        // Each stage goes back to the producer as soon as its store has read it
        // (the global writes complete in the background).  With warp 2 issuing
        // MMAs (no shortcut), this warp also hands the stages out: a stage's
        // next use may start (io_full) once its store has read it, and every
        // stage's first use at once.
        constexpr bool hand_out = kSplit;
        if (lane == 0) {
            const uint32_t sio = sbase + p.off_r;
            const uint64_t pol = policy_evict_first();
            int stage = 0;
            uint32_t phase = 0;
            if (hand_out)
                for (int s = 0; s < p.r_stages; ++s)
                    mbar_arrive(bars.io_full(s));
            [[maybe_unused]] long long n_st = 0;  // stages stored (trace index)
            bool ok = true;
            for (int mt = mt_first; ok && mt < mt_end; mt += mt_step) {
                int w0, h0, b0;
                tile_origin<kRes>(p, mt, w0, h0, b0);
                for (int rs = 0; rs < stages_per_tile; ++rs) {
                    if (!mbar_wait(bars.out_ready(stage), phase, ctl, kDevTimeoutProducer)) {
                        ok = false;
                        break;
                    }
                    X1CB_TRACE_AT(p.trace, 7, n_st);
                    const int o1 = group * (p.NC / 32) + rs * plan_stage_ch<kRes>(p);
                    if (kPair && mt >= p.num_m_tiles) {
                        // (a pair's tile past the last one: nothing to store)
                    } else if (plan_pool<kRes>(p))  // pooled tile at pooled coordinates ((w0 + 1) / 2, ...)
                        tma_store_5d_hint(&tmO, sio + stage * kRSlotBytes + kRSlotBytes / 2, 0,
                                          (w0 + 1) / 2, (h0 + 1) / 2, o1, b0, pol);
                    else if (p.io_swz)
                        tma_store_5d_hint(&tmO, sio + stage * plan_r_slot<kRes>(p), 0, w0 / 4, h0, o1, b0,
                                          pol);
                    else if (p.io_wide)
                        tma_store_4d_hint(&tmO, sio + stage * plan_r_slot<kRes>(p), w0 * 4, h0, o1, b0, pol);
                    else
                        tma_store_5d_hint(&tmO, sio + stage * plan_r_slot<kRes>(p), 0, w0, h0, o1, b0, pol);
                    if (!kPair || mt < p.num_m_tiles) {
                        bulk_commit();
                        bulk_wait_read<0>();
                    }
                    X1CB_TRACE_AT(p.trace, 8, n_st);
                    ++n_st;
                    mbar_arrive(bars.io_empty(stage));
                    if (hand_out)
                        mbar_arrive(bars.io_full(stage));
                    if (++stage == p.r_stages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // Every store must have finished (read and written) before exit.
            bulk_wait_all();
        }
        __syncwarp();
    } else if (warp == 1 || (kSplit && warp == 2)) {
        // ---- MMA issuers (warp 2 only when it has no shortcut to load) -------------
        // The whole warp runs the loop (waits are warp votes, so it stays
        // converged) and one elected lane issues each MMA and commit.  With two
        // issuing warps, warp 1 takes the CTA's even tiles and warp 2 the odd
        // ones, each stepping its ring and slot counters over the other's tiles.
        const int mw = warp == 1 ? 0 : 1;
        if (!kPair || leader) {  // (CTA pairs: rank 0 issues every MMA, M = 256)
            // The issue loop is kept free of divisions and descriptor rebuilds:
            // the dependent integer work between two MMAs would otherwise cost
            // more than the MMA itself (64-128 tensor cycles).  A descriptor's
            // start-address field is the byte address / 16 and every operand
            // lies below 256 KB, so moving an operand by `b` bytes is adding
            // b / 16 to its descriptor.
            const uint32_t idesc = idesc_i8(kPair ? 2 * kTileRows : kTileRows, p.nmma);
            // (folded stem: output row y reads input row 2y + dr, two input rows
            // of tw 32-byte pixels per GEMM row group)
            const uint64_t a_desc0 =
                plan_halo<kRes>(p) == 3 ? smem_desc_sw32(sbase + p.off_a, static_cast<uint32_t>(2 * p.tw * 32))
                : plan_halo<kRes>(p)    ? smem_desc_rows16(sbase + p.off_a, static_cast<uint32_t>(p.a_half))
                            : smem_desc_sw32(sbase + p.off_a);
            const uint32_t h3_row_step = static_cast<uint32_t>(p.tw * 32) >> 4;  // next tap
            const uint64_t b_desc0 = smem_desc_sw32(sbase + p.off_w);
            // Streamed weights: each ring stage carries its K blocks' weights
            // right after its activation part (same 32-byte swizzle layout as the
            // resident weights), so the stage's weight descriptor is the first
            // stage's plus the stage offset.
            const uint64_t w_desc0 = smem_desc_sw32(sbase + p.off_a + p.a_part);
            const uint64_t fold_a = smem_desc_sw32(sbase + p.off_ba);
            const uint64_t fold_b0 = smem_desc_sw32(sbase + p.off_bb);
            const uint32_t a_sub_step = static_cast<uint32_t>(p.rows * 32) >> 4;  // next K block in a box
            const uint32_t a_slot_step = static_cast<uint32_t>(p.a_slot) >> 4;
            // next K block of weights (CTA pairs: each CTA holds NC/2 rows of it)
            const uint32_t b_kb_step = static_cast<uint32_t>((kPair ? p.NC / 2 : p.NC) * 32) >> 4;
            const uint32_t b_sub_step = static_cast<uint32_t>(p.nmma * 32) >> 4;  // next N slice
            const int boxes = plan_halo<kRes>(p) ? p.C1 : p.kb_per_tile / p.a_kc;
            const int kc = p.a_kc;
            // Halo form: tap (dr, ds) reads the slot dr*row_pitch + ds rows on and
            // the weights of K block (dr*3 + ds)*C1 + c1.
            const uint32_t hp = static_cast<uint32_t>(p.row_pitch);
            // Descriptor offset of tap t (units of 16 bytes): the row shift of the
            // framed tile; in the stride-2 form also the tap's plane.
            uint32_t tap_off[9];
#pragma unroll
            for (int t = 0; t < 9; ++t) {
                const uint32_t dr = t / 3, ds = t % 3;
                tap_off[t] = plan_halo<kRes>(p) == 2
                                 ? ((dr & 1) * 2 + (ds & 1)) * (2 * p.a_half >> 4) +
                                       (dr >> 1) * hp + (ds >> 1)
                                 : dr * hp + ds;
            }
            // (streamed: the nine taps of one channel block are consecutive)
            const uint64_t b_tap_step =
                p.wstream ? b_kb_step : static_cast<uint64_t>(p.C1) * b_kb_step;
            const int n_slots = p.n_slots;
            // This warp's part of the activation ring: all of it, or with two MMA
            // warps its half (see a_ring_pos), taken in order.
            const int ring_len = kSplit ? p.a_stages / 2 : p.a_stages;
            const int ring_begin = mw * ring_len, ring_end = ring_begin + ring_len;
            const uint64_t ring_desc0 = a_desc0 + static_cast<uint64_t>(ring_begin) * a_slot_step;
            int a_stage = ring_begin;
            uint32_t a_phase = 0;
            uint64_t a_slot_desc = ring_desc0;
            int acc = 0;
            uint32_t acc_phase = 0;
            [[maybe_unused]] long long n_box = 0, n_sub = 0;  // trace indices
            bool ok = __all_sync(0xffffffffu, mma_wait<kPair>(bars.w_full(), 0, ctl, kDevTimeoutMma));
            if (ok && p.inject == 1 && mw == 0) {
                const WaitCtl planted{abort_flag, &g_dev_status, p.wait_limit_ns};
                ok = __all_sync(0xffffffffu,  // test hook
                                mbar_wait(bars.never(), 0, planted, kDevTimeoutMma));
            }
            int tile = 0;  // the CTA's tile count
            for (int mt = mt_first; ok && mt < mt_end; mt += mt_step, ++tile) {
                if (kSplit && (tile & 1) != mw) {
                    // the other issuer's tile (its boxes are in the other half of
                    // the ring): its accumulator slots
                    for (acc += p.n_subs; acc >= n_slots; acc -= n_slots)
                        acc_phase ^= 1u;
                    n_box += boxes;
                    n_sub += p.n_subs;
                    continue;
                }
                int st = a_stage;
                uint32_t ph = a_phase;
                uint64_t sd = a_slot_desc;
                for (int j = 0; ok && j < p.n_subs; ++j) {
                    if (!__all_sync(0xffffffffu, mma_wait<kPair>(bars.acc_empty(acc), acc_phase ^ 1u,
                                                           ctl, kDevTimeoutMma))) {
                        ok = false;
                        break;
                    }
                    if (lane == 0)
                        X1CB_TRACE_AT(p.trace, 2, n_sub);
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * p.nmma);
                    const bool last_sub = j == p.n_subs - 1;
                    st = a_stage;
                    ph = a_phase;
                    sd = a_slot_desc;
                    uint64_t bd = b_desc0 + static_cast<uint64_t>(j) * b_sub_step;
                    uint32_t accumulate = 0;
                    for (int box = 0; box < boxes; ++box) {
                        // The slot was written by TMA and is read by the MMA, both in the
                        // async proxy; the barrier's transaction count orders them.
                        if (j == 0 && !__all_sync(0xffffffffu, mma_wait<kPair>(bars.a_full(st), ph, ctl,
                                                                         kDevTimeoutMma))) {
                            ok = false;
                            break;
                        }
                        if (j == 0) {
                            if (lane == 0)
                                X1CB_TRACE_AT(p.trace, 1, n_box);
                            ++n_box;
                        }
                        uint64_t ad = sd;
                        if (p.wstream)  // this stage's own weights (one N slice: j == 0)
                            bd = w_desc0 + (sd - a_desc0);
                        if (plan_halo<kRes>(p) == 3) {
                            // filter row dr: the slot dr input rows on, weight K block dr
                            for (int dr = 0; dr < p.R; ++dr)
                                mma_issue<kPair>(d_tmem, ad + static_cast<uint64_t>(dr) * h3_row_step,
                                       bd + static_cast<uint64_t>(dr) * b_kb_step, idesc,
                                       dr == 0 ? accumulate : 1u);
                            bd += static_cast<uint64_t>(p.R) * b_kb_step;
                        } else if (plan_halo<kRes>(p)) {
#pragma unroll
                            for (int t = 0; t < 9; ++t)
                                mma_issue<kPair>(d_tmem, ad + tap_off[t],
                                       bd + static_cast<uint64_t>(t) * b_tap_step, idesc,
                                       t == 0 ? accumulate : 1u);
                            bd += b_kb_step;
                        } else if (kc == 4) {
                            mma_issue<kPair>(d_tmem, ad, bd, idesc, accumulate);
                            mma_issue<kPair>(d_tmem, ad + a_sub_step, bd + b_kb_step, idesc, 1u);
                            mma_issue<kPair>(d_tmem, ad + 2 * a_sub_step, bd + 2 * b_kb_step, idesc, 1u);
                            mma_issue<kPair>(d_tmem, ad + 3 * a_sub_step, bd + 3 * b_kb_step, idesc, 1u);
                            bd += 4 * b_kb_step;
                        } else if (kc == 2) {
                            mma_issue<kPair>(d_tmem, ad, bd, idesc, accumulate);
                            mma_issue<kPair>(d_tmem, ad + a_sub_step, bd + b_kb_step, idesc, 1u);
                            bd += 2 * b_kb_step;
                        } else {
                            mma_issue<kPair>(d_tmem, ad, bd, idesc, accumulate);
                            bd += b_kb_step;
                        }
                        accumulate = 1u;
                        if (last_sub)
                            mma_commit_to<kPair>(bars.a_empty(st));  // slot free once these MMAs finish
                        if (++st == ring_end) {
                            st = ring_begin;
                            ph ^= 1u;
                            sd = ring_desc0;
                        } else {
                            sd += a_slot_step;
                        }
                    }
                    if (!ok)
                        break;
                    if (fold)  // + bias: constant A tile x digit rows of this slot's channels
                        mma_issue<kPair>(d_tmem, fold_a, fold_b0 + static_cast<uint64_t>(j) * b_sub_step,
                               idesc, 1u);
                    mma_commit_to<kPair>(bars.acc_full(acc));
                    if (lane == 0)
                        X1CB_TRACE_AT(p.trace, 3, n_sub);
                    ++n_sub;
                    if (++acc == n_slots) {
                        acc = 0;
                        acc_phase ^= 1u;
                    }
                }
                a_stage = st;
                a_phase = ph;
                a_slot_desc = sd;
            }
            // Make sure no MMA is still reading shared memory or writing TMEM.
            mma_commit_to<kPair>(bars.mma_done());
            if (lane == 0 && !mbar_drain(bars.mma_done(), 0, drain_ns))
                atomicOr(&g_dev_status, kDevDrainFailed);
        }
        __syncwarp();
    } else {
        // ---- epilogue ---------------------------------------------------------------
        const EpiCtx cx{&p, bars, ctl, tmem_base, smem + p.off_r, io_ticket, cm, cC,
                        group, mt_first, mt_step, mt_end};
        const bool k1 = kRes && static_cast<long long>(p.m_r) == (1ll << (p.S - 1));
        if (mode == 3 && k1)
            epilogue_warp<kRes, 3, (kRes != 0)>(cx, warp, lane);
        else if (mode == 3)
            epilogue_warp<kRes, 3>(cx, warp, lane);
        else if (mode == 2 && k1)
            epilogue_warp<kRes, 2, (kRes != 0)>(cx, warp, lane);
        else if (mode == 2)
            epilogue_warp<kRes, 2>(cx, warp, lane);
        else if (mode == 1)
            epilogue_warp<kRes, 1>(cx, warp, lane);
        else
            epilogue_warp<kRes, 0>(cx, warp, lane);
        __syncwarp();
    }

    // ---- tear-down ---------------------------------------------------------------
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0)
        X1CB_TRACE_AT(p.trace, 15, 1);
    if (kPair) {
        // neither CTA of a pair leaves while the other may still reach it (its
        // copies complete on rank 0's barriers, its arrivals cross over)
        if (threadIdx.x == 0) {
            mbar_arrive_cluster(mapa_shared(bars.exit_bar(), rank ^ 1u));
            if (!mbar_drain(bars.exit_bar(), 0, 2 * p.wait_limit_ns + drain_ns))
                atomicOr(&g_dev_status, kDevDrainFailed);
        }
        __syncthreads();
    }
    if (warp == 1) {
        tc_fence_after();
        if (kPair)
            tmem_dealloc_pair(tmem_base, kTmemCols);
        else
            tmem_dealloc(tmem_base, kTmemCols);
    }
}

}  // namespace

// ---- host side --------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 get_encode()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// elem_strides (optional): the traversal step per dimension; a box of
// n * step elements along a strided dimension loads n of them.
int encode_map(CUtensorMap *m, const void *base, int rank, const uint64_t *dims,
               const uint64_t *strides_bytes, const uint32_t *box, CUtensorMapSwizzle swz,
               CUtensorMapDataType dtype, const uint32_t *elem_strides)
{
    auto fn = get_encode();
    if (!fn)
        return X1CB_ERR_CUDA;
    cuuint64_t d[5];
    cuuint64_t s[4];
    cuuint32_t bx[5], es[5];
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        bx[i] = box[i];
        es[i] = elem_strides ? elem_strides[i] : 1;
    }
    for (int i = 0; i < rank - 1; ++i)
        s[i] = strides_bytes[i];
    CUresult r = fn(m, dtype, static_cast<cuuint32_t>(rank),
                    const_cast<void *>(base), d, s, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? X1CB_OK : X1CB_ERR_CUDA;
}

// Function attributes are per device: the dynamic shared-memory opt-in is set
// once for every (device, kernel) pair, under a lock, before the first launch
// of that kernel on that device.
int opt_in_smem(const void *kern, int which)
{
    constexpr int kMaxDev = 64, kKinds = 8;
    static std::mutex mu;
    static bool done[kMaxDev][kKinds] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev || which < 0 ||
        which >= kKinds)
        return X1CB_ERR_CUDA;
    std::lock_guard<std::mutex> lk(mu);
    if (!done[dev][which]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit) !=
            cudaSuccess)
            return X1CB_ERR_CUDA;
        done[dev][which] = true;
    }
    return X1CB_OK;
}


// Choose the pixel tile: tw x th pixels of tg images, at most 128 GEMM rows,
// for a layer of kb K blocks per tile.
// Cost = MMA rows issued over the whole problem, with a penalty for
// contiguous global runs shorter than 512 bytes (up to 47 % for single
// 32-byte pixels); for a row count that is not a multiple of 8 (activation
// boxes then carry one K block each instead of up to four: 10 %, or 35 % for
// more than 4 K blocks per tile, where the box count sets the pace -- measured
// on the 7x7 512 -> 2048 expand conv: 88 us with 125-row tiles of 16 boxes,
// 58 us with 120-row tiles of 4); and 10 % for shortcut/output stages that
// cannot use the 128-byte swizzle (tw or the row not whole 4-pixel groups:
// bank conflicts in the epilogue); ties go to more rows, then to longer runs.
void choose_tile(int B, int Wp, int Hp, int kb, int &tw, int &th, int &tg)
{
    double best = 1e300;
    int best_rows = 0, best_seg = 0;
    tw = th = tg = 1;
    const int max_w = std::min(Wp, kTileRows);
    for (int w = 1; w <= max_w; ++w) {
        const int max_h = std::min(Hp, kTileRows / w);
        for (int h = 1; h <= max_h; ++h) {
            const int g = std::min(kTileRows / (w * h), B);
            const double tiles = static_cast<double>((Wp + w - 1) / w) * ((Hp + h - 1) / h) *
                                 ((B + g - 1) / g);
            const int seg = (w == Wp) ? w * h * 32 : w * 32;
            double cost = tiles * kTileRows;
            if (seg < 512)
                cost *= 1.0 + (512 - seg) / 1024.0;
            const int rows = w * h * g;
            if (rows % 8 != 0)
                cost *= kb > 4 ? 1.35 : 1.1;
            if (w % 4 != 0 || Wp % 4 != 0)
                cost *= 1.1;
            const bool tie = cost <= best * (1 + 1e-12) && cost >= best * (1 - 1e-12);
            if (cost < best * (1 - 1e-12) ||
                (tie && (rows > best_rows || (rows == best_rows && seg > best_seg)))) {
                best_seg = seg;
                best = cost;
                best_rows = rows;
                tw = w;
                th = h;
                tg = g;
            }
        }
    }
}

// Halo form of the 3x3 convolution: th rows of tg images per tile, each image
// row with its one-pixel frame taking W+2 GEMM rows and each image th+2 rows
// of them.  Every pixel of the tile must land in the 128 GEMM rows; fewest
// tiles wins, ties go to taller tiles (longer contiguous runs).
void choose_halo_tile(int B, int H, int W, int &th, int &tg)
{
    const int pitch = W + 2;
    long long best = -1;
    th = tg = 1;
    for (int h = 1; h <= H; ++h) {
        for (int g = 1; g <= B; ++g) {
            const long long last = static_cast<long long>(g - 1) * (h + 2) * pitch +
                                   static_cast<long long>(h - 1) * pitch + (W - 1);
            if (last >= kTileRows)
                break;
            const long long tiles = static_cast<long long>((H + h - 1) / h) * ((B + g - 1) / g);
            if (best < 0 || tiles < best || (tiles == best && h > th)) {
                best = tiles;
                th = h;
                tg = g;
            }
        }
    }
}

int plan_conv(ConvPlan &p, int B, int H, int W, int Ic, int Oc, int R, int has_res, int S,
              int m_r, int num_sms)
{
    return plan_conv_ex(p, B, H, W, Ic, Oc, R, has_res, S, m_r, num_sms, ConvGeom{});
}

int plan_conv_ex(ConvPlan &p, int B, int H, int W, int Ic, int Oc, int R, int has_res, int S,
                 int m_r, int num_sms, const ConvGeom &g)
{
    std::memset(&p, 0, sizeof(p));
    p.B = B;
    p.H = H;
    p.W = W;
    p.Ic = Ic;
    p.Oc = Oc;
    p.R = R;
    p.pad = (R - 1) / 2;
    // Filter width: R (square), or 1 for a column filter over a width-folded
    // image (each pixel already holds its row's taps in its channels).
    p.Rw = g.Rw > 0 ? g.Rw : R;
    p.padw = (p.Rw - 1) / 2;
    p.C1 = Ic / 32;
    p.O1 = Oc / 32;
    p.has_res = has_res;
    p.S = S;
    p.m_r = m_r;
    p.stride = g.stride < 1 ? 1 : g.stride;
    p.stride_w = g.stride_w > 0 ? g.stride_w : p.stride;
    p.Hin = g.Hin ? g.Hin : H;
    p.Win = g.Win ? g.Win : W;
    p.C1b = g.Ic2 / 32;
    p.stride2 = g.stride2 < 1 ? 1 : g.stride2;
    p.Hin2 = g.Hin2;
    p.Win2 = g.Win2;
    if (p.stride > 8 || p.stride_w > 8 || p.stride2 > 8 || g.Ic2 % 32 || g.Ic2 < 0)
        return X1CB_ERR_SHAPE;  // the TMA's traversal step is at most 8
    // Every tapped input pixel must exist for some output: (H-1)*stride + R - 1
    // - pad < Hin + pad, and the output extent is the convolution's.
    if ((p.Hin + 2 * p.pad - R) / p.stride + 1 != H ||
        (p.Win + 2 * p.padw - p.Rw) / p.stride_w + 1 != W)
        return X1CB_ERR_SHAPE;
    // Column strides other than the row stride exist only for the folded stem.
    if (p.stride_w != p.stride && !(g.pool && p.Rw == 1 && p.stride_w == 1 && p.stride == 2))
        return X1CB_ERR_SHAPE;
    if (p.C1b && ((H - 1) * p.stride2 >= p.Hin2 || (W - 1) * p.stride2 >= p.Win2))
        return X1CB_ERR_SHAPE;
    p.pool = g.pool ? 1 : 0;
    if (p.pool && (Oc != 64 || has_res || p.C1b))
        return X1CB_ERR_SHAPE;  // pooled tiles use the upper half of 64-channel stages
    p.Hpo = p.pool ? (H - 1) / 2 + 1 : 0;
    p.Wpo = p.pool ? (W - 1) / 2 + 1 : 0;
    // A stride-1 1x1 without a second source sees the image as one row of H*W
    // pixels (tiles may span image rows); otherwise tiles are 2-D.
    const bool flat = R == 1 && p.stride == 1 && p.C1b == 0 && !p.pool;
    if (flat) {
        p.Wp = H * W;
        p.Hp = 1;
        p.Wpi = H * W;
        p.Hpi = 1;
    } else {
        p.Wp = W;
        p.Hp = H;
        p.Wpi = p.Win;
        p.Hpi = p.Hin;
    }
    // The 3x3 convolution uses the halo form whenever one framed image row fits
    // in the 128 GEMM rows: at stride 1 one framed tile (halo = 1); at stride 2
    // four phase planes of the input region (halo = 2): plane (pr, pc) holds
    // the input pixels of row parity pr and column parity pc, so output pixel
    // (y, x) reads tap (dr, ds) at plane (dr & 1, ds & 1), position
    // (y + dr / 2, x + ds / 2) -- again a row shift of one framed tile.
    p.halo = (R == 3 && p.Rw == 3 && p.C1b == 0 && !p.pool &&
              ((p.stride == 1 && W + 2 <= kTileRows) || (p.stride == 2 && W + 1 <= 126)))
                 ? p.stride
                 : 0;
    // The folded stem (column filter, rows at stride 2, columns at stride 1,
    // one channel block, pooled): one slot of input rows per tile (halo = 3).
    if (p.pool && p.Rw == 1 && p.stride == 2 && p.stride_w == 1 && p.C1 == 1 && p.C1b == 0)
        p.halo = 3;
    if (p.halo == 2) {
        // th output rows of tg images per tile; a plane is (th+1) x (W+1)
        // pixels (row pitch W+1); GEMM row m = (g*(th+1) + y)*(W+1) + x.
        const int pitch = W + 1;
        long long best = -1;
        p.th = p.tg = 1;
        for (int h = 1; h <= H; ++h)
            for (int g = 1; g <= B; ++g) {
                const long long last = static_cast<long long>(g - 1) * (h + 1) * pitch +
                                       static_cast<long long>(h - 1) * pitch + (W - 1);
                if (last >= kTileRows)
                    break;
                const long long tiles = static_cast<long long>((H + h - 1) / h) * ((B + g - 1) / g);
                if (best < 0 || tiles < best || (tiles == best && h > p.th)) {
                    best = tiles;
                    p.th = h;
                    p.tg = g;
                }
            }
        p.tw = W;
        p.row_pitch = pitch;
        p.plane_m = (p.th + 1) * pitch;
        const int need_rows = std::max(p.tg * p.plane_m, kTileRows + pitch + 1);
        p.a_half = ((need_rows + 7) / 8) * 8 * 16;
    } else if (p.halo == 3) {
        // 8 x 16 conv pixels (GEMM row m = y*8 + x) pooled to 3 x 7: conv
        // columns 0-6 and rows 0-14 of the tile feed the pooled pixels.
        p.tw = 8;
        p.th = 16;
        p.tg = 1;
        p.pw = 3;
        p.ph = 7;
        p.row_pitch = p.tw;
        p.plane_m = p.tw * p.th;
        p.a_half = 0;
    } else if (p.halo) {
        choose_halo_tile(B, H, W, p.th, p.tg);
        p.tw = W;
        p.row_pitch = W + 2;
        p.plane_m = (p.th + 2) * (W + 2);
        // Slot rows: the framed tile, and every row a shifted 128-row view can
        // touch (rows past the frame only feed GEMM rows that are not pixels).
        const int need_rows = std::max(p.tg * p.plane_m, kTileRows + 2 * p.row_pitch + 2);
        p.a_half = ((need_rows + 7) / 8) * 8 * 16;
    } else if (p.pool) {
        // pw x ph pooled pixels per tile, (2pw+1) x (2ph+1) conv pixels: fewest
        // tiles, ties to more pooled pixels per tile.
        long long best = -1;
        for (int pw = 1; 2 * pw + 1 <= kTileRows; ++pw)
            for (int ph = 1; (2 * pw + 1) * (2 * ph + 1) <= kTileRows; ++ph) {
                const long long t = static_cast<long long>((p.Wpo + pw - 1) / pw) *
                                    ((p.Hpo + ph - 1) / ph);
                if (best < 0 || t < best || (t == best && pw * ph > p.pw * p.ph)) {
                    best = t;
                    p.pw = pw;
                    p.ph = ph;
                }
            }
        p.tw = 2 * p.pw + 1;
        p.th = 2 * p.ph + 1;
        p.tg = 1;
        p.row_pitch = p.tw;
        p.plane_m = p.tw * p.th;
        p.a_half = 0;
    } else {
        choose_tile(B, p.Wp, p.Hp, R * p.Rw * p.C1 + p.C1b, p.tw, p.th, p.tg);
        p.row_pitch = p.tw;
        p.plane_m = p.tw * p.th;
        p.a_half = 0;
    }
    p.rows = p.tw * p.th * p.tg;
    // pooled tiles (64 channels: stages of two chunks): every 16-byte piece of
    // the pooled stage is one epilogue thread's (a turn has 128)
    if (p.pool && p.pw * p.ph * (Oc / 32) * 2 > 128)
        return X1CB_ERR_SHAPE;
    p.nTw = p.pool ? (p.Wpo + p.pw - 1) / p.pw : (p.Wp + p.tw - 1) / p.tw;
    p.nTh = p.pool ? (p.Hpo + p.ph - 1) / p.ph : (p.Hp + p.th - 1) / p.th;
    p.nTg = (B + p.tg - 1) / p.tg;
    const long long mtiles = static_cast<long long>(p.nTw) * p.nTh * p.nTg;
    if (mtiles > INT_MAX / 2)
        return X1CB_ERR_SHAPE;
    p.num_m_tiles = static_cast<int>(mtiles);
    p.kb_a = R * p.Rw * p.C1;
    p.kb_per_tile = p.kb_a + p.C1b;

    const int fixed = 1024 /*alignment slack*/ + 64 /*misc*/ + Bars::count(48, 12) * 8 + 64;
    // (halo = 3: 2*th + R - 2 input rows of tw 32-byte pixels)
    const int h3_bytes = (2 * p.th + R - 2) * p.tw * 32;
    const int min_slot = p.halo == 3   ? (h3_bytes + 1023) / 1024 * 1024
                         : p.halo      ? (p.halo == 2 ? 8 : 2) * p.a_half
                                       : kASlotBytes;
    int chosen = 0;
    long long chosen_work = -1;
    // A 64-channel layer (the stem) is one CTA group of N = 64.  Largest NC
    // first: the activation is read once per group, and N = 256 MMAs do twice
    // the work of N = 128 ones per instruction.  (Measured: the 7x7, 512 ->
    // 2048 expand conv ran 75 us with NC = 256 and a 5-slot ring, 136 us with
    // NC = 128 and a 22-slot ring -- the ring depth does not pay for the
    // halved MMAs and doubled re-reads.)
    for (int NC = std::min(Oc, 512); NC >= 64; NC -= (NC > 128 ? 128 : 64)) {
        const int nmma = NC >= 256 ? 256 : (NC >= 128 ? 128 : 64);
        // (a group must be whole MMAs: no 384-channel groups of one N = 256 MMA)
        if (Oc % NC || (NC == 64 && Oc != 64) || NC % nmma)
            continue;
        const int n_subs = NC / nmma;
        const int a_min = n_subs > 1 ? (p.halo ? p.C1 : p.kb_per_tile) + 2 : (p.halo ? 2 : 4);
        const int r_min = has_res ? 4 : 2;
        const long long need = static_cast<long long>(p.kb_per_tile) * NC * 32 + NC * 12 +
                               static_cast<long long>(a_min) * min_slot + r_min * kRSlotBytes +
                               fixed;
        if (need > kSmemLimit || a_min > 48)
            continue;
        const long long work = mtiles * (Oc / NC);
        if (chosen == 0 || (chosen_work < num_sms && work > chosen_work)) {
            chosen = NC;
            chosen_work = work;
        }
        if (work >= num_sms)
            break;
    }
    // When no resident copy fits (large fan-in), the weights are streamed:
    // 128 output channels per CTA, each ring stage bringing its K blocks'
    // weights from L2 next to its activations.
    p.wstream = chosen == 0 ? 1 : 0;
    if (p.wstream && p.halo == 3)
        return X1CB_ERR_SHAPE;
    if (p.wstream)
        chosen = Oc == 64 ? 64 : 128;
    p.NC = chosen;
    p.n_groups = Oc / p.NC;
    p.nmma = p.NC >= 256 ? 256 : (p.NC >= 128 ? 128 : 64);
    p.n_subs = p.NC / p.nmma;
    p.O2 = Oc < 128 ? Oc : 128;
    p.stage_ch = p.NC >= 128 ? kRChunks : p.NC / 32;
    p.n_slots = kTmemCols / p.nmma;

    // A shortcut layer whose resident weights take more than 96 KB runs on CTA
    // pairs when its group is one N = 256 MMA (each CTA then holds half the
    // weights); otherwise it stages its shortcut and result in 8 KB pieces
    // (two 32-channel chunks), so that four stages stay in flight beside an
    // activation ring of whole 16 KB boxes.  (Measured on the 7x7 512 -> 2048
    // expand conv, 128 KB of weights: with 16 KB stages only two fit beside
    // the activation boxes.)
    const int full_wbytes = p.wstream ? 0 : p.kb_per_tile * p.NC * 32;
    p.pair = (has_res && full_wbytes > 96 * 1024 && p.NC == 256 && p.n_subs == 1)
                 ? 1
                 : 0;
    const int wbytes = p.pair ? full_wbytes / 2 : full_wbytes;
    if (has_res && !p.pair && wbytes > 96 * 1024)
        p.stage_ch = kRChunks / 2;
    const int r_slot = has_res ? p.stage_ch * kTileRows * 32 : kRSlotBytes;
    // The activation ring budget: with a shortcut the I/O ring (shortcut in,
    // result out) needs the space -- its depth sets the bytes in flight -- so
    // about two tiles' K blocks plus two; without one the activations are most
    // of the traffic and get up to 112 KB in flight while the I/O stages only
    // stage results.  The bias-fold tiles are reserved when the rings still
    // reach their minimum beside them.
    // (Measured on the 1x1 128 -> 512 with shortcut, B = 2048: 326 us with
    // 24 KB of activation ring and seven I/O stages, 314 us with 40 KB and
    // six, 329 us with 40 KB and five.  A deep fan-in with a shortcut -- 8 or
    // more K blocks per tile -- gets two tiles of K blocks.  Without a
    // shortcut, 1x1 512 -> 128 at B = 1024: 107.4 us with six 16 KB boxes,
    // 104.4 with seven; 256 -> 128 at 56x56, B = 256: 72.1 us with four,
    // 65.7 with seven.)
    const int a_bytes_want =
        p.wstream ? 4 * 4 * kASlotBytes
        : !has_res ? 28 * kASlotBytes
        : p.kb_per_tile < 8 ? std::min(2 * p.kb_per_tile + 2, 10) * kASlotBytes
                            : std::min(2 * p.kb_per_tile, 24) * kASlotBytes;
    // Several K blocks per activation box (fewer, larger copies) when each
    // K-block tile starts on a 256-byte swizzle atom (row count a multiple of
    // 8) and the budget holds one box more than the ring's minimum.  With two
    // accumulator slots per tile the whole tile's K blocks stay in the ring
    // until the second slot's MMAs are done.  (Measured on the 1x1 128 -> 512
    // with shortcut: two 16 KB boxes, each a whole tile, 380 us against 314
    // with five 8 KB boxes.)
    auto ring_min = [&](int kc) { return p.n_subs > 1 ? p.kb_per_tile / kc + 1 : 2; };
    int kc_first = 1;
    if (!p.halo)
        for (int kc = 4; kc > 1; kc /= 2)
            if (p.C1 % kc == 0 && p.C1b % kc == 0 && p.rows % 8 == 0 &&
                (ring_min(kc) + 1) * kc * kASlotBytes <= a_bytes_want) {
                kc_first = kc;
                break;
            }
    const int r_lo = has_res ? 4 : 2, r_hi = has_res ? 12 : 4;
    auto layout = [&](int fold, int a, int r) {
        p.fold_room = fold;
        p.a_stages = a;
        p.r_stages = r;
        p.off_w = 0;
        p.off_ba = p.off_w + wbytes;
        p.off_bb = p.off_ba + (fold ? kTileRows * 32 : 0);
        p.off_a = p.off_bb + (fold ? (p.pair ? p.NC / 2 : p.NC) * 32 : 0);
        p.off_r = p.off_a + a * p.a_slot;
        // The per-channel bias/offset table (modes 0-2) and the fold digit rows
        // (mode 3) are never used together, so they share space when folding
        // is possible.
        p.off_cc = fold ? p.off_bb : p.off_r + r * r_slot;
        p.off_cm = (fold ? p.off_r + r * r_slot : p.off_cc + p.NC * 8);
        p.off_bar = (p.off_cm + p.NC * 4 + 7) & ~7;
        p.off_misc = p.off_bar + Bars::count(a, r) * 8;
        p.smem_bytes = p.off_misc + 16 + 1024;  // + alignment slack of the base
        return p.smem_bytes <= kSmemLimit;
    };
    // Largest box first; fewer K blocks per box when its ring does not fit
    // beside the weights and the I/O ring.
    bool placed = false;
    for (int kc = kc_first; kc >= 1 && !placed; kc /= 2) {
        p.a_kc = kc;
        // Halo form: one slot per channel block, all of a tile's blocks in the
        // ring when two accumulator slots share them; slots stay 1024-byte
        // aligned.  (the stride-2 halo form: four planes of two K halves)
        p.a_part = p.halo == 3 ? (h3_bytes + 1023) / 1024 * 1024
                   : p.halo    ? ((p.halo == 2 ? 8 : 2) * p.a_half + 1023) / 1024 * 1024
                               : p.a_kc * kASlotBytes;
        p.w_part = p.wstream ? (p.halo ? 9 : p.a_kc) * p.NC * 32 : 0;
        p.a_slot = p.a_part + p.w_part;
        const int a_min = p.halo ? (p.n_subs > 1 ? p.C1 + 1 : 2) : ring_min(p.a_kc);
        const int a_want = std::max(a_min, p.wstream      ? 4
                                           : p.halo == 3 ? 12  // one slot per tile: a deep ring
                                                         : a_bytes_want / p.a_slot);
        // A projection layer whose boxes hold several K blocks takes a deeper
        // floor of output stages before its activation ring may grow.
        // (Measured on the Res3.1 Conv3 with its stride-2 projection,
        // B = 256: 69.8 us with four 16 KB boxes and three output stages,
        // 73.1 with five and two, 72.0 with three and four.)
        for (int r_floor = p.C1b && kc > 1 ? std::max(r_lo, 3) : r_lo; r_floor >= r_lo && !placed; --r_floor)
            for (int fold = 1; fold >= 0 && !placed; --fold)
                for (int a = a_want; a >= a_min && !placed; --a)
                    for (int r = r_hi; r >= r_floor && !placed; --r)
                        placed = layout(fold, a, r);
    }
    if (!placed)
        return X1CB_ERR_SHAPE;
    // Two MMA warps (see the plan field) on an even ring of at least 4 slots:
    // each takes half of it.
    // (Measured: the folded stem, whose one box per tile feeds R MMAs, ran 17 %
    // faster with a second issuer; the 3x3 halo form, bound by its six-slot
    // activation ring behind 144 KB of weights, gained nothing, and a 1x1 with
    // 4 K blocks per box lost 35 % to the half ring's exposed load latency.)
    p.n_mma_warps = (p.halo == 3 && !has_res && !p.wstream && p.nmma <= 128 && p.n_subs == 1 &&
                     p.n_slots % 2 == 0 && p.a_stages % 2 == 0 && p.a_stages >= 4)
                        ? 2
                        : 1;
    p.io_wide = p.tw * 4 <= 256 && !p.pool ? 1 : 0;  // TMA boxes span at most 256 elements
    // The swizzled stages need whole 4-pixel groups and 1024-byte aligned stages.
    p.io_swz = (p.tw % 4 == 0 && p.Wp % 4 == 0 && p.off_r % 1024 == 0 && !p.pool) ? 1 : 0;

    // Pairs: units are clusters of two CTAs, each taking pair tiles.
    const int per_unit = p.pair ? 2 : 1;
    const long long work = (mtiles + per_unit - 1) / per_unit * p.n_groups;
    long long grid = std::min<long long>(num_sms / per_unit, work);
    grid = (grid / p.n_groups) * p.n_groups;
    if (grid < p.n_groups)
        grid = p.n_groups;
    p.grid = static_cast<int>(grid) * per_unit;
    p.wait_limit_ns = 2000000000ull;
    return X1CB_OK;
}

int launch_conv(const ConvPlan &p, const int8_t *x, const int8_t *w, const int32_t *bias,
                const int32_t *mult, const int8_t *r, int8_t *out, cudaStream_t stream,
                const int8_t *x2, const int8_t *w2)
{
    if (p.C1b && (!x2 || !w2))
        return X1CB_ERR_NULL;
    CUtensorMap tmA, tmW, tmR, tmO, tmA2, tmW2;
    // Activations: dims (32 ch, Wp, Hp, B, C1) -- channel blocks outermost so a
    // box (32, tw, th, tg, a_kc) lands as a_kc K-block tiles one after another.
    // Halo form: dims (32 ch, W, H, C1, B), box (16, tw+2, th+2, 1, tg) -- one K
    // half of the framed tile as 16-byte rows, zeros outside the image.
    if (p.halo == 2) {
        // Stride-2 planes: dims (32 ch, Win, Hin, C1, B) at traversal step 2;
        // a box of (2(W+1), 2(th+1)) elements lands one (W+1) x (th+1) plane.
        const uint64_t dims[5] = {32, (uint64_t)p.Win, (uint64_t)p.Hin, (uint64_t)p.C1,
                                  (uint64_t)p.B};
        const uint64_t str[4] = {32, (uint64_t)p.Win * 32, (uint64_t)p.Hin * p.Win * 32,
                                 (uint64_t)p.C1 * p.Hin * p.Win * 32};
        const uint32_t box[5] = {16, (uint32_t)(2 * p.row_pitch), (uint32_t)(2 * (p.th + 1)), 1,
                                 (uint32_t)p.tg};
        const uint32_t es[5] = {1, 2, 2, 1, 1};
        if (int e = encode_map(&tmA, x, 5, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE,
                               CU_TENSOR_MAP_DATA_TYPE_UINT8, es))
            return e;
    } else if (p.halo == 3) {
        // Folded stem: dims (32 ch, Win, Hin, B, 1); a box of the tile's tw
        // columns and all 2*th + R - 2 input rows it needs, 32-byte swizzle.
        const uint64_t dims[5] = {32, (uint64_t)p.Wpi, (uint64_t)p.Hpi, (uint64_t)p.B, 1};
        const uint64_t str[4] = {32, (uint64_t)p.Wpi * 32, (uint64_t)p.Hpi * p.Wpi * 32,
                                 (uint64_t)p.B * p.Hpi * p.Wpi * 32};
        const uint32_t box[5] = {32, (uint32_t)p.tw, (uint32_t)(2 * p.th + p.R - 2), 1, 1};
        if (int e = encode_map(&tmA, x, 5, dims, str, box, CU_TENSOR_MAP_SWIZZLE_32B))
            return e;
    } else if (p.halo) {
        const uint64_t dims[5] = {32, (uint64_t)p.W, (uint64_t)p.H, (uint64_t)p.C1,
                                  (uint64_t)p.B};
        const uint64_t str[4] = {32, (uint64_t)p.W * 32, (uint64_t)p.H * p.W * 32,
                                 (uint64_t)p.C1 * p.H * p.W * 32};
        const uint32_t box[5] = {16, (uint32_t)p.row_pitch, (uint32_t)(p.th + 2), 1,
                                 (uint32_t)p.tg};
        if (int e = encode_map(&tmA, x, 5, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE))
            return e;
    } else {
        // Input extent (Wpi, Hpi); a strided map loads every stride-th pixel,
        // so a box of tw*stride x th*stride elements lands tw x th pixels.
        const uint64_t dims[5] = {32, (uint64_t)p.Wpi, (uint64_t)p.Hpi, (uint64_t)p.B,
                                  (uint64_t)p.C1};
        const uint64_t str[4] = {32, (uint64_t)p.Wpi * 32, (uint64_t)p.C1 * p.Hpi * p.Wpi * 32,
                                 (uint64_t)p.Hpi * p.Wpi * 32};
        const uint32_t box[5] = {32, (uint32_t)(p.tw * p.stride), (uint32_t)(p.th * p.stride),
                                 (uint32_t)p.tg, (uint32_t)p.a_kc};
        const uint32_t es[5] = {1, (uint32_t)p.stride, (uint32_t)p.stride, 1, 1};
        if (int e = encode_map(&tmA, x, 5, dims, str, box, CU_TENSOR_MAP_SWIZZLE_32B,
                               CU_TENSOR_MAP_DATA_TYPE_UINT8, es))
            return e;
    }
    // Second source (projection shortcut): dims (32, Win2, Hin2, B, C1b), the
    // same box at its own stride.
    tmA2 = tmA;
    if (p.C1b) {
        const uint64_t dims[5] = {32, (uint64_t)p.Win2, (uint64_t)p.Hin2, (uint64_t)p.B,
                                  (uint64_t)p.C1b};
        const uint64_t str[4] = {32, (uint64_t)p.Win2 * 32,
                                 (uint64_t)p.C1b * p.Hin2 * p.Win2 * 32,
                                 (uint64_t)p.Hin2 * p.Win2 * 32};
        const uint32_t box[5] = {32, (uint32_t)(p.tw * p.stride2), (uint32_t)(p.th * p.stride2),
                                 (uint32_t)p.tg, (uint32_t)p.a_kc};
        const uint32_t es[5] = {1, (uint32_t)p.stride2, (uint32_t)p.stride2, 1, 1};
        if (int e = encode_map(&tmA2, x2, 5, dims, str, box, CU_TENSOR_MAP_SWIZZLE_32B,
                               CU_TENSOR_MAP_DATA_TYPE_UINT8, es))
            return e;
    }
    // Weights [Oc/128][KB][128][32]: dims (32, 128, KB, Oc/128); box (32,128,1,NC/128)
    // (CTA pairs: one 128-row block, each CTA's half of a 256-channel group).
    {
        const uint64_t dims[4] = {32, (uint64_t)p.O2, (uint64_t)p.kb_a, (uint64_t)(p.Oc / p.O2)};
        const uint64_t str[3] = {32, (uint64_t)p.O2 * 32, (uint64_t)p.kb_a * p.O2 * 32};
        const uint32_t box[4] = {32, (uint32_t)p.O2, 1,
                                 (uint32_t)(p.pair ? 1 : p.NC / p.O2)};
        if (int e = encode_map(&tmW, w, 4, dims, str, box, CU_TENSOR_MAP_SWIZZLE_32B))
            return e;
    }
    tmW2 = tmW;
    if (p.C1b) {
        const uint64_t dims[4] = {32, (uint64_t)p.O2, (uint64_t)p.C1b, (uint64_t)(p.Oc / p.O2)};
        const uint64_t str[3] = {32, (uint64_t)p.O2 * 32, (uint64_t)p.C1b * p.O2 * 32};
        const uint32_t box[4] = {32, (uint32_t)p.O2, 1, (uint32_t)(p.NC / p.O2)};
        if (int e = encode_map(&tmW2, w2, 4, dims, str, box, CU_TENSOR_MAP_SWIZZLE_32B))
            return e;
    }
    // Shortcut and output, no swizzle: one box is one I/O stage [tg][4][th][tw][32].
    // Wide form: the same bytes as 8-byte elements, dims (4*Wp, Hp, O1, B) and
    // box (4*tw, th, 4, tg), so a box row is one contiguous run of tw*32 bytes.
    if (p.io_swz) {
        // 128-byte rows: dims (16 x 8 bytes, Wp/4, Hp, O1, B), box (16, tw/4, th, 4, tg).
        const uint64_t dims[5] = {16, (uint64_t)p.Wp / 4, (uint64_t)p.Hp, (uint64_t)p.O1,
                                  (uint64_t)p.B};
        const uint64_t str[4] = {128, (uint64_t)p.Wp * 32, (uint64_t)p.Hp * p.Wp * 32,
                                 (uint64_t)p.O1 * p.Hp * p.Wp * 32};
        const uint32_t box[5] = {16, (uint32_t)p.tw / 4, (uint32_t)p.th, (uint32_t)p.stage_ch,
                                 (uint32_t)p.tg};
        if (int e = encode_map(&tmO, out, 5, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B,
                               CU_TENSOR_MAP_DATA_TYPE_UINT64))
            return e;
        if (p.has_res) {
            if (int e = encode_map(&tmR, r, 5, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B,
                                   CU_TENSOR_MAP_DATA_TYPE_UINT64))
                return e;
        } else {
            tmR = tmO;  // unused
        }
    } else if (p.io_wide) {
        const uint64_t dims[4] = {(uint64_t)p.Wp * 4, (uint64_t)p.Hp, (uint64_t)p.O1,
                                  (uint64_t)p.B};
        const uint64_t str[3] = {(uint64_t)p.Wp * 32, (uint64_t)p.Hp * p.Wp * 32,
                                 (uint64_t)p.O1 * p.Hp * p.Wp * 32};
        const uint32_t box[4] = {(uint32_t)p.tw * 4, (uint32_t)p.th, (uint32_t)p.stage_ch,
                                 (uint32_t)p.tg};
        if (int e = encode_map(&tmO, out, 4, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE,
                               CU_TENSOR_MAP_DATA_TYPE_UINT64))
            return e;
        if (p.has_res) {
            if (int e = encode_map(&tmR, r, 4, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE,
                                   CU_TENSOR_MAP_DATA_TYPE_UINT64))
                return e;
        } else {
            tmR = tmO;  // unused
        }
    } else if (p.pool) {
        // pooled output [B, Oc/32, Hpo, Wpo, 32]: box of the tile's pooled pixels
        const uint64_t dims[5] = {32, (uint64_t)p.Wpo, (uint64_t)p.Hpo, (uint64_t)p.O1,
                                  (uint64_t)p.B};
        const uint64_t str[4] = {32, (uint64_t)p.Wpo * 32, (uint64_t)p.Hpo * p.Wpo * 32,
                                 (uint64_t)p.O1 * p.Hpo * p.Wpo * 32};
        const uint32_t box[5] = {32, (uint32_t)p.pw, (uint32_t)p.ph, (uint32_t)p.stage_ch, 1};
        if (int e = encode_map(&tmO, out, 5, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE))
            return e;
        tmR = tmO;  // unused
    } else {
        const uint64_t dims[5] = {32, (uint64_t)p.Wp, (uint64_t)p.Hp, (uint64_t)p.O1,
                                  (uint64_t)p.B};
        const uint64_t str[4] = {32, (uint64_t)p.Wp * 32, (uint64_t)p.Hp * p.Wp * 32,
                                 (uint64_t)p.O1 * p.Hp * p.Wp * 32};
        const uint32_t box[5] = {32, (uint32_t)p.tw, (uint32_t)p.th, (uint32_t)p.stage_ch,
                                 (uint32_t)p.tg};
        if (int e = encode_map(&tmO, out, 5, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE))
            return e;
        if (p.has_res) {
            if (int e = encode_map(&tmR, r, 5, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE))
                return e;
        } else {
            tmR = tmO;  // unused
        }
    }
    const bool narrow = p.has_res && p.stage_ch == kRChunks / 2;
    auto kern = p.pair                ? conv_bn_act_kernel<3, false>
                : narrow              ? conv_bn_act_kernel<2, false>
                : p.has_res           ? conv_bn_act_kernel<1, false>
                : p.n_mma_warps > 1   ? conv_bn_act_kernel<0, true>
                                      : conv_bn_act_kernel<0, false>;
    if (int e = opt_in_smem(reinterpret_cast<const void *>(kern),
                            p.pair ? 6 : narrow ? 4 : p.has_res ? 1 : (p.n_mma_warps > 1 ? 3 : 0)))
        return e;
    ConvPlan q = p;
    q.trace = trace_table();
    // Every launch is a programmatic dependent of the preceding kernel on the
    // stream: its CTAs may start (shared-memory set-up, TMEM allocation) as
    // that kernel's CTAs leave, and wait for it to complete before touching
    // global memory (griddep_wait in the kernel).
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(q.grid, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = q.smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (!p.pair) {
        if (cudaLaunchKernelEx(&cfg, kern, tmA, tmW, tmR, tmO, tmA2, tmW2, bias, mult, q) !=
            cudaSuccess)
            return X1CB_ERR_CUDA;
        return cudaGetLastError() == cudaSuccess ? X1CB_OK : X1CB_ERR_CUDA;
    }
    // CTA pairs: clusters of two, no more than can be resident at once (the
    // kernel is persistent with a static assignment of pair tiles), a whole
    // number of clusters per channel group.
    cfg.gridDim = dim3(2, 1, 1);
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
    int resident = 0;
    if (cudaOccupancyMaxActiveClusters(&resident, kern, &cfg) != cudaSuccess || resident < 1) {
        cudaGetLastError();
        return X1CB_ERR_CUDA;
    }
    int clusters = std::min(q.grid / 2, resident);
    clusters = std::max(q.n_groups, clusters / q.n_groups * q.n_groups);
    if (clusters > resident)
        return X1CB_ERR_SHAPE;  // fewer resident pairs than channel groups
    q.grid = 2 * clusters;
    cfg.gridDim = dim3(q.grid, 1, 1);
    if (cudaLaunchKernelEx(&cfg, kern, tmA, tmW, tmR, tmO, tmA2, tmW2, bias, mult, q) !=
        cudaSuccess)
        return X1CB_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? X1CB_OK : X1CB_ERR_CUDA;
}

// The library's kernels live in separate translation units compiled without
// relocatable device code, where a device variable cannot be shared by
// declaration: the other kernels receive these addresses as parameters.
int device_words(unsigned int **status, unsigned int **forms)
{
    void *ps = nullptr, *pf = nullptr;
    if (cudaGetSymbolAddress(&ps, g_dev_status) != cudaSuccess ||
        cudaGetSymbolAddress(&pf, g_dev_forms) != cudaSuccess)
        return X1CB_ERR_CUDA;
    *status = static_cast<unsigned int *>(ps);
    *forms = static_cast<unsigned int *>(pf);
    return X1CB_OK;
}

unsigned long long *trace_table()
{
#ifdef X1CB_TRACE
    void *t = nullptr;
    return cudaGetSymbolAddress(&t, g_trace) == cudaSuccess
               ? static_cast<unsigned long long *>(t)
               : nullptr;
#else
    return nullptr;
#endif
}

long long copy_trace(unsigned long long *host, long long words, bool clear)
{
#ifdef X1CB_TRACE
    const long long n = words < kTraceWords ? words : kTraceWords;
    if (n > 0 && cudaMemcpyFromSymbol(host, g_trace, n * sizeof(unsigned long long)) != cudaSuccess)
        return -1;
    if (clear && cudaMemset(trace_table(), 0, sizeof(g_trace)) != cudaSuccess)
        return -1;
    return n;
#else
    (void)host;
    (void)words;
    (void)clear;
    return 0;
#endif
}

unsigned int read_and_clear_dev_status(bool clear)
{
    unsigned int v = 0;
    cudaMemcpyFromSymbol(&v, g_dev_status, sizeof(v));
    if (clear) {
        const unsigned int z = 0;
        cudaMemcpyToSymbol(g_dev_status, &z, sizeof(z));
    }
    return v;
}

unsigned int read_and_clear_dev_forms(bool clear)
{
    unsigned int v = 0;
    cudaMemcpyFromSymbol(&v, g_dev_forms, sizeof(v));
    if (clear) {
        const unsigned int z = 0;
        cudaMemcpyToSymbol(g_dev_forms, &z, sizeof(z));
    }
    return v;
}

}  // namespace x1cb
