// Conv2 -> Conv3 of the Res3.x bottleneck in one kernel: the 3x3 convolution
// (+ folded BN + ReLU, requantised to int8) feeds the 1x1 convolution (+ folded
// BN + shortcut Sum + ReLU) through on-chip memory, so Conv2's output never
// travels through HBM.  This is the merge of two consecutive convolutions
// that the Inspur MLPerf ResNet50 convolution-merge article names in section
// 2.1 (its A100 kernel merged only Conv3 with the shortcut, section 2.2).
//
// Both weight sets must stay on chip (3x3: 144 KB for 128 channels, 1x1: up to
// 64 KB), more than one SM's shared memory next to the rings, so the kernel
// runs on pairs of CTAs (a cluster of two) that share every MMA
// (tcgen05 cta_group::2): A is split by rows -- each CTA loads its own halo
// tile and keeps its own Conv2 output as Conv3's A operand -- and B by
// columns, so each CTA holds half of each weight set.  Rank 0 issues every
// MMA (M = 256: 128 rows per CTA); each CTA's TMEM receives its own rows.
//
// Per CTA (20 warps):
//   warp 0      TMA producer: its weight halves once, then the halo tile of
//               each channel block (one 3x3 A slot, nine row-shifted views),
//               completion counted on rank 0's barriers
//   warp 1      TMEM owner (both ranks); MMA issuer (rank 0): Conv2 of pair
//               tile i, then Conv3 of pair tile i-1 in 128-channel chunks
//   warp 2      TMA producer of the shortcut stages (own rows)
//   warp 3      TMA store of finished output stages (own rows)
//   warps 4-19  epilogue, 4 turns per TMEM lane quarter over one ring of
//               accumulators: the MMA issuer fills four 128-column TMEM slots
//               in issue order with Conv2 tiles and Conv3 chunks (item k in
//               slot k % 4), and turn g takes items g, g+4, ...: a Conv2 item
//               is requantised into this CTA's Conv3 A buffer in shared
//               memory, a Conv3 item gets the shortcut Sum and is
//               requantised into an output stage.  All 16 warps share both
//               kinds of work (Conv3's is ~4x Conv2's per tile).
// Every wait is bounded; a wait that runs out raises the CTA's abort flag and
// a status bit, and both CTAs leave through a bounded exit handshake.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <climits>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "x1cb_epi.cuh"
#include "x1cb_internal.h"
#include "x1cb_ptx.cuh"
#include "x1cb_trace.cuh"

namespace x1cb {

namespace {

constexpr int kA3Bufs = 2;           // Conv3 A buffers (Conv2 results) in shared memory
constexpr int kSlots = 4;            // 128-column accumulator slots (= epilogue turns)
constexpr int kA3Bytes = 128 * 128;  // Conv3 A buffer: 128 rows x 128 channels
static_assert(kEpiWarps == 4 * kSlots, "one epilogue turn per accumulator slot");
static_assert(kSlots * 128 == kTmemCols, "the slots fill the TMEM");
constexpr int kHalfRows = 64;      // B rows (output channels) each CTA holds per MMA

struct ChainBars {
    uint32_t base;
    int a_stages, r_stages;
    __device__ uint32_t at(int i) const { return base + 8u * static_cast<uint32_t>(i); }
    __device__ uint32_t w_full() const { return at(0); }
    __device__ uint32_t mma_done() const { return at(1); }
    __device__ uint32_t exit_bar() const { return at(2); }
    __device__ uint32_t a_full(int s) const { return at(3 + s); }
    __device__ uint32_t a_empty(int s) const { return at(3 + a_stages + s); }
    __device__ uint32_t acc_full(int k) const { return at(3 + 2 * a_stages + k); }
    __device__ uint32_t acc_empty(int k) const { return at(7 + 2 * a_stages + k); }
    __device__ uint32_t a3_full(int k) const { return at(11 + 2 * a_stages + k); }
    __device__ uint32_t a3_empty(int k) const { return at(13 + 2 * a_stages + k); }
    __device__ uint32_t io_full(int s) const { return at(15 + 2 * a_stages + s); }
    __device__ uint32_t out_ready(int s) const { return at(15 + 2 * a_stages + r_stages + s); }
    __device__ uint32_t io_empty(int s) const { return at(15 + 2 * a_stages + 2 * r_stages + s); }
    static int count(int a, int r) { return 15 + 2 * a + 3 * r; }
};

// Own halo tile of pair tile `pt`: tile 2*pt + rank of the halo tiling (full
// image width, th rows of tg images).  Past the last tile the origin lies
// beyond the batch: loads read zeros and nothing is stored.
__device__ __forceinline__ void chain_origin(const ChainPlan &p, int mt, int &h0, int &b0)
{
    h0 = (mt % p.nTh) * p.th;
    b0 = (mt / p.nTh) * p.tg;
}

// Requantisation of 32 accumulators (channels ch..ch+31) in the form chosen
// for the layer.  The constant table holds int32 biases in the all-32-bit
// form and int64 offsets otherwise, so the channel offset is applied per form.
template <bool kRes>
__device__ __forceinline__ void requant_any(int mode, const uint32_t *v, const int32_t *cm,
                                            const long long *cC, int ch, const uint32_t *rw,
                                            int m_r, int S, int mr2, const uint32_t (&rsel)[4],
                                            uint32_t *ow)
{
    if (mode == 2)
        requant_hi32<kRes, true, false, 8>(v, cm + ch,
                                           reinterpret_cast<const int32_t *>(cC) + ch, rw, mr2,
                                           rsel, ow);
    else if (mode == 1)
        requant_fast<kRes, 8>(v, cm + ch, cC + ch, rw, mr2, rsel, ow);
    else
        requant32<kRes>(v, cm + ch, cC + ch, rw, m_r, S, ow);
}

// Per-layer constants of the chosen form into shared memory (see the
// convolution kernel's prologue): mode 2: m*2^(33-S) and the bias; mode 1:
// m*2^(32-S) and bias*m' + 2^31; mode 0: m and bias*m + 2^(S-1).
__device__ __forceinline__ int pick_form(const int32_t *bias, const int32_t *mult, int n, int m_r,
                                         int S, int K, bool res)
{
    bool fast = true, hi = true;
    for (int o = threadIdx.x; o < n; o += blockDim.x) {
        fast = fast && fast_form_ok(mult[o], bias[o], m_r, S, K, res);
        hi = hi && hi32_ok(mult[o], bias[o], S, K);
    }
    const bool all_fast = __syncthreads_and(fast ? 1 : 0) != 0;
    const bool all_hi = __syncthreads_and(hi ? 1 : 0) != 0 && hi32_layer_ok(m_r, S, res);
    return all_hi ? 2 : (all_fast ? 1 : 0);
}

__device__ __forceinline__ void fill_consts(int mode, const int32_t *bias, const int32_t *mult,
                                            int n, int S, int32_t *cm, long long *cC)
{
    int32_t *cb = reinterpret_cast<int32_t *>(cC);
    for (int o = threadIdx.x; o < n; o += blockDim.x) {
        const long long mm = mult[o];
        if (mode == 2) {
            cm[o] = static_cast<int32_t>(mm * (1ll << (33 - S)));
            cb[o] = bias[o];
        } else if (mode == 1) {
            const long long mp = mm * (1ll << (32 - S));
            cm[o] = static_cast<int32_t>(mp);
            cC[o] = static_cast<long long>(bias[o]) * mp + (1ll << 31);
        } else {
            cm[o] = static_cast<int32_t>(mm);
            cC[o] = static_cast<long long>(bias[o]) * mm + (1ll << (S - 1));
        }
    }
}

// Shortcut operands of the chosen Conv3 form (see the convolution kernel).
__device__ __forceinline__ int shortcut_operands(int mode, int m_r, int S, uint32_t (&rsel)[4])
{
    const int sh = 32 - S;
    const int k8 = mode >= 2 ? 0 : (sh < 0 ? 0 : (sh / 8 < 3 ? sh / 8 : 3));
    const int mr2 =
        mode == 1 ? static_cast<int>(static_cast<long long>(m_r) * (1ll << (sh - 8 * k8)))
                  : (mode >= 2 ? static_cast<int>(static_cast<long long>(m_r) / (1ll << (S - 1)))
                               : 0);
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        uint32_t sel = 0;
        for (int i = 0; i < 4; ++i) {
            const uint32_t nib = i < k8 ? 4u : (i == k8 ? static_cast<uint32_t>(b) : 8u | b);
            sel |= nib << (4 * i);
        }
        rsel[b] = sel;
    }
    return mr2;
}

// Epilogue of one warp over the accumulator ring: the MMA issuer fills the
// four slots in issue order with Conv2 tiles and Conv3 chunks (item k in slot
// k % 4), and turn g takes items g, g+4, ... (it owns slot g, so it sees every
// phase of its slot in order).  kM2 / kM3: the exact form of each layer when
// it is the all-32-bit one (2), or -1 for the form chosen at run time
// (generic, 64-bit or all-32-bit); kK1: the shortcut scale is 1.
struct ChainEpi {
    const ChainPlan *p;
    ChainBars bars;
    WaitCtl ctl;
    uint32_t tmem_base;
    uint8_t *smem;
    volatile int *io_ticket;
    const int32_t *cm2;
    const long long *cc2;
    const int32_t *cm3;
    const long long *cc3;
    int n_my, mode2, mode3;
};

template <int kM, bool kRes, bool kK1>
__device__ __forceinline__ void requant_chain(int mode, const uint32_t *v, const int32_t *cm,
                                          const long long *cC, int ch, const uint32_t *rw,
                                          int m_r, int S, int mr2, const uint32_t (&rsel)[4],
                                          uint32_t *ow)
{
    if (kM == 2)
    requant_hi32<kRes, true, kK1, 8>(v, cm + ch, reinterpret_cast<const int32_t *>(cC) + ch,
                                     rw, mr2, rsel, ow);
    else
    requant_any<kRes>(mode, v, cm, cC, ch, rw, m_r, S, mr2, rsel, ow);
}

template <int kM2, int kM3, bool kK1>
__device__ __forceinline__ void chain_epilogue(const ChainEpi &ce, int warp, int lane)
{
    const ChainPlan &p = *ce.p;
    const ChainBars &bars = ce.bars;
    const WaitCtl &ctl = ce.ctl;
    const uint32_t tmem_base = ce.tmem_base;
    uint8_t *smem = ce.smem;
    volatile int *io_ticket = ce.io_ticket;
    const int32_t *cm2 = ce.cm2;
    const long long *cc2 = ce.cc2;
    const int32_t *cm3 = ce.cm3;
    const long long *cc3 = ce.cc3;
    const int n_my = ce.n_my;
    const int mode2 = ce.mode2, mode3 = ce.mode3;
    // Item order is the MMA issuer's: Conv2 of tile i, then Conv3 of tile
    // i - 1 in n_chunks chunks.  Each turn owns slot `turn` (items k with
    // k % 4 == turn), so it sees every phase of its slot in order.
    const int q = warp & 3;
    const int turn = (warp - kEpiWarp0) >> 2;
    const int row = q * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t tslot = tmem_base + lane_addr + static_cast<uint32_t>(turn * 128);
    const uint32_t empty0 = mapa_shared(bars.acc_empty(turn), 0);
    // Conv3 output rows: this row's place in an output stage (halo rows
    // outside the image are computed and not stored).
    const int plane_t = p.tw * p.th;
    const int xi = row % p.row_pitch;
    const int yi = (row % p.plane_m) / p.row_pitch;
    const int gi = row / p.plane_m;
    const bool in_box = xi < p.tw && yi < p.th && gi < p.tg;
    const int row_off = in_box ? ((gi * kRChunks) * plane_t + yi * p.tw + xi) * 32 : 0;
    const int chunk_stride = plane_t * 32;
    const int swz_mask = p.io_swz ? 0x70 : 0;
    uint32_t rsel3[4];
    const int mr2 = shortcut_operands(mode3, p.m_r, p.S, rsel3);
    const uint32_t rsel2[4] = {0, 0, 0, 0};
    int k = 0;             // item index in issue order
    uint32_t kph = 0;      // parity of this turn's slot at its next item
    int c3_st = 0;         // shortcut ring slot and phase of the next Conv3 chunk
    uint32_t c3_ph = 0;
    bool ok = true;
    const bool tr = q == 0 && lane == 0;  // one trace writer per turn
    for (int i = 0; ok && i <= n_my; ++i) {
        if (i < n_my) {
            if ((k & 3) == turn) {
                // Conv2 of tile i -> int8 -> A buffer i % 2 of this CTA.
                const int b = i & 1;
                if (!__all_sync(0xffffffffu,
                                mbar_wait(bars.acc_full(turn), kph, ctl, kDevTimeoutEpilogue)) ||
                    !__all_sync(0xffffffffu,
                                mbar_wait(bars.a3_empty(b),
                                          static_cast<uint32_t>((i >> 1) & 1) ^ 1u, ctl,
                                          kDevTimeoutEpilogue))) {
                    ok = false;
                    break;
                }
                if (tr)
                    X1CB_TRACE_AT(p.trace, 6, i);
                tc_fence_after();
                uint8_t *a3 = smem + p.off_a3 + b * kA3Bytes;
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t v[32], ow[8];
                    __syncwarp();
                    tmem_ld_32x32b_x32_sync(tslot + static_cast<uint32_t>(c * 32), v);
                    requant_chain<kM2, false, false>(mode2, v, cm2, cc2, c * 32, nullptr, 0, p.S, 0,
                                                 rsel2, ow);
                    // K block c of the A buffer: two 16-byte halves, rows 16 bytes apart.
                    uint4 *dst = reinterpret_cast<uint4 *>(a3 + c * (kA3Bytes / 4) + row * 16);
                    dst[0] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                    dst[(kA3Bytes / 8) / 16] = make_uint4(ow[4], ow[5], ow[6], ow[7]);
                }
                fence_proxy_async_smem();  // read by the MMA (async proxy, rank 0's issue)
                tc_fence_before();
                __syncwarp();
                if (tr)
                    X1CB_TRACE_AT(p.trace, 7, i);
                if (lane == 0) {
                    mbar_arrive_cluster(empty0);
                    mbar_arrive_cluster(mapa_shared(bars.a3_full(b), 0));
                }
                kph ^= 1u;
            }
            ++k;
        }
        if (i >= 1) {
            const int j = i - 1;
            for (int c = 0; c < p.n_chunks; ++c, ++k) {
                // Conv3 of tile j, output chunk c: shortcut stage n = j*n_chunks + c,
                // ring slot n % r_stages and phase (n / r_stages) & 1, counted
                // over every chunk (this turn's or not)
                const int n = j * p.n_chunks + c;
                const int st = c3_st;
                const uint32_t st_phase = c3_ph;
                if (++c3_st == p.r_stages) {
                    c3_st = 0;
                    c3_ph ^= 1u;
                }
                if ((k & 3) != turn)
                    continue;
                // Stages are taken in order (the ticket), so each stage's
                // previous phase is complete before its arrival is awaited.
                if (!__all_sync(0xffffffffu,
                                mbar_wait(bars.acc_full(turn), kph, ctl, kDevTimeoutEpilogue))) {
                    ok = false;
                    break;
                }
                if (tr)
                    X1CB_TRACE_AT(p.trace, 8, n);
                if (!__all_sync(0xffffffffu, ticket_wait(io_ticket, static_cast<int>(n), ctl,
                                                         kDevTimeoutEpilogue)) ||
                    !__all_sync(0xffffffffu, mbar_wait(bars.io_full(st), st_phase, ctl,
                                                       kDevTimeoutEpilogue))) {
                    ok = false;
                    break;
                }
                if (tr)
                    X1CB_TRACE_AT(p.trace, 9, n);
                if (lane == 0)
                    atomicMax(const_cast<int *>(io_ticket), static_cast<int>(n + 1));
                tc_fence_after();
                uint8_t *stage = smem + p.off_r + st * kRSlotBytes;
#pragma unroll 1
                for (int cs = 0; cs < kRChunks; ++cs) {
                    const int ch = c * 128 + cs * 32;
                    uint32_t v[32];
                    __syncwarp();
                    tmem_ld_32x32b_x32_sync(tslot + static_cast<uint32_t>(cs * 32), v);
                    const int o = row_off + cs * chunk_stride;
                    const int sw = swz_mask & (o >> 3);
                    uint4 *pa = reinterpret_cast<uint4 *>(stage + (o ^ sw));
                    uint4 *pb = reinterpret_cast<uint4 *>(stage + ((o + 16) ^ sw));
                    const uint4 ra = *pa, rb = *pb;
                    const uint32_t rw[8] = {ra.x, ra.y, ra.z, ra.w, rb.x, rb.y, rb.z, rb.w};
                    uint32_t ow[8];
                    requant_chain<kM3, true, kK1>(mode3, v, cm3, cc3, ch, rw, p.m_r, p.S, mr2,
                                                 rsel3, ow);
                    if (in_box) {
                        *pa = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                        *pb = make_uint4(ow[4], ow[5], ow[6], ow[7]);
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (tr)
                    X1CB_TRACE_AT(p.trace, 10, n);
                if (lane == 0) {
                    mbar_arrive(bars.out_ready(st));
                    mbar_arrive_cluster(empty0);
                }
                kph ^= 1u;
            }
        }
    }
}

// Epilogue of the 3x3 alone on CTA pairs (kC3 = false): the MMA issuer puts
// pair tile i's accumulator in slot i % 4 and turn g takes tiles g, g+4, ...
// (it owns slot g, so it sees every phase of it in order).  Each tile is
// requantised into one output stage (128 channels of the tile's rows) in
// stage order (the ticket), which the store warp writes back.
template <int kM2>
__device__ __forceinline__ void conv2_epilogue(const ChainEpi &ce, int warp, int lane)
{
    const ChainPlan &p = *ce.p;
    const ChainBars &bars = ce.bars;
    const WaitCtl &ctl = ce.ctl;
    const int q = warp & 3;
    const int turn = (warp - kEpiWarp0) >> 2;
    const int row = q * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t tslot = ce.tmem_base + lane_addr + static_cast<uint32_t>(turn * 128);
    const uint32_t empty0 = mapa_shared(bars.acc_empty(turn), 0);
    // This row's place in an output stage (halo rows outside the image are
    // computed and not stored).
    const int plane_t = p.tw * p.th;
    const int xi = row % p.row_pitch;
    const int yi = (row % p.plane_m) / p.row_pitch;
    const int gi = row / p.plane_m;
    const bool in_box = xi < p.tw && yi < p.th && gi < p.tg;
    const int row_off = in_box ? ((gi * kRChunks) * plane_t + yi * p.tw + xi) * 32 : 0;
    const int chunk_stride = plane_t * 32;
    const int swz_mask = p.io_swz ? 0x70 : 0;
    const uint32_t rsel[4] = {0, 0, 0, 0};
    uint32_t kph = 0;
    const bool tr = q == 0 && lane == 0;
    // output stage of tile i: ring slot i % r_stages, phase (i / r_stages) & 1,
    // advanced by counters (kSlots tiles per step)
    int st = turn % p.r_stages;
    uint32_t st_phase = static_cast<uint32_t>((turn / p.r_stages) & 1);
    for (int i = turn; i < ce.n_my; i += kSlots) {
        if (!__all_sync(0xffffffffu,
                        mbar_wait(bars.acc_full(turn), kph, ctl, kDevTimeoutEpilogue)))
            return;
        if (tr)
            X1CB_TRACE_AT(p.trace, 6, i);
        if (!__all_sync(0xffffffffu, ticket_wait(ce.io_ticket, i, ctl, kDevTimeoutEpilogue)) ||
            !__all_sync(0xffffffffu,
                        mbar_wait(bars.io_full(st), st_phase, ctl, kDevTimeoutEpilogue)))
            return;
        if (lane == 0)
            atomicMax(const_cast<int *>(ce.io_ticket), i + 1);
        tc_fence_after();
        uint8_t *stage = ce.smem + p.off_r + st * kRSlotBytes;
#pragma unroll 1
        for (int cs = 0; cs < kRChunks; ++cs) {
            uint32_t v[32], ow[8];
            __syncwarp();
            tmem_ld_32x32b_x32_sync(tslot + static_cast<uint32_t>(cs * 32), v);
            requant_chain<kM2, false, false>(ce.mode2, v, ce.cm2, ce.cc2, cs * 32, nullptr, 0,
                                             p.S, 0, rsel, ow);
            const int o = row_off + cs * chunk_stride;
            const int sw = swz_mask & (o >> 3);
            if (in_box) {
                *reinterpret_cast<uint4 *>(stage + (o ^ sw)) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                *reinterpret_cast<uint4 *>(stage + ((o + 16) ^ sw)) =
                    make_uint4(ow[4], ow[5], ow[6], ow[7]);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (tr)
            X1CB_TRACE_AT(p.trace, 7, i);
        if (lane == 0) {
            mbar_arrive(bars.out_ready(st));
            mbar_arrive_cluster(empty0);
        }
        kph ^= 1u;
        for (int a = 0; a < kSlots; ++a)
            if (++st == p.r_stages) {
                st = 0;
                st_phase ^= 1u;
            }
    }
}

// kC3 = true: Conv2 -> Conv3 fused; false: the 3x3 alone (Conv2's layout,
// output stored like Conv3's).
template <bool kC3>
__global__ void __launch_bounds__(kThreads, 1)
    chain23_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW2,
                   const __grid_constant__ CUtensorMap tmW3,
                   const __grid_constant__ CUtensorMap tmR, const __grid_constant__ CUtensorMap tmO,
                   const int32_t *__restrict__ b2, const int32_t *__restrict__ m2,
                   const int32_t *__restrict__ b3, const int32_t *__restrict__ m3,
                   unsigned int *dev_status, unsigned int *dev_forms, const ChainPlan p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;

    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + p.off_misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + p.off_misc + 4);
    // Conv3 items take the shortcut stages' arrivals in stage order (ticket).
    volatile int *io_ticket = reinterpret_cast<volatile int *>(smem + p.off_misc + 8);
    ChainBars bars{sbase + static_cast<uint32_t>(p.off_bar), p.a_stages, p.r_stages};
    const WaitCtl ctl{abort_flag, dev_status, p.wait_limit_ns};
    const uint64_t drain_ns = 200000000ull;
    const int pair0 = blockIdx.x / 2;
    const int pair_step = gridDim.x / 2;
    const int n_my = pair0 < p.n_pairs ? (p.n_pairs - pair0 + pair_step - 1) / pair_step : 0;

    // ---- set-up -----------------------------------------------------------------
    // Trace events (trace builds): 0 producer box n may load; 1 MMA sees tile
    // n's first box; 2 MMA has a slot for tile n's Conv2; 3 ... committed it;
    // 4 MMA sees tile n's Conv2 result; 5 MMA committed Conv3 chunk n; 6/7
    // epilogue starts/ends tile n's Conv2; 8/9/10 epilogue sees the
    // accumulator / shortcut of chunk n, is done; 11/12 store warp sees chunk
    // n / has read it; 13 shortcut chunk n issued; 14 weights seen; 15 start, end.
    if (threadIdx.x == 0)
        X1CB_TRACE_AT(p.trace, 15, 0);
    if (threadIdx.x == 0) {
        *abort_flag = 0;
        *io_ticket = 0;
        mbar_init(bars.w_full(), 1);
        mbar_init(bars.mma_done(), kC3 ? 1 : p.issuers);  // each MMA issuer's final commit
        mbar_init(bars.exit_bar(), 1);
        for (int s = 0; s < p.a_stages; ++s) {
            mbar_init(bars.a_full(s), 1);
            mbar_init(bars.a_empty(s), 1);
        }
        // Arrival counts: commits arrive once (multicast to both CTAs); the
        // epilogue barriers on rank 0 take one arrival per warp of a lane
        // quarter from each CTA (4 x 2).
        for (int k = 0; k < kSlots; ++k) {
            mbar_init(bars.acc_full(k), 1);
            mbar_init(bars.acc_empty(k), 8);
        }
        for (int k = 0; k < kA3Bufs; ++k) {
            mbar_init(bars.a3_full(k), 8);
            mbar_init(bars.a3_empty(k), 1);
        }
        for (int s = 0; s < p.r_stages; ++s) {
            mbar_init(bars.io_full(s), 1);
            mbar_init(bars.out_ready(s), 4);
            mbar_init(bars.io_empty(s), 1);
        }
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmW2);
        if (kC3) {
            tma_prefetch_desc(&tmW3);
            tma_prefetch_desc(&tmR);
        }
        tma_prefetch_desc(&tmO);
    }
    // Global memory only after the preceding grid (programmatic dependent
    // launch: this CTA may have started while it drained).
    griddep_wait();
    // Exact forms of the two layers (every CTA takes the same decision).
    int32_t *cm2 = reinterpret_cast<int32_t *>(smem + p.off_cm2);
    long long *cc2 = reinterpret_cast<long long *>(smem + p.off_cc2);
    int32_t *cm3 = reinterpret_cast<int32_t *>(smem + p.off_cm3);
    long long *cc3 = reinterpret_cast<long long *>(smem + p.off_cc3);
    const int mode2 = pick_form(b2, m2, p.Cm, 0, p.S, 9 * p.Cm, false);
    const int mode3 = kC3 ? pick_form(b3, m3, p.Cout, p.m_r, p.S, p.Cm, true) : mode2;
    fill_consts(mode2, b2, m2, p.Cm, p.S, cm2, cc2);
    if (kC3)
        fill_consts(mode3, b3, m3, p.Cout, p.S, cm3, cc3);
    if (threadIdx.x == 0)
        atomicOr(dev_forms, (1u << mode2) | (1u << mode3));
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish_pair();
        tc_fence_before();
    }
    __syncthreads();
    // Both CTAs' barriers are initialised and their TMEM allocated before any
    // traffic crosses between them.
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ---- producer: weight halves, then halo tiles --------------------------------
        // Slots of the halo ring are issued in rounds by n_iss lanes, which wait
        // for their slots together and issue as one (see the convolution
        // kernel's producer: one thread issues a tensor copy only every several
        // hundred cycles; n_iss <= a_stages / 2 keeps each slot barrier's
        // parity unambiguous).
        const int n_iss = max(1, min(kAIssuers, p.a_stages / 2));
        if (lane == 0) {
            const uint32_t wfull0 = mapa_shared(bars.w_full(), 0);
            const int half = static_cast<int>(rank) * kHalfRows;
            const uint32_t w2_bytes = 9 * p.C1 * kHalfRows * 32;
            const uint32_t w3_bytes = kC3 ? p.n_chunks * p.C1 * kHalfRows * 32 : 0;
            if (leader)  // both CTAs' halves complete on rank 0's barrier
                mbar_arrive_expect_tx(bars.w_full(), 2 * (w2_bytes + w3_bytes));
            for (int kb = 0; kb < 9 * p.C1; ++kb)
                tma2_load_4d(sbase + p.off_w2 + kb * kHalfRows * 32, &tmW2, wfull0, 0, half, kb,
                             0);
            if (kC3)
                for (int c = 0; c < p.n_chunks; ++c)
                    for (int kb = 0; kb < p.C1; ++kb)
                        tma2_load_4d(sbase + p.off_w3 + (c * p.C1 + kb) * kHalfRows * 32, &tmW3,
                                     wfull0, 0, half, kb, c);
        }
        __syncwarp();
        if (lane < kAIssuers) {
            const uint32_t abytes =
                static_cast<uint32_t>((p.stride == 2 ? 8 : 2) * 16 * p.plane_m * p.tg);
            const uint64_t pol = policy_evict_first();
            const long long total = static_cast<long long>(n_my) * p.C1;
            long long issued = 0;
            // This lane's slot n = base + lane: pair tile i, channel block c1
            // and the ring position of the next box of each half, advanced by
            // counters.  Fused: one ring (pos0).  The 3x3 alone: two MMA
            // warps, even pair tiles in slots [0, a/2), odd ones in [a/2, a),
            // each half consumed in order by its warp.
            const bool split = !kC3 && p.issuers == 2;
            const int half = split ? p.a_stages / 2 : p.a_stages;
            int i = 0, c1 = 0, pos0 = 0, pos1 = 0;
            uint32_t ph0 = 0u, ph1 = 0u;
            auto step = [&]() {  // past box (i, c1)
                if (split && (i & 1)) {
                    if (++pos1 == half) {
                        pos1 = 0;
                        ph1 ^= 1u;
                    }
                } else if (++pos0 == half) {
                    pos0 = 0;
                    ph0 ^= 1u;
                }
                if (++c1 == p.C1) {
                    c1 = 0;
                    ++i;
                }
            };
            for (int k = 0; k < lane && k < n_iss; ++k)
                step();
            for (long long base = 0; base < total; base += n_iss) {
                const long long n = base + lane;
                const bool have = lane < n_iss && n < total;
                const bool odd = split && (i & 1);
                const int stage = odd ? half + pos1 : pos0;
                const uint32_t phase = odd ? ph1 : ph0;
                if (!mbar_wait_lanes(kAIssuerMask, have, bars.a_empty(stage), phase ^ 1u, ctl,
                                     kDevTimeoutProducer))
                    break;
                if (have) {
                    X1CB_TRACE_AT(p.trace, 0, n);
                    const int mt = 2 * (pair0 + i * pair_step) + static_cast<int>(rank);
                    int h0, b0;
                    chain_origin(p, mt, h0, b0);
                    if (leader)
                        mbar_arrive_expect_tx(bars.a_full(stage), 2 * abytes);
                    const uint32_t slot = sbase + p.off_a + stage * p.a_slot;
                    const uint32_t full0 = mapa_shared(bars.a_full(stage), 0);
                    if (!kC3 && p.stride == 2) {
                        // plane (pr, pc) from input (pc - 1, 2*h0 - 1 + pr), step 2,
                        // each K half a box
                        for (int pl = 0; pl < 4; ++pl)
                            for (int hf = 0; hf < 2; ++hf)
                                tma2_load_5d_hint(slot + static_cast<uint32_t>((2 * pl + hf) *
                                                                               p.a_half),
                                                  &tmA, full0, 16 * hf, (pl & 1) - 1,
                                                  2 * h0 - 1 + (pl >> 1), c1, b0, pol);
                    } else {
                        tma2_load_5d_hint(slot, &tmA, full0, 0, -1, h0 - 1, c1, b0, pol);
                        tma2_load_5d_hint(slot + p.a_half, &tmA, full0, 16, -1, h0 - 1, c1, b0,
                                          pol);
                    }
                }
                issued = base + n_iss < total ? base + n_iss : total;
                for (int k = 0; k < n_iss; ++k)
                    step();
            }
            // Both CTAs' copies complete on rank 0's barriers: rank 0 lets every
            // copy still in flight land (the MMA has normally seen them all)
            // before the exit handshake releases either CTA.
            __syncwarp(kAIssuerMask);
            if (leader && lane == 0) {
                if (!mbar_drain(bars.w_full(), 0, drain_ns))
                    atomicOr(dev_status, kDevDrainFailed);
                // the latest box of every slot (split ring: walk back until
                // both halves' slots are seen)
                unsigned int seen = 0;
                const unsigned int all = (1u << p.a_stages) - 1u;
                for (long long k = issued - 1; k >= 0 && seen != all && k >= issued - 4 * p.a_stages;
                     --k) {
                    int st;
                    uint32_t ph;
                    if (split) {
                        const long long t = k / p.C1, li = (t >> 1) * p.C1 + (k - t * p.C1);
                        st = static_cast<int>((t & 1) * half + li % half);
                        ph = static_cast<uint32_t>((li / half) & 1);
                    } else {
                        st = static_cast<int>(k % p.a_stages);
                        ph = static_cast<uint32_t>((k / p.a_stages) & 1);
                    }
                    if (seen & (1u << st))
                        continue;
                    seen |= 1u << st;
                    if (!mbar_drain(bars.a_full(st), ph, drain_ns))
                        atomicOr(dev_status, kDevDrainFailed);
                }
            }
        }
        __syncwarp();
    } else if (warp == 2 && kC3) {
        // ---- shortcut stages (own rows) ------------------------------------------------
        if (lane == 0) {
            const uint32_t rbytes = static_cast<uint32_t>(kRChunks * p.rows * 32);
            const uint64_t pol = policy_evict_first();
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            bool ok = true;
            for (int i = 0; ok && i < n_my; ++i) {
                const int mt = 2 * (pair0 + i * pair_step) + static_cast<int>(rank);
                int h0, b0;
                chain_origin(p, mt, h0, b0);
                for (int c = 0; c < p.n_chunks; ++c) {
                    if (!mbar_wait(bars.io_empty(stage), phase ^ 1u, ctl, kDevTimeoutProducer)) {
                        ok = false;
                        break;
                    }
                    X1CB_TRACE_AT(p.trace, 13, issued);
                    mbar_arrive_expect_tx(bars.io_full(stage), rbytes);
                    const uint32_t dst = sbase + p.off_r + stage * kRSlotBytes;
                    if (p.io_swz)
                        tma_load_5d_hint(dst, &tmR, bars.io_full(stage), 0, 0, h0, c * kRChunks,
                                         b0, pol);
                    else
                        tma_load_4d_hint(dst, &tmR, bars.io_full(stage), 0, h0, c * kRChunks, b0,
                                         pol);
                    ++issued;
                    if (++stage == p.r_stages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            const long long last = issued < p.r_stages ? issued : p.r_stages;
            for (long long k = issued - last; k < issued; ++k)
                if (!mbar_drain(bars.io_full(static_cast<int>(k % p.r_stages)),
                                static_cast<uint32_t>((k / p.r_stages) & 1), drain_ns))
                    atomicOr(dev_status, kDevDrainFailed);
        }
        __syncwarp();
    } else if (warp == 3) {
        // ---- stores of finished output stages (own rows) -------------------------------
        // The 3x3 alone has no shortcut to load: this warp hands the stages
        // out, each one's first use at once and its next use as soon as its
        // store has read it.
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            if (!kC3)
                for (int s = 0; s < p.r_stages; ++s)
                    mbar_arrive(bars.io_full(s));
            for (int i = 0; ok && i < n_my; ++i) {
                const int mt = 2 * (pair0 + i * pair_step) + static_cast<int>(rank);
                int h0, b0;
                chain_origin(p, mt, h0, b0);
                for (int c = 0; c < p.n_chunks; ++c) {
                    if (!mbar_wait(bars.out_ready(stage), phase, ctl, kDevTimeoutProducer)) {
                        ok = false;
                        break;
                    }
                    X1CB_TRACE_AT(p.trace, 11, static_cast<long long>(i) * p.n_chunks + c);
                    const uint32_t src = sbase + p.off_r + stage * kRSlotBytes;
                    if (mt < p.num_m_tiles) {
                        if (p.io_swz)
                            tma_store_5d_hint(&tmO, src, 0, 0, h0, c * kRChunks, b0, pol);
                        else
                            tma_store_4d_hint(&tmO, src, 0, h0, c * kRChunks, b0, pol);
                        bulk_commit();
                        bulk_wait_read<0>();
                    }
                    X1CB_TRACE_AT(p.trace, 12, static_cast<long long>(i) * p.n_chunks + c);
                    mbar_arrive(kC3 ? bars.io_empty(stage) : bars.io_full(stage));
                    if (++stage == p.r_stages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            bulk_wait_all();
        }
        __syncwarp();
    } else if (warp == 1 || (!kC3 && warp == 2)) {
        // ---- MMA issuers (rank 0) ------------------------------------------------------
        if (leader && !kC3 && warp - 1 < p.issuers) {
            // The 3x3 alone: warp 1 issues the even pair tiles and warp 2 the odd
            // ones (one thread issues an MMA only every ~92 cycles, an M = 256,
            // N = 128 one takes 64 on the tensor pipe), each from its half of
            // the halo ring and into slots i % 4 (two per warp).
            const int mw = warp - 1;
            const int nw = p.issuers;                 // issuing warps: ring parts, tile step
            const int half = p.a_stages / nw;
            const uint32_t idesc = idesc_i8(256, 128);
            const uint64_t a_desc0 =
                smem_desc_rows16(sbase + p.off_a, static_cast<uint32_t>(p.a_half));
            const uint64_t w2_desc0 = smem_desc_sw32(sbase + p.off_w2);
            const uint32_t kb_step = (kHalfRows * 32) >> 4;
            const uint32_t a_slot_step = static_cast<uint32_t>(p.a_slot) >> 4;
            const uint32_t hp = static_cast<uint32_t>(p.row_pitch);
            // Descriptor offset of tap (dr, ds), units of 16 bytes: the row shift of
            // the framed tile; at stride 2 also the tap's phase plane.
            uint32_t tap_off[9];
#pragma unroll
            for (int t = 0; t < 9; ++t) {
                const uint32_t dr = t / 3, ds = t % 3;
                tap_off[t] = p.stride == 2 ? ((dr & 1) * 2 + (ds & 1)) * (2 * p.a_half >> 4) +
                                                 (dr >> 1) * hp + (ds >> 1)
                                           : dr * hp + ds;
            }
            const uint64_t ring_desc0 = a_desc0 + static_cast<uint64_t>(mw * half) * a_slot_step;
            int pos = 0;
            uint32_t ph = 0;
            uint64_t sd = ring_desc0;
            bool ok = __all_sync(0xffffffffu, mbar_wait_cl(bars.w_full(), 0, ctl, kDevTimeoutMma));
            for (int i = mw; ok && i < n_my; i += nw) {
                const int slot = i & 3;
                const uint32_t sph = static_cast<uint32_t>((i >> 2) & 1);
                if (!__all_sync(0xffffffffu, mbar_wait_cl(bars.acc_empty(slot), sph ^ 1u, ctl,
                                                          kDevTimeoutMma)))
                    break;
                if (lane == 0)
                    X1CB_TRACE_AT(p.trace, 2, i);
                tc_fence_after();
                const uint32_t d = tmem_base + static_cast<uint32_t>(slot * 128);
                for (int c1 = 0; c1 < p.C1; ++c1) {
                    const int st = mw * half + pos;
                    if (!__all_sync(0xffffffffu,
                                    mbar_wait_cl(bars.a_full(st), ph, ctl, kDevTimeoutMma))) {
                        ok = false;
                        break;
                    }
                    if (c1 == 0 && lane == 0)
                        X1CB_TRACE_AT(p.trace, 1, i);
                    tc_fence_after();
#pragma unroll
                    for (int t = 0; t < 9; ++t)
                        mma_i8_pair(d, sd + tap_off[t],
                                    w2_desc0 + static_cast<uint64_t>(t * p.C1 + c1) * kb_step,
                                    idesc, (c1 | t) ? 1u : 0u);
                    mma_commit_pair(bars.a_empty(st));
                    if (++pos == half) {
                        pos = 0;
                        ph ^= 1u;
                        sd = ring_desc0;
                    } else {
                        sd += a_slot_step;
                    }
                }
                if (!ok)
                    break;
                mma_commit_pair(bars.acc_full(slot));
                if (lane == 0)
                    X1CB_TRACE_AT(p.trace, 3, i);
            }
            mma_commit_pair(bars.mma_done());
            if (lane == 0 && !mbar_drain(bars.mma_done(), 0, drain_ns))
                atomicOr(dev_status, kDevDrainFailed);
        } else if (leader && kC3) {
            const uint32_t idesc = idesc_i8(256, 128);
            const uint64_t a_desc0 =
                smem_desc_rows16(sbase + p.off_a, static_cast<uint32_t>(p.a_half));
            const uint64_t w2_desc0 = smem_desc_sw32(sbase + p.off_w2);
            const uint64_t w3_desc0 = smem_desc_sw32(sbase + p.off_w3);
            const uint64_t a3_desc0 = smem_desc_rows16(sbase + p.off_a3, kA3Bytes / 8);
            const uint32_t kb_step = (kHalfRows * 32) >> 4;      // next K block of a weight half
            const uint32_t a_slot_step = static_cast<uint32_t>(p.a_slot) >> 4;
            const uint32_t a3_kb_step = (kA3Bytes / 4) >> 4;     // next K block of an A buffer
            const uint32_t a3_buf_step = kA3Bytes >> 4;
            const uint32_t hp = static_cast<uint32_t>(p.row_pitch);
            int st = 0;
            uint32_t ph = 0;
            uint64_t sd = a_desc0;
            int slot = 0;        // accumulator slot of the next item (Conv2 tile or Conv3 chunk)
            uint32_t sph = 0;    // and its use parity
            bool ok = __all_sync(0xffffffffu, mbar_wait_cl(bars.w_full(), 0, ctl, kDevTimeoutMma));
            if (lane == 0)
                X1CB_TRACE_AT(p.trace, 14, 0);
            for (int i = 0; ok && i <= n_my; ++i) {
                if (i < n_my) {
                    // Conv2 of pair tile i: 4 channel blocks x 9 taps into the next slot.
                    if (!__all_sync(0xffffffffu, mbar_wait_cl(bars.acc_empty(slot), sph ^ 1u, ctl,
                                                              kDevTimeoutMma))) {
                        ok = false;
                        break;
                    }
                    if (lane == 0)
                        X1CB_TRACE_AT(p.trace, 2, i);
                    tc_fence_after();
                    const uint32_t d = tmem_base + static_cast<uint32_t>(slot * 128);
                    for (int c1 = 0; c1 < p.C1; ++c1) {
                        if (!__all_sync(0xffffffffu, mbar_wait_cl(bars.a_full(st), ph, ctl,
                                                                  kDevTimeoutMma))) {
                            ok = false;
                            break;
                        }
                        if (c1 == 0 && lane == 0)
                            X1CB_TRACE_AT(p.trace, 1, i);
                        tc_fence_after();
#pragma unroll
                        for (int t = 0; t < 9; ++t)
                            mma_i8_pair(d, sd + (t / 3) * hp + (t % 3),
                                        w2_desc0 + static_cast<uint64_t>(t * p.C1 + c1) * kb_step,
                                        idesc, (c1 | t) ? 1u : 0u);
                        mma_commit_pair(bars.a_empty(st));
                        if (++st == p.a_stages) {
                            st = 0;
                            ph ^= 1u;
                            sd = a_desc0;
                        } else {
                            sd += a_slot_step;
                        }
                    }
                    if (!ok)
                        break;
                    mma_commit_pair(bars.acc_full(slot));
                    if (lane == 0)
                        X1CB_TRACE_AT(p.trace, 3, i);
                    if (++slot == kSlots) {
                        slot = 0;
                        sph ^= 1u;
                    }
                }
                if (kC3 && i >= 1) {
                    // Conv3 of pair tile i - 1: A = its Conv2 result (buffer (i-1) % 2),
                    // one 128-channel chunk per slot.
                    const int j = i - 1, b = j & 1;
                    if (!__all_sync(0xffffffffu, mbar_wait_cl(bars.a3_full(b), (j >> 1) & 1, ctl,
                                                              kDevTimeoutMma))) {
                        ok = false;
                        break;
                    }
                    if (lane == 0)
                        X1CB_TRACE_AT(p.trace, 4, j);
                    tc_fence_after();
                    const uint64_t ad = a3_desc0 + static_cast<uint64_t>(b) * a3_buf_step;
                    for (int c = 0; c < p.n_chunks; ++c) {
                        if (!__all_sync(0xffffffffu, mbar_wait_cl(bars.acc_empty(slot), sph ^ 1u,
                                                                  ctl, kDevTimeoutMma))) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t d = tmem_base + static_cast<uint32_t>(slot * 128);
                        for (int kb = 0; kb < p.C1; ++kb)
                            mma_i8_pair(d, ad + static_cast<uint64_t>(kb) * a3_kb_step,
                                        w3_desc0 +
                                            static_cast<uint64_t>(c * p.C1 + kb) * kb_step,
                                        idesc, kb ? 1u : 0u);
                        mma_commit_pair(bars.acc_full(slot));
                        if (lane == 0)
                            X1CB_TRACE_AT(p.trace, 5, static_cast<long long>(j) * p.n_chunks + c);
                        if (++slot == kSlots) {
                            slot = 0;
                            sph ^= 1u;
                        }
                    }
                    if (!ok)
                        break;
                    mma_commit_pair(bars.a3_empty(b));
                }
            }
            mma_commit_pair(bars.mma_done());
            if (lane == 0 && !mbar_drain(bars.mma_done(), 0, drain_ns))
                atomicOr(dev_status, kDevDrainFailed);
        }
        __syncwarp();
    } else {
        // ---- epilogue: items of the accumulator ring (see chain_epilogue) ---------------
        // One instantiation per pair of exact forms in use: the fast path keeps
        // its operands in registers (a form chosen at run time would share
        // arrays across forms and push them to local memory).
        const ChainEpi ce{&p, bars, ctl, tmem_base, smem, io_ticket, cm2, cc2, cm3, cc3, n_my,
                          mode2, mode3};
        const bool k1 = static_cast<long long>(p.m_r) == (1ll << (p.S - 1));
        if (!kC3) {
            if (mode2 == 2)
                conv2_epilogue<2>(ce, warp, lane);
            else
                conv2_epilogue<-1>(ce, warp, lane);
        } else if (mode2 == 2 && mode3 == 2 && k1) {
            chain_epilogue<2, 2, true>(ce, warp, lane);
        } else if (mode2 == 2 && mode3 == 2) {
            chain_epilogue<2, 2, false>(ce, warp, lane);
        } else {
            chain_epilogue<-1, -1, false>(ce, warp, lane);
        }
    }

    // ---- tear-down: neither CTA leaves while the other may still reach it ----------
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0)
        X1CB_TRACE_AT(p.trace, 15, 1);
    if (threadIdx.x == 0) {
        mbar_arrive_cluster(mapa_shared(bars.exit_bar(), rank ^ 1u));
        if (!mbar_drain(bars.exit_bar(), 0, 2 * p.wait_limit_ns + drain_ns))
            atomicOr(dev_status, kDevDrainFailed);
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}

}  // namespace

// ---- host side --------------------------------------------------------------

namespace {

// Plan of the CTA-pair kernel: c3 = fused Conv2 -> Conv3, else the 3x3 alone
// (Cout = Cm).
int plan_pair(ChainPlan &p, int B, int H, int W, int Cm, int Cout, int S, int m_r, bool c3,
              int stride = 1, int Hin = 0, int Win = 0)
{
    std::memset(&p, 0, sizeof(p));
    // (stride 2: the 3x3 alone, pad 1, output (Hin-1)/2+1 x (Win-1)/2+1, a
    // plane row of W+1 pixels within the 128 GEMM rows)
    if (stride != 1 && (c3 || stride != 2 || W + 1 > 126 || H != (Hin - 1) / 2 + 1 ||
                        W != (Win - 1) / 2 + 1))
        return X1CB_ERR_SHAPE;
    // One 128-channel Conv2 (its output is Conv3's whole K), a halo tile row
    // that fits the 128 GEMM rows, and output rows that the I/O maps can move
    // whole (4-pixel groups, or rows of at most 256 8-byte units).
    if ((!c3 && Cout != Cm) || Cm != 128 || Cout < 128 || Cout % 128 || Cout > 1024 || W + 2 > kTileRows || H < 1 ||
        W < 1 || B < 1)
        return X1CB_ERR_SHAPE;
    if (W % 4 != 0 && 4 * W > 256)
        return X1CB_ERR_SHAPE;
    p.c3 = c3 ? 1 : 0;
    p.stride = stride;
    p.Hin = stride == 2 ? Hin : H;
    p.Win = stride == 2 ? Win : W;
    p.B = B;
    p.H = H;
    p.W = W;
    p.Cm = Cm;
    p.Cout = Cout;
    p.S = S;
    p.m_r = m_r;
    p.C1 = Cm / 32;
    p.n_chunks = Cout / 128;
    if (stride == 2) {
        // th output rows of tg images; a plane is (th+1) x (W+1) pixels, GEMM
        // row m = (g*(th+1) + y)*(W+1) + x; fewest tiles, ties to taller ones
        const int pitch = W + 1;
        long long best = -1;
        p.th = p.tg = 1;
        for (int h = 1; h <= H; ++h)
            for (int g = 1; g <= B; ++g) {
                const long long last = static_cast<long long>(g - 1) * (h + 1) * pitch +
                                       static_cast<long long>(h - 1) * pitch + (W - 1);
                if (last >= kTileRows)
                    break;
                const long long t = static_cast<long long>((H + h - 1) / h) * ((B + g - 1) / g);
                if (best < 0 || t < best || (t == best && h > p.th)) {
                    best = t;
                    p.th = h;
                    p.tg = g;
                }
            }
        p.tw = W;
        p.row_pitch = pitch;
        p.plane_m = (p.th + 1) * pitch;
        const int need_rows = std::max(p.tg * p.plane_m, kTileRows + pitch + 1);
        p.a_half = ((need_rows + 7) / 8) * 8 * 16;
        p.a_slot = (8 * p.a_half + 1023) / 1024 * 1024;  // four planes of two K halves
    } else {
        choose_halo_tile(B, H, W, p.th, p.tg);
        p.tw = W;
        p.row_pitch = W + 2;
        p.plane_m = (p.th + 2) * (W + 2);
        const int need_rows = std::max(p.tg * p.plane_m, kTileRows + 2 * p.row_pitch + 2);
        p.a_half = ((need_rows + 7) / 8) * 8 * 16;
        p.a_slot = (2 * p.a_half + 1023) / 1024 * 1024;
    }
    p.rows = p.tw * p.th * p.tg;
    p.nTh = (H + p.th - 1) / p.th;
    p.nTg = (B + p.tg - 1) / p.tg;
    const long long tiles = static_cast<long long>(p.nTh) * p.nTg;
    if (tiles > INT_MAX / 4)
        return X1CB_ERR_SHAPE;
    p.num_m_tiles = static_cast<int>(tiles);
    p.n_pairs = (p.num_m_tiles + 1) / 2;
    p.io_swz = W % 4 == 0 ? 1 : 0;

    const int w2_bytes = 9 * p.C1 * kHalfRows * 32;
    const int w3_bytes = c3 ? p.n_chunks * p.C1 * kHalfRows * 32 : 0;
    auto layout = [&](int a, int r) {
        p.a_stages = a;
        p.r_stages = r;
        p.off_w2 = 0;
        p.off_w3 = w2_bytes;
        p.off_a3 = (p.off_w3 + w3_bytes + 1023) / 1024 * 1024;
        p.off_a = p.off_a3 + (c3 ? kA3Bufs * kA3Bytes : 0);
        p.off_r = p.off_a + a * p.a_slot;
        p.off_cm2 = p.off_r + r * kRSlotBytes;
        p.off_cc2 = p.off_cm2 + p.Cm * 4;
        p.off_cm3 = p.off_cc2 + p.Cm * 8;
        p.off_cc3 = p.off_cm3 + p.Cout * 4;
        p.off_bar = (p.off_cc3 + p.Cout * 8 + 7) & ~7;
        p.off_misc = p.off_bar + ChainBars::count(a, r) * 8;
        p.smem_bytes = p.off_misc + 16 + 1024;
        return p.smem_bytes <= kSmemLimit;
    };
    bool placed = false;
    if (c3) {
        // Deepest shortcut ring beside at least four halo slots (fewer if needed).
        for (int a = 4; a >= 2 && !placed; --a)
            for (int r = 8; r >= 2 && !placed; --r)
                placed = layout(a, r);
    } else {
        // The 3x3 alone holds half its weights per CTA (72 KB) and no Conv3
        // operands: a deep halo ring (up to four tiles of channel blocks, an
        // even number: half for each MMA warp) beside output stages for each
        // epilogue turn.  At stride 2 a channel block's four planes take
        // 20 KB: one issuing warp over the whole ring, the ring first, then
        // the stages (measured on the Res3.1 conv2, B = 256: two issuers with
        // two 20 KB slots each 69.2 us against 64.7 on one SM per tile; one
        // issuer with five slots and three stages 47.5 us, 47.5 with two
        // stages, 48.8-48.9 with four slots).
        p.issuers = stride == 2 ? 1 : 2;
        if (stride == 2)
            for (int a = 16; a >= 4 && !placed; --a)
                for (int r = kSlots - 1; r >= 2 && !placed; --r)
                    placed = layout(a, r);
        for (int r = kSlots; r >= 2 && !placed; --r)
            for (int a = 16; a >= 4 && !placed; a -= 2)
                placed = layout(a, r);
    }
    if (!placed)
        return X1CB_ERR_SHAPE;
    p.grid = 2 * std::max(1, std::min(74, p.n_pairs));
    p.wait_limit_ns = 2000000000ull;
    return X1CB_OK;
}

}  // namespace

int plan_chain(ChainPlan &p, int B, int H, int W, int Cm, int Cout, int S, int m_r)
{
    return plan_pair(p, B, H, W, Cm, Cout, S, m_r, true);
}

int plan_conv2_pair(ChainPlan &p, int B, int H, int W, int S, int stride, int Hin, int Win)
{
    return plan_pair(p, B, H, W, 128, 128, S, 0, false, stride, Hin, Win);
}

// Clusters of two CTAs of chain23_kernel that fit on the current device at
// once with `smem` bytes of shared memory each (cached per device and size).
int resident_clusters(int smem, int &clusters, bool c3)
{
    static std::mutex mu;
    static int cached[2][64] = {}, cached_smem[2][64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return X1CB_ERR_CUDA;
    const int k = c3 ? 1 : 0;
    auto kern = c3 ? chain23_kernel<true> : chain23_kernel<false>;
    std::lock_guard<std::mutex> lk(mu);
    if (cached[k][dev] == 0 || cached_smem[k][dev] != smem) {
        if (int e = opt_in_smem(reinterpret_cast<const void *>(kern), c3 ? 2 : 5))
            return e;
        cudaLaunchConfig_t cfg;
        std::memset(&cfg, 0, sizeof(cfg));
        cfg.gridDim = dim3(2, 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
            cudaGetLastError();
            return X1CB_ERR_CUDA;
        }
        cached[k][dev] = n;
        cached_smem[k][dev] = smem;
    }
    clusters = cached[k][dev];
    return X1CB_OK;
}

int launch_chain(const ChainPlan &p, const int8_t *y1, const int8_t *w2, const int32_t *b2,
                 const int32_t *m2, const int8_t *w3, const int32_t *b3, const int32_t *m3,
                 const int8_t *x, int8_t *out, cudaStream_t stream)
{
    CUtensorMap tmA, tmW2, tmW3, tmR, tmO;
    if (p.stride == 2) {
        // Stride-2 planes: dims (32, Win, Hin, C1, B) at traversal step 2; a box
        // of (2(W+1), 2(th+1)) elements lands one (W+1) x (th+1) plane.
        const uint64_t dims[5] = {32, (uint64_t)p.Win, (uint64_t)p.Hin, (uint64_t)p.C1,
                                  (uint64_t)p.B};
        const uint64_t str[4] = {32, (uint64_t)p.Win * 32, (uint64_t)p.Hin * p.Win * 32,
                                 (uint64_t)p.C1 * p.Hin * p.Win * 32};
        const uint32_t box[5] = {16, (uint32_t)(2 * p.row_pitch), (uint32_t)(2 * (p.th + 1)), 1,
                                 (uint32_t)p.tg};
        const uint32_t es[5] = {1, 2, 2, 1, 1};
        if (int e = encode_map(&tmA, y1, 5, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE,
                               CU_TENSOR_MAP_DATA_TYPE_UINT8, es))
            return e;
    } else {  // Conv2 input, halo form: dims (32, W, H, C1, B), box (16, W+2, th+2, 1, tg)
        const uint64_t dims[5] = {32, (uint64_t)p.W, (uint64_t)p.H, (uint64_t)p.C1,
                                  (uint64_t)p.B};
        const uint64_t str[4] = {32, (uint64_t)p.W * 32, (uint64_t)p.H * p.W * 32,
                                 (uint64_t)p.C1 * p.H * p.W * 32};
        const uint32_t box[5] = {16, (uint32_t)p.row_pitch, (uint32_t)(p.th + 2), 1,
                                 (uint32_t)p.tg};
        if (int e = encode_map(&tmA, y1, 5, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE))
            return e;
    }
    {  // Conv2 weights [1][9*C1][128][32]: one CTA's half = 64 rows of a K block
        const uint64_t dims[4] = {32, 128, (uint64_t)(9 * p.C1), 1};
        const uint64_t str[3] = {32, 4096, (uint64_t)(9 * p.C1) * 4096};
        const uint32_t box[4] = {32, kHalfRows, 1, 1};
        if (int e = encode_map(&tmW2, w2, 4, dims, str, box, CU_TENSOR_MAP_SWIZZLE_32B))
            return e;
    }
    if (p.c3) {  // Conv3 weights [Cout/128][C1][128][32]
        const uint64_t dims[4] = {32, 128, (uint64_t)p.C1, (uint64_t)p.n_chunks};
        const uint64_t str[3] = {32, 4096, (uint64_t)p.C1 * 4096};
        const uint32_t box[4] = {32, kHalfRows, 1, 1};
        if (int e = encode_map(&tmW3, w3, 4, dims, str, box, CU_TENSOR_MAP_SWIZZLE_32B))
            return e;
    } else {
        tmW3 = tmW2;  // unused
    }
    const uint64_t O1 = p.Cout / 32;
    if (p.io_swz) {  // 128-byte rows of 4 pixels: (16 x 8 B, W/4, H, O1, B)
        const uint64_t dims[5] = {16, (uint64_t)p.W / 4, (uint64_t)p.H, O1, (uint64_t)p.B};
        const uint64_t str[4] = {128, (uint64_t)p.W * 32, (uint64_t)p.H * p.W * 32,
                                 O1 * p.H * p.W * 32};
        const uint32_t box[5] = {16, (uint32_t)p.W / 4, (uint32_t)p.th, (uint32_t)kRChunks,
                                 (uint32_t)p.tg};
        if (int e = encode_map(&tmO, out, 5, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B,
                               CU_TENSOR_MAP_DATA_TYPE_UINT64))
            return e;
        if (!p.c3)
            tmR = tmO;  // unused
        else if (int e = encode_map(&tmR, x, 5, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B,
                                    CU_TENSOR_MAP_DATA_TYPE_UINT64))
            return e;
    } else {  // whole rows of W*32 bytes as 8-byte units: (4W, H, O1, B)
        const uint64_t dims[4] = {(uint64_t)p.W * 4, (uint64_t)p.H, O1, (uint64_t)p.B};
        const uint64_t str[3] = {(uint64_t)p.W * 32, (uint64_t)p.H * p.W * 32,
                                 O1 * p.H * p.W * 32};
        const uint32_t box[4] = {(uint32_t)p.W * 4, (uint32_t)p.th, (uint32_t)kRChunks,
                                 (uint32_t)p.tg};
        if (int e = encode_map(&tmO, out, 4, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE,
                               CU_TENSOR_MAP_DATA_TYPE_UINT64))
            return e;
        if (!p.c3)
            tmR = tmO;  // unused
        else if (int e = encode_map(&tmR, x, 4, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE,
                                    CU_TENSOR_MAP_DATA_TYPE_UINT64))
            return e;
    }
    auto kern = p.c3 ? chain23_kernel<true> : chain23_kernel<false>;
    if (int e = opt_in_smem(reinterpret_cast<const void *>(kern), p.c3 ? 2 : 5))
        return e;
    // The kernel is persistent with a static assignment of pair tiles, so it
    // must not launch more clusters than can be resident at once: a cluster
    // needs two SMs of one GPC, and a GPC with an odd number of free SMs
    // leaves one over.
    int clusters = 0;
    if (int e = resident_clusters(p.smem_bytes, clusters, p.c3 != 0))
        return e;
    const int grid = 2 * std::max(1, std::min(clusters, p.n_pairs));
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = p.smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // a programmatic dependent of the preceding kernel (see the kernel's
    // griddep_wait)
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    unsigned int *dev_status = nullptr, *dev_forms = nullptr;
    if (int e = device_words(&dev_status, &dev_forms))
        return e;
    ChainPlan q = p;
    q.trace = trace_table();
    if (cudaLaunchKernelEx(&cfg, kern, tmA, tmW2, tmW3, tmR, tmO, b2, m2, b3, m3,
                           dev_status, dev_forms, q) != cudaSuccess)
        return X1CB_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? X1CB_OK : X1CB_ERR_CUDA;
}

}  // namespace x1cb
