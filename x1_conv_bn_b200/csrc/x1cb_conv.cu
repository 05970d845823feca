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
//  * one persistent CTA per SM, 12 warps, warp-specialised:
//      warp 0      TMA producer: weights (once, resident in shared memory) and
//                  the activation tiles (one 128-row x 32-byte K block per slot)
//      warp 1      MMA issuer: tcgen05.mma.kind::i8 into TMEM (int32), owner
//                  of the TMEM allocation
//      warp 2      TMA producer: shortcut (residual) tiles, far ahead of use
//      warps 4-11  epilogue: tcgen05.ld, exact int64 requantisation, 16-byte
//                  stores of NC/32HW32 output straight from registers
//  * a tile is 128 GEMM rows = tw x th pixels of tg images, chosen per shape
//    so that whole TMA boxes cover the image (16 px x 8 images for 28x28 1x1)
//  * TMEM holds 512 int32 columns; the accumulator ring lets the MMA of the
//    next tile run while the epilogue drains the previous one
//  * every wait is bounded; on timeout the CTA raises an abort flag, records
//    a status bit, lets in-flight copies and MMAs land, frees TMEM, and exits.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <climits>
#include <cstdint>
#include <cstring>

#include "x1cb_internal.h"
#include "x1cb_plan.h"
#include "x1cb_ptx.cuh"

namespace x1cb {

// Sticky device status word (timeouts).  Read and cleared by the API.
__device__ unsigned int g_dev_status;

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
    __device__ uint32_t r_full(int s) const { return at(3 + 2 * a_stages + s); }
    __device__ uint32_t r_empty(int s) const { return at(3 + 2 * a_stages + r_stages + s); }
    __device__ uint32_t acc_full(int s) const { return at(3 + 2 * a_stages + 2 * r_stages + s); }
    __device__ uint32_t acc_empty(int s) const
    {
        return at(3 + 2 * a_stages + 2 * r_stages + 4 + s);
    }
    static int count(int a, int r) { return 3 + 2 * a + 2 * r + 8; }
};

__device__ __forceinline__ void tile_origin(const ConvPlan &p, int mt, int &w0, int &h0, int &b0)
{
    const int iw = mt % p.nTw;
    const int ih = (mt / p.nTw) % p.nTh;
    const int ig = mt / (p.nTw * p.nTh);
    w0 = iw * p.tw;
    h0 = ih * p.th;
    b0 = ig * p.tg;
}

// Requantise 32 accumulators of one pixel (channels n0..n0+31 of this CTA's
// group) and pack them as 32 int8 bytes.
template <bool kRes>
__device__ __forceinline__ void requant32(const uint32_t (&v)[32], const int32_t *cm,
                                          const long long *cC, const uint32_t (&rw)[8],
                                          int m_r, int S, uint32_t (&ow)[8])
{
#pragma unroll
    for (int q = 0; q < 8; ++q)
        ow[q] = 0u;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
        long long t = static_cast<long long>(static_cast<int>(v[k])) * cm[k] + cC[k];
        if (kRes) {
            const int r = static_cast<int>(static_cast<int8_t>((rw[k >> 2] >> (8 * (k & 3))) & 0xFF));
            t += static_cast<long long>(r) * m_r;
        }
        const long long y = t >> S;  // arithmetic shift: floor(t / 2^S)
        const int yc = y < 0 ? 0 : (y > 127 ? 127 : static_cast<int>(y));
        ow[k >> 2] |= static_cast<uint32_t>(yc) << (8 * (k & 3));
    }
}

template <bool kRes>
__global__ void __launch_bounds__(kThreads, 1)
    conv_bn_act_kernel(const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmW,
                       const __grid_constant__ CUtensorMap tmR, int8_t *__restrict__ out,
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
    Bars bars{sbase + static_cast<uint32_t>(p.off_bar), p.a_stages, p.r_stages};
    const WaitCtl ctl{abort_flag, &g_dev_status, p.wait_limit_ns};
    const uint64_t drain_ns = 200000000ull;  // 0.2 s for copies/MMAs already issued

    const int group = blockIdx.x % p.n_groups;
    const int mt_first = blockIdx.x / p.n_groups;
    const int mt_step = gridDim.x / p.n_groups;

    // ---- set-up ---------------------------------------------------------------
    if (threadIdx.x == 0) {
        *abort_flag = 0;
        mbar_init(bars.w_full(), 1);
        mbar_init(bars.mma_done(), 1);
        mbar_init(bars.never(), 1);
        for (int s = 0; s < p.a_stages; ++s) {
            mbar_init(bars.a_full(s), 1);
            mbar_init(bars.a_empty(s), 1);
        }
        for (int s = 0; s < p.r_stages; ++s) {
            mbar_init(bars.r_full(s), 1);
            mbar_init(bars.r_empty(s), kEpiWarps);
        }
        for (int s = 0; s < 4; ++s) {
            mbar_init(bars.acc_full(s), 1);
            mbar_init(bars.acc_empty(s), kEpiWarps);
        }
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmW);
        if (kRes)
            tma_prefetch_desc(&tmR);
    }
    // Folded-BN constants of this CTA's channels: C = bias*m + 2^(S-1), so
    // that t = acc*m + C (+ r*m_r) needs one wide multiply-add per term.
    for (int n = threadIdx.x; n < p.NC; n += blockDim.x) {
        const int o = group * p.NC + n;
        const long long mm = mult[o];
        cm[n] = static_cast<int32_t>(mm);
        cC[n] = static_cast<long long>(bias[o]) * mm + (1ll << (p.S - 1));
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ---- producer: resident weights, then activation K blocks ---------------
        if (lane == 0) {
            const uint32_t sw = sbase + p.off_w;
            const uint32_t wbytes = static_cast<uint32_t>(p.kb_per_tile * p.NC * 32);
            mbar_arrive_expect_tx(bars.w_full(), wbytes);
            for (int kb = 0; kb < p.kb_per_tile; ++kb)
                tma_load_4d(sw + kb * p.NC * 32, &tmW, bars.w_full(), 0, 0, kb,
                            group * (p.NC / 128));
            const uint32_t abytes = static_cast<uint32_t>(p.rows * 32);
            const uint32_t sa = sbase + p.off_a;
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            bool ok = true;
            for (int mt = mt_first; ok && mt < p.num_m_tiles; mt += mt_step) {
                int w0, h0, b0;
                tile_origin(p, mt, w0, h0, b0);
                for (int kb = 0; kb < p.kb_per_tile; ++kb) {
                    const int tap = kb / p.C1, c1 = kb % p.C1;
                    const int dr = tap / p.R, ds = tap % p.R;
                    if (!mbar_wait(bars.a_empty(stage), phase ^ 1u, ctl, kDevTimeoutProducer)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(bars.a_full(stage), abytes);
                    tma_load_5d(sa + stage * kASlotBytes, &tmA, bars.a_full(stage), 0,
                                w0 + ds - p.pad, h0 + dr - p.pad, c1, b0);
                    ++issued;
                    if (++stage == p.a_stages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // Let every copy still in flight land before shared memory goes away.
            if (!mbar_drain(bars.w_full(), 0, drain_ns))
                atomicOr(&g_dev_status, kDevDrainFailed);
            const long long last = issued < p.a_stages ? issued : p.a_stages;
            for (long long i = issued - last; i < issued; ++i) {
                const int s = static_cast<int>(i % p.a_stages);
                const uint32_t ph = static_cast<uint32_t>((i / p.a_stages) & 1);
                if (!mbar_drain(bars.a_full(s), ph, drain_ns))
                    atomicOr(&g_dev_status, kDevDrainFailed);
            }
        }
        __syncwarp();
    } else if (warp == 2) {
        // ---- producer: shortcut tiles (issued as early as the ring allows) ------
        if (kRes && lane == 0) {
            const uint32_t rbytes = static_cast<uint32_t>(kRChunks * p.rows * 32);
            const uint32_t sr = sbase + p.off_r;
            const int stages_per_tile = p.NC / (32 * kRChunks);
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            bool ok = true;
            for (int mt = mt_first; ok && mt < p.num_m_tiles; mt += mt_step) {
                int w0, h0, b0;
                tile_origin(p, mt, w0, h0, b0);
                for (int rs = 0; rs < stages_per_tile; ++rs) {
                    if (!mbar_wait(bars.r_empty(stage), phase ^ 1u, ctl, kDevTimeoutProducer)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(bars.r_full(stage), rbytes);
                    tma_load_5d(sr + stage * kRSlotBytes, &tmR, bars.r_full(stage), 0, w0, h0,
                                group * (p.NC / 32) + rs * kRChunks, b0);
                    ++issued;
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
                if (!mbar_drain(bars.r_full(s), ph, drain_ns))
                    atomicOr(&g_dev_status, kDevDrainFailed);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---- MMA issuer -----------------------------------------------------------
        if (lane == 0) {
            const uint32_t idesc = idesc_i8(kTileRows, p.nmma);
            const uint32_t sa = sbase + p.off_a;
            const uint32_t sw = sbase + p.off_w;
            const int n_slots = kTmemCols / p.nmma;
            int a_stage = 0;
            uint32_t a_phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = mbar_wait(bars.w_full(), 0, ctl, kDevTimeoutMma);
            if (ok && p.inject == 1)
                ok = mbar_wait(bars.never(), 0, ctl, kDevTimeoutMma);  // test hook
            for (int mt = mt_first; ok && mt < p.num_m_tiles; mt += mt_step) {
                int st = a_stage;
                uint32_t ph = a_phase;
                for (int j = 0; ok && j < p.n_subs; ++j) {
                    if (!mbar_wait(bars.acc_empty(acc), acc_phase ^ 1u, ctl, kDevTimeoutMma)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * p.nmma);
                    st = a_stage;
                    ph = a_phase;
                    for (int kb = 0; kb < p.kb_per_tile; ++kb) {
                        if (j == 0) {
                            if (!mbar_wait(bars.a_full(st), ph, ctl, kDevTimeoutMma)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                        }
                        const uint64_t adesc = smem_desc_sw32(sa + st * kASlotBytes);
                        const uint64_t bdesc =
                            smem_desc_sw32(sw + (kb * p.NC + j * p.nmma) * 32);
                        mma_i8(d_tmem, adesc, bdesc, idesc, kb > 0 ? 1u : 0u);
                        if (j == p.n_subs - 1)
                            mma_commit(bars.a_empty(st));  // slot free once these MMAs finish
                        if (++st == p.a_stages) {
                            st = 0;
                            ph ^= 1u;
                        }
                    }
                    if (!ok)
                        break;
                    mma_commit(bars.acc_full(acc));
                    if (++acc == n_slots) {
                        acc = 0;
                        acc_phase ^= 1u;
                    }
                }
                a_stage = st;
                a_phase = ph;
            }
            // Make sure no MMA is still reading shared memory or writing TMEM.
            mma_commit(bars.mma_done());
            if (!mbar_drain(bars.mma_done(), 0, drain_ns))
                atomicOr(&g_dev_status, kDevDrainFailed);
        }
        __syncwarp();
    } else if (warp >= kEpiWarp0) {
        // ---- epilogue ---------------------------------------------------------------
        const int q = warp & 3;           // TMEM lane quarter this warp may access
        const int half = (warp - kEpiWarp0) >> 2;  // which chunks of a stage
        const int row = q * 32 + lane;    // GEMM row = pixel of the tile
        const int plane_t = p.tw * p.th;
        const int xi = row % p.tw;
        const int yi = (row / p.tw) % p.th;
        const int gi = row / plane_t;
        const bool in_box = row < p.rows;
        const long long HWp = static_cast<long long>(p.Hp) * p.Wp;
        const int n_slots = kTmemCols / p.nmma;
        const int stages_per_sub = p.nmma / (32 * kRChunks);
        const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
        const uint8_t *sr = smem + p.off_r;
        int acc = 0;
        uint32_t acc_phase = 0;
        int r_stage = 0;
        uint32_t r_phase = 0;
        bool ok = true;
        for (int mt = mt_first; ok && mt < p.num_m_tiles; mt += mt_step) {
            int w0, h0, b0;
            tile_origin(p, mt, w0, h0, b0);
            const int b = b0 + gi, hh = h0 + yi, ww = w0 + xi;
            const bool valid = in_box && b < p.B && hh < p.Hp && ww < p.Wp;
            const long long pix_off =
                (static_cast<long long>(b) * p.O1 * HWp + static_cast<long long>(hh) * p.Wp + ww) *
                32;
            for (int j = 0; ok && j < p.n_subs; ++j) {
                // Every lane waits; the vote keeps the warp's decision uniform so
                // that the .sync.aligned TMEM loads below always run converged.
                if (!__all_sync(0xffffffffu,
                                mbar_wait(bars.acc_full(acc), acc_phase, ctl, kDevTimeoutEpilogue))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int rl = 0; rl < stages_per_sub; ++rl) {
                    if (kRes && !__all_sync(0xffffffffu, mbar_wait(bars.r_full(r_stage), r_phase,
                                                                   ctl, kDevTimeoutEpilogue))) {
                        ok = false;
                        break;
                    }
#pragma unroll 1
                    for (int c = half; c < kRChunks; c += 2) {
                        const int cs = rl * kRChunks + c;           // chunk within the sub
                        const int gch = j * (p.nmma / 32) + cs;     // chunk within the group
                        uint32_t v[32];
                        __syncwarp();
                        tmem_ld_32x32b_x32(tmem_base + lane_addr +
                                               static_cast<uint32_t>(acc * p.nmma + cs * 32),
                                           v);
                        tmem_wait_ld(v);
                        if (valid) {
                            uint32_t rw[8];
                            if (kRes) {
                                const uint4 *rp = reinterpret_cast<const uint4 *>(
                                    sr + r_stage * kRSlotBytes +
                                    ((gi * kRChunks + c) * plane_t + yi * p.tw + xi) * 32);
                                const uint4 ra = rp[0], rb = rp[1];
                                rw[0] = ra.x; rw[1] = ra.y; rw[2] = ra.z; rw[3] = ra.w;
                                rw[4] = rb.x; rw[5] = rb.y; rw[6] = rb.z; rw[7] = rb.w;
                            } else {
#pragma unroll
                                for (int k = 0; k < 8; ++k)
                                    rw[k] = 0u;
                            }
                            uint32_t ow[8];
                            requant32<kRes>(v, cm + gch * 32, cC + gch * 32, rw, p.m_r, p.S, ow);
                            const int o1 = group * (p.NC / 32) + gch;
                            uint4 *op = reinterpret_cast<uint4 *>(
                                out + pix_off + static_cast<long long>(o1) * HWp * 32);
                            op[0] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                            op[1] = make_uint4(ow[4], ow[5], ow[6], ow[7]);
                        }
                    }
                    if (kRes) {
                        __syncwarp();
                        if (lane == 0)
                            mbar_arrive(bars.r_empty(r_stage));
                        if (++r_stage == p.r_stages) {
                            r_stage = 0;
                            r_phase ^= 1u;
                        }
                    }
                }
                if (!ok)
                    break;
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(bars.acc_empty(acc));
                if (++acc == n_slots) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
        }
        __syncwarp();
    }

    // ---- tear-down ---------------------------------------------------------------
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

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

int encode_map(CUtensorMap *m, const void *base, int rank, const uint64_t *dims,
               const uint64_t *strides_bytes, const uint32_t *box, CUtensorMapSwizzle swz)
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
        es[i] = 1;
    }
    for (int i = 0; i < rank - 1; ++i)
        s[i] = strides_bytes[i];
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, static_cast<cuuint32_t>(rank),
                    const_cast<void *>(base), d, s, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? X1CB_OK : X1CB_ERR_CUDA;
}

}  // namespace

// Choose the pixel tile: tw x th pixels of tg images, at most 128 GEMM rows.
// Cost = MMA rows issued over the whole problem, with a mild penalty for
// contiguous global runs shorter than 512 bytes; ties go to more rows, then
// to longer runs.
void choose_tile(int B, int Wp, int Hp, int &tw, int &th, int &tg)
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
                cost *= 1.0 + (512 - seg) / 4096.0;
            const int rows = w * h * g;
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

int plan_conv(ConvPlan &p, int B, int H, int W, int Ic, int Oc, int R, int has_res, int S,
              int m_r, int num_sms)
{
    std::memset(&p, 0, sizeof(p));
    p.B = B;
    p.H = H;
    p.W = W;
    p.Ic = Ic;
    p.Oc = Oc;
    p.R = R;
    p.pad = (R - 1) / 2;
    p.C1 = Ic / 32;
    p.O1 = Oc / 32;
    p.has_res = has_res;
    p.S = S;
    p.m_r = m_r;
    if (R == 1) {
        p.Wp = H * W;
        p.Hp = 1;
    } else {
        p.Wp = W;
        p.Hp = H;
    }
    choose_tile(B, p.Wp, p.Hp, p.tw, p.th, p.tg);
    p.rows = p.tw * p.th * p.tg;
    p.nTw = (p.Wp + p.tw - 1) / p.tw;
    p.nTh = (p.Hp + p.th - 1) / p.th;
    p.nTg = (B + p.tg - 1) / p.tg;
    const long long mtiles = static_cast<long long>(p.nTw) * p.nTh * p.nTg;
    if (mtiles > INT_MAX / 2)
        return X1CB_ERR_SHAPE;
    p.num_m_tiles = static_cast<int>(mtiles);
    p.kb_per_tile = R * R * p.C1;

    const int fixed = 1024 /*alignment slack*/ + 64 /*misc*/ + Bars::count(48, 8) * 8 + 64;
    int chosen = 0;
    long long chosen_work = -1;
    for (int NC = std::min(Oc, 512); NC >= 128; NC -= 128) {
        if (Oc % NC)
            continue;
        const int nmma = NC >= 256 ? 256 : 128;
        const int n_subs = NC / nmma;
        const int a_min = n_subs > 1 ? p.kb_per_tile + 2 : 4;
        const int r_min = has_res ? 4 : 0;
        const long long need = static_cast<long long>(p.kb_per_tile) * NC * 32 + NC * 12 +
                               a_min * kASlotBytes + r_min * kRSlotBytes + fixed;
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
    if (chosen == 0)
        return X1CB_ERR_SHAPE;  // weights of 128 output channels do not fit on chip
    p.NC = chosen;
    p.n_groups = Oc / p.NC;
    p.nmma = p.NC >= 256 ? 256 : 128;
    p.n_subs = p.NC / p.nmma;

    const int wbytes = p.kb_per_tile * p.NC * 32;
    const int a_min = p.n_subs > 1 ? p.kb_per_tile + 2 : 4;
    const int rem = kSmemLimit - fixed - wbytes - p.NC * 12;
    // Split what is left between the two rings: the activation ring first gets
    // a tile's K blocks plus a few (capped), the shortcut ring the rest.
    const int a_want = std::max(a_min, std::min(p.kb_per_tile + 4, 12));
    if (has_res) {
        p.r_stages = std::max(4, std::min(8, (rem - a_want * kASlotBytes) / kRSlotBytes));
        p.a_stages = std::max(a_min, std::min(48, (rem - p.r_stages * kRSlotBytes) / kASlotBytes));
    } else {
        p.r_stages = 0;
        p.a_stages = std::max(a_min, std::min(48, rem / kASlotBytes));
    }

    p.off_w = 0;
    p.off_a = p.off_w + wbytes;
    p.off_r = p.off_a + p.a_stages * kASlotBytes;
    p.off_cc = p.off_r + p.r_stages * kRSlotBytes;
    p.off_cm = p.off_cc + p.NC * 8;
    p.off_bar = (p.off_cm + p.NC * 4 + 7) & ~7;
    p.off_misc = p.off_bar + Bars::count(p.a_stages, p.r_stages) * 8;
    p.smem_bytes = p.off_misc + 16 + 1024;
    if (p.smem_bytes > kSmemLimit)
        return X1CB_ERR_SHAPE;

    const long long work = mtiles * p.n_groups;
    long long grid = std::min<long long>(num_sms, work);
    grid = (grid / p.n_groups) * p.n_groups;
    if (grid < p.n_groups)
        grid = p.n_groups;
    p.grid = static_cast<int>(grid);
    p.wait_limit_ns = 2000000000ull;
    return X1CB_OK;
}

int launch_conv(const ConvPlan &p, const int8_t *x, const int8_t *w, const int32_t *bias,
                const int32_t *mult, const int8_t *r, int8_t *out, cudaStream_t stream)
{
    CUtensorMap tmA, tmW, tmR;
    // Activations: dims (32 ch, Wp, Hp, C1, B); box (32, tw, th, 1, tg).
    {
        const uint64_t dims[5] = {32, (uint64_t)p.Wp, (uint64_t)p.Hp, (uint64_t)p.C1,
                                  (uint64_t)p.B};
        const uint64_t str[4] = {32, (uint64_t)p.Wp * 32, (uint64_t)p.Hp * p.Wp * 32,
                                 (uint64_t)p.C1 * p.Hp * p.Wp * 32};
        const uint32_t box[5] = {32, (uint32_t)p.tw, (uint32_t)p.th, 1, (uint32_t)p.tg};
        if (int e = encode_map(&tmA, x, 5, dims, str, box, CU_TENSOR_MAP_SWIZZLE_32B))
            return e;
    }
    // Weights [Oc/128][KB][128][32]: dims (32, 128, KB, Oc/128); box (32,128,1,NC/128).
    {
        const uint64_t dims[4] = {32, 128, (uint64_t)p.kb_per_tile, (uint64_t)(p.Oc / 128)};
        const uint64_t str[3] = {32, 4096, (uint64_t)p.kb_per_tile * 4096};
        const uint32_t box[4] = {32, 128, 1, (uint32_t)(p.NC / 128)};
        if (int e = encode_map(&tmW, w, 4, dims, str, box, CU_TENSOR_MAP_SWIZZLE_32B))
            return e;
    }
    if (p.has_res) {
        // Shortcut: dims (32, Wp, Hp, O1, B); box (32, tw, th, 4, tg), no swizzle.
        const uint64_t dims[5] = {32, (uint64_t)p.Wp, (uint64_t)p.Hp, (uint64_t)p.O1,
                                  (uint64_t)p.B};
        const uint64_t str[4] = {32, (uint64_t)p.Wp * 32, (uint64_t)p.Hp * p.Wp * 32,
                                 (uint64_t)p.O1 * p.Hp * p.Wp * 32};
        const uint32_t box[5] = {32, (uint32_t)p.tw, (uint32_t)p.th, (uint32_t)kRChunks,
                                 (uint32_t)p.tg};
        if (int e = encode_map(&tmR, r, 5, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE))
            return e;
    } else {
        tmR = tmA;  // unused
    }
    auto kern = p.has_res ? conv_bn_act_kernel<true> : conv_bn_act_kernel<false>;
    static bool attr_set[2] = {false, false};
    if (!attr_set[p.has_res]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit) !=
            cudaSuccess)
            return X1CB_ERR_CUDA;
        attr_set[p.has_res] = true;
    }
    kern<<<p.grid, kThreads, p.smem_bytes, stream>>>(tmA, tmW, tmR, out, bias, mult, p);
    return cudaGetLastError() == cudaSuccess ? X1CB_OK : X1CB_ERR_CUDA;
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

}  // namespace x1cb
