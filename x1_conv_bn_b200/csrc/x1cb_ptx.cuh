// Thin inline-PTX wrappers for sm_100a: mbarriers (with bounded waits), TMA
// tensor loads, tcgen05 MMA / TMEM.  Device-only; included by the kernels.
#pragma once
#include <cstdint>
#include <cuda.h>

namespace x1cb {

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---- mbarrier ---------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Control block shared by every wait of one CTA: a CTA-wide abort flag in
// shared memory, the wait limit, and the device status word to report into.
struct WaitCtl {
    volatile int *abort_flag;  // shared memory
    unsigned int *status;      // global status word (sticky bits)
    uint64_t limit_ns;
};

// As mbar_try_wait, but a thread whose phase is not complete is suspended
// until it completes or about `hint_ns` nanoseconds pass, instead of coming
// straight back to poll: waiting warps leave the issue slots to working ones.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity,
                                                    uint32_t hint_ns)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Wait for phase `parity` of barrier `bar`.  Returns false (and never spins
// forever) when the CTA was told to abort or when the wait exceeded the
// limit; in the latter case it raises the abort flag and records `code`.
// After one plain poll the thread sleeps on the barrier (20 us per try), and
// the abort flag and the limit are checked every eighth try.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, const WaitCtl &ctl,
                                          unsigned int code)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait_sleep(bar, parity, 20000u))
            return true;
        if ((it & 7u) == 0) {
            if (*ctl.abort_flag)
                return false;
            if (globaltimer_ns() - t0 > ctl.limit_ns) {
                *ctl.abort_flag = 1;
                atomicOr(ctl.status, code);
                return false;
            }
        }
    }
}

// Non-blocking probe of phase `parity` (mbarrier.test_wait never suspends
// the thread).
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Warp-synchronous bounded wait of the lanes in `mask` (lanes 0..n-1 of a
// converged warp): each lane with want = true waits for phase `parity` of its
// own barrier, and all return together once every lane's phase is complete,
// so the lanes stay converged and issue their next instructions (tensor
// copies) as one.  A first non-blocking probe of all of them; then the whole
// warp takes the lanes' barriers in turn with the sleeping wait, which wakes
// when the phase completes and leaves the issue slots to the other warps
// meanwhile (a warp spinning on the probe measured 10 % off the epilogue's
// pace).  Returns false for all lanes when the CTA was told to abort or a
// wait ran out of time (then that wait raised the abort flag and recorded
// `code`).
__device__ __forceinline__ bool mbar_wait_lanes(unsigned mask, bool want, uint32_t bar,
                                                uint32_t parity, const WaitCtl &ctl,
                                                unsigned int code)
{
    const bool ready = !want || mbar_test_wait(bar, parity);
    if (__all_sync(mask, ready))
        return true;
    const int n = 32 - __clz(mask);
    for (int l = 0; l < n; ++l) {
        const uint32_t b = __shfl_sync(mask, bar, l);
        const uint32_t ph = __shfl_sync(mask, parity, l);
        const bool w = __shfl_sync(mask, (want && !ready) ? 1 : 0, l) != 0;
        if (w && !__all_sync(mask, mbar_wait(b, ph, ctl, code)))
            return false;
    }
    return true;
}

// Bounded wait until a monotonic shared-memory counter reaches at least
// `want` (napping between polls); same abort and limit rules as mbar_wait.
__device__ __forceinline__ bool ticket_wait(const volatile int *ticket, int want,
                                            const WaitCtl &ctl, unsigned int code)
{
    if (*ticket >= want)
        return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        __nanosleep(32);
        if (*ticket >= want)
            return true;
        if ((it & 15u) == 0) {
            if (*ctl.abort_flag)
                return false;
            if (globaltimer_ns() - t0 > ctl.limit_ns) {
                *ctl.abort_flag = 1;
                atomicOr(ctl.status, code);
                return false;
            }
        }
    }
}

// Bounded wait that ignores the abort flag: used on the way out to let copies
// and MMAs already in flight land before shared memory and TMEM are released.
__device__ __forceinline__ bool mbar_drain(uint32_t bar, uint32_t parity, uint64_t limit_ns)
{
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > limit_ns)
            return false;
    }
    return true;
}

// ---- TMA (tiled tensor loads, no multicast) ---------------------------------

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *m)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *m, uint32_t bar,
                                            int c0, int c1, int c2, int c3)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

// Tiled tensor stores from shared memory complete in bulk groups.  Every
// coordinate must be >= 0; elements outside the tensor are not written.
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Wait until at most N committed bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read()
{
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Wait until every committed bulk group has completed (writes done).
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Orders this thread's generic-proxy shared-memory writes before later
// async-proxy (TMA) accesses.
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Byte permute (prmt.b32, default mode): each selector nibble picks one of
// the 8 bytes of {b, a}; a set high bit in the nibble replicates that byte's
// sign bit instead of copying it.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// Four outputs of the exact fast requantisation (see requant32_fast):
//   t_e = acc_e * m_e + c_e  (+ rs_e * mr2, rs_e = shortcut byte e permuted by rsel_e)
//   y_e = max(min(hi32(t_e), 127), 0), four bytes packed into one word.
#ifndef X1CB_PACK_PRMT
// byte packing by multiply-adds (runs on the FMA pipe, which has headroom)
#define PACK4                                          \
    "mad.lo.u32 p, y1, 256, y0;\n\t"                 \
    "mad.lo.u32 y2, y3, 256, y2;\n\t"                \
    "mad.lo.u32 %0, y2, 65536, p;\n\t"
#else
#define PACK4                                          \
    "prmt.b32 p, y0, y1, 0x0040;\n\t"                \
    "prmt.b32 y2, y2, y3, 0x0040;\n\t"               \
    "prmt.b32 %0, p, y2, 0x5410;\n\t"
#endif
template <bool kRes>
__device__ __forceinline__ uint32_t requant4_fast(uint32_t a0, uint32_t a1, uint32_t a2,
                                                  uint32_t a3, int4 m, longlong2 c01,
                                                  longlong2 c23, uint32_t rword,
                                                  const uint32_t (&rsel)[4], int mr2)
{
    uint32_t d;
    if (kRes) {
        asm("{\n\t"
            ".reg .b64 t0, t1, t2, t3;\n\t"
            ".reg .b32 r0, r1, r2, r3, l0, l1, l2, l3, y0, y1, y2, y3, p;\n\t"
            "mad.wide.s32 t0, %1, %5, %9;\n\t"
            "mad.wide.s32 t1, %2, %6, %10;\n\t"
            "mad.wide.s32 t2, %3, %7, %11;\n\t"
            "mad.wide.s32 t3, %4, %8, %12;\n\t"
            "prmt.b32 r0, %13, 0, %14;\n\t"
            "prmt.b32 r1, %13, 0, %15;\n\t"
            "prmt.b32 r2, %13, 0, %16;\n\t"
            "prmt.b32 r3, %13, 0, %17;\n\t"
            "mad.wide.s32 t0, r0, %18, t0;\n\t"
            "mad.wide.s32 t1, r1, %18, t1;\n\t"
            "mad.wide.s32 t2, r2, %18, t2;\n\t"
            "mad.wide.s32 t3, r3, %18, t3;\n\t"
            "mov.b64 {l0, y0}, t0;\n\t"
            "mov.b64 {l1, y1}, t1;\n\t"
            "mov.b64 {l2, y2}, t2;\n\t"
            "mov.b64 {l3, y3}, t3;\n\t"
            "min.relu.s32 y0, y0, 127;\n\t"
            "min.relu.s32 y1, y1, 127;\n\t"
            "min.relu.s32 y2, y2, 127;\n\t"
            "min.relu.s32 y3, y3, 127;\n\t"
            PACK4
            "}"
            : "=r"(d)
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(m.x), "r"(m.y), "r"(m.z), "r"(m.w),
              "l"(c01.x), "l"(c01.y), "l"(c23.x), "l"(c23.y), "r"(rword), "r"(rsel[0]),
              "r"(rsel[1]), "r"(rsel[2]), "r"(rsel[3]), "r"(mr2));
    } else {
        asm("{\n\t"
            ".reg .b64 t0, t1, t2, t3;\n\t"
            ".reg .b32 l0, l1, l2, l3, y0, y1, y2, y3, p;\n\t"
            "mad.wide.s32 t0, %1, %5, %9;\n\t"
            "mad.wide.s32 t1, %2, %6, %10;\n\t"
            "mad.wide.s32 t2, %3, %7, %11;\n\t"
            "mad.wide.s32 t3, %4, %8, %12;\n\t"
            "mov.b64 {l0, y0}, t0;\n\t"
            "mov.b64 {l1, y1}, t1;\n\t"
            "mov.b64 {l2, y2}, t2;\n\t"
            "mov.b64 {l3, y3}, t3;\n\t"
            "min.relu.s32 y0, y0, 127;\n\t"
            "min.relu.s32 y1, y1, 127;\n\t"
            "min.relu.s32 y2, y2, 127;\n\t"
            "min.relu.s32 y3, y3, 127;\n\t"
            PACK4
            "}"
            : "=r"(d)
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(m.x), "r"(m.y), "r"(m.z), "r"(m.w),
              "l"(c01.x), "l"(c01.y), "l"(c23.x), "l"(c23.y));
    }
    return d;
}

// Four outputs of the exact all-32-bit form (see requant_hi32):
//   y2_e = hi32((acc_e + bias_e) * m_e) + 1 (+ r_e * k),  r_e = shortcut byte e
//   out_e = min(max(y2_e, 0), 255) >> 1, four bytes packed into one word.
// kAddBias = false: the accumulator already holds acc + bias (folded into the
// MMA), so the four additions are skipped and b is ignored.  kK1: k == 1.
// The high word is a plain multiply-high and the small addend a separate add
// (with k == 1, h + r + 1 is one three-input add).  The clamp to [0, 255] and
// the packing are one saturating convert-and-pack per two outputs
// (cvt.pack.sat.u8.s32: d = c << 16 | sat(a) << 8 | sat(b)), and the halving
// is done on the packed word: each byte is at most 255, so a shift of the
// whole word by one and a mask of the bits that crossed a byte boundary
// halve the four bytes exactly.
template <bool kRes, bool kAddBias = true, bool kK1 = false>
__device__ __forceinline__ uint32_t requant4_hi32(uint32_t a0, uint32_t a1, uint32_t a2,
                                                  uint32_t a3, int4 m, int4 b, uint32_t rword,
                                                  const uint32_t (&rsel)[4], int k)
{
    const uint32_t av[4] = {a0, a1, a2, a3};
    const int mv[4] = {m.x, m.y, m.z, m.w};
    const int bv[4] = {b.x, b.y, b.z, b.w};
    int y[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int u = kAddBias ? static_cast<int>(av[e]) + bv[e] : static_cast<int>(av[e]);
        const int h = __mulhi(u, mv[e]);
        int c = 1;
        if (kRes) {
            int r;  // the shortcut byte, sign-extended
            asm("prmt.b32 %0, %1, 0, %2;" : "=r"(r) : "r"(rword), "r"(rsel[e]));
            c = kK1 ? r + 1 : r * k + 1;
        }
        y[e] = h + c;
    }
    uint32_t hi, d;
    asm("cvt.pack.sat.u8.s32.b32 %0, %1, %2, %3;" : "=r"(hi) : "r"(y[3]), "r"(y[2]), "r"(0));
    asm("cvt.pack.sat.u8.s32.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(y[1]), "r"(y[0]), "r"(hi));
    return (d >> 1) & 0x7f7f7f7fu;
}

// L2 policy for data read or written once: evict it first.
__device__ __forceinline__ uint64_t policy_evict_first()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ void tma_load_4d_hint(uint32_t dst, const CUtensorMap *m, uint32_t bar,
                                                 int c0, int c1, int c2, int c3, uint64_t pol)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%3, %4, %5, %6}], [%2], %7;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
        "l"(pol)
        : "memory");
}

__device__ __forceinline__ void tma_load_5d_hint(uint32_t dst, const CUtensorMap *m, uint32_t bar,
                                                 int c0, int c1, int c2, int c3, int c4,
                                                 uint64_t pol)
{
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%3, %4, %5, %6, %7}], [%2], %8;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
        "r"(c4), "l"(pol)
        : "memory");
}

__device__ __forceinline__ void tma_store_4d_hint(const CUtensorMap *m, uint32_t src, int c0,
                                                  int c1, int c2, int c3, uint64_t pol)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group.L2::cache_hint"
        " [%0, {%2, %3, %4, %5}], [%1], %6;" ::"l"(reinterpret_cast<uint64_t>(m)),
        "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "l"(pol)
        : "memory");
}

__device__ __forceinline__ void tma_store_5d_hint(const CUtensorMap *m, uint32_t src, int c0,
                                                  int c1, int c2, int c3, int c4, uint64_t pol)
{
    asm volatile(
        "cp.async.bulk.tensor.5d.global.shared::cta.tile.bulk_group.L2::cache_hint"
        " [%0, {%2, %3, %4, %5, %6}], [%1], %7;" ::"l"(reinterpret_cast<uint64_t>(m)),
        "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "l"(pol)
        : "memory");
}

// ---- tcgen05: TMEM, MMA, loads -----------------------------------------------

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     dst_smem),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before()
{
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after()
{
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major operand stored with the
// 32-byte swizzle: rows of 32 bytes (= 32 int8 = one MMA K step), 8-row
// groups `group_bytes` apart (256: back to back).  The swizzle follows the
// address, so a start moved by a multiple of 256 bytes keeps its pattern.
__device__ __forceinline__ uint64_t smem_desc_sw32(uint32_t saddr, uint32_t group_bytes = 256)
{
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);          // start address
    d |= static_cast<uint64_t>(1) << 16;                          // leading offset (unused here)
    d |= static_cast<uint64_t>((group_bytes >> 4) & 0x3FFFu) << 32;  // between 8-row groups
    d |= static_cast<uint64_t>(1) << 46;                          // descriptor version
    d |= static_cast<uint64_t>(6) << 61;                          // 32-byte swizzle
    return d;
}

// Shared-memory matrix descriptor for a K-major operand without swizzle whose
// rows are 16 bytes apart (8-row core matrices back to back, 128 bytes each)
// and whose two 16-byte K halves are `half_bytes` apart.  Rows are linear in
// the address, so a descriptor shifted by n rows is this one plus n.
__device__ __forceinline__ uint64_t smem_desc_rows16(uint32_t saddr, uint32_t half_bytes)
{
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);           // start address
    d |= static_cast<uint64_t>((half_bytes >> 4) & 0x3FFFu) << 16;  // K-direction core-matrix stride
    d |= static_cast<uint64_t>(128 >> 4) << 32;                     // M-direction 8-row stride
    d |= static_cast<uint64_t>(1) << 46;                            // descriptor version
    return d;                                                       // layout 0: no swizzle
}

// Instruction descriptor: s8 x s8 -> s32, both operands K-major, M x N.
__host__ __device__ constexpr uint32_t idesc_i8(uint32_t M, uint32_t N)
{
    return (2u << 4)            // D format: s32
           | (1u << 7)          // A: signed int8
           | (1u << 10)         // B: signed int8
           | ((N >> 3) << 17)   // N
           | ((M >> 4) << 24);  // M
}

// One MMA step D (+)= A x B, s8 x s8 -> s32 in TMEM.  Warp-wide: every lane
// of the issuing warp calls it with the same operands and one elected lane
// issues, so the warp stays converged and its operand arithmetic is
// warp-uniform.  accumulate = 0 overwrites D.
__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on `bar` when every MMA issued so far by the warp's elected lane
// is done (warp-wide, like mma_i8).
__device__ __forceinline__ void mma_commit(uint32_t bar)
{
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}"
        ::"r"(bar)
        : "memory");
}

// tcgen05.ld of 32 lanes x 32 consecutive 32-bit columns (thread t gets lane
// base + t) followed by its wait in one statement, so the registers are
// defined only once the data has arrived.
__device__ __forceinline__ void tmem_ld_32x32b_x32_sync(uint32_t taddr, uint32_t (&v)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, "
        "[%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
          "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
          "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
          "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
          "=r"(v[31])
        : "r"(taddr)
        : "memory");
}

// ---- pairs of CTAs (a cluster of two sharing one tcgen05 MMA) --------------
//
// With cta_group::2 one MMA spans the two CTAs of a cluster: A is split by rows
// (each CTA supplies its own 128 rows from its own shared memory), B by columns
// (each CTA holds half of N), and each CTA's TMEM receives its own 128 rows of
// the result.  Rank 0 issues the MMAs; both CTAs load their operands and
// drain their accumulators.

// Programmatic dependent launch: wait until the grids this one depends on
// (the preceding kernel on the stream) have completed and their memory is
// visible; a no-op when the kernel was launched without the attribute.
__device__ __forceinline__ void griddep_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Address of the same shared-memory variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank)
{
    uint32_t d;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(saddr), "r"(rank));
    return d;
}

// Arrive on a barrier given by its shared::cluster address (possibly in the
// other CTA), releasing this thread's prior writes at cluster scope.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_bar)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar)
                 : "memory");
}

// Both CTAs of the cluster: every thread arrives and waits (hardware barrier;
// used once after set-up, when both CTAs are known to be running).
__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(20000u)
        : "memory");
    return ok != 0;
}

// Bounded wait with cluster-scope acquire (for barriers that the other CTA
// arrives on); same abort and limit rules as mbar_wait.
__device__ __forceinline__ bool mbar_wait_cl(uint32_t bar, uint32_t parity, const WaitCtl &ctl,
                                             unsigned int code)
{
    if (mbar_try_wait_cluster(bar, parity))
        return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait_cluster(bar, parity))
            return true;
        if ((it & 7u) == 0) {
            if (*ctl.abort_flag)
                return false;
            if (globaltimer_ns() - t0 > ctl.limit_ns) {
                *ctl.abort_flag = 1;
                atomicOr(ctl.status, code);
                return false;
            }
        }
    }
}

// Tiled loads into this CTA's shared memory whose completion is counted on a
// barrier of rank 0 (cluster_bar: its shared::cluster address), so that the
// MMA issuer sees both CTAs' operands land on one barrier.  No multicast.
__device__ __forceinline__ void tma2_load_4d(uint32_t dst, const CUtensorMap *m,
                                             uint32_t cluster_bar, int c0, int c1, int c2,
                                             int c3)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(cluster_bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

__device__ __forceinline__ void tma2_load_5d_hint(uint32_t dst, const CUtensorMap *m,
                                                  uint32_t cluster_bar, int c0, int c1, int c2,
                                                  int c3, int c4, uint64_t pol)
{
    asm volatile(
        "cp.async.bulk.tensor.5d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%3, %4, %5, %6, %7}], [%2], %8;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(cluster_bar), "r"(c0), "r"(c1), "r"(c2),
        "r"(c3), "r"(c4), "l"(pol)
        : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     dst_smem),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr),
                 "r"(ncols)
                 : "memory");
}

// One MMA step over both CTAs (M = 256: 128 rows from each), warp-wide with an
// elected issuing lane; rank 0 only.
__device__ __forceinline__ void mma_i8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on barrier `bar` (same offset) in both CTAs when the pair MMAs
// issued so far are done (warp-wide, elected lane).
__device__ __forceinline__ void mma_commit_pair(uint32_t bar)
{
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster"
        ".b64 [%0], %1;\n\t}" ::"r"(bar),
        "h"(static_cast<uint16_t>(3))
        : "memory");
}

}  // namespace x1cb
