// Exact requantisation forms of the fused epilogue and the per-layer checks
// that select them (device code shared by the convolution kernels).
//
// Every form computes, per output element, exactly
//   t = (acc + bias) * m (+ r * m_r) + 2^(S-1),  out = min(max(t >> S, 0), 127)
// (the Inspur MLPerf ResNet50 convolution-merge article, sections 2.2 and
// 3.4: Bn, Sum and Relu applied to the accumulator before the write-back);
// the cheaper forms are used only where their integer ranges make them exact.
#pragma once
#include <climits>
#include <cstdint>

#include "x1cb_ptx.cuh"

namespace x1cb {

// Generic exact requantisation of 32 accumulators of one pixel (channels
// n0..n0+31 of this CTA's group), packed as 32 int8 bytes:
//   t = acc*m + C (+ r*m_r),  C = bias*m + 2^(S-1),  y = clamp(t >> S, 0, 127).
template <bool kRes>
__device__ __forceinline__ void requant32(const uint32_t *v, const int32_t *cm,
                                          const long long *cC, const uint32_t *rw, int m_r,
                                          int S, uint32_t *ow)
{
#pragma unroll
    for (int q = 0; q < 8; ++q)
        ow[q] = 0u;
#pragma unroll 8
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

// Exact fast form of the same requantisation, used when the CTA's constants
// allow it (checked in the prologue).  With s = 32 - S >= 0 every term is
// pre-scaled by 2^s: m' = m*2^s, C' = bias*m' + 2^31, and the residual term
// becomes (r*2^(8*k8)) * (m_r*2^(s - 8*k8)).  Then
//     t' = acc*m' + C' + r*m_r*2^s = t * 2^s,
// so floor(t / 2^S) = floor(t' / 2^32) is exactly the high word of t' (no
// shift, no 64-bit compare).  All three products fit their 32-bit operands and
// the sum stays below 2^63 (prologue check), so nothing is approximated.
// Processes n4 groups of 4 channels.
template <bool kRes, int kGroups>
__device__ __forceinline__ void requant_fast(const uint32_t *v, const int32_t *cm,
                                             const long long *cC, const uint32_t *rw, int mr2,
                                             const uint32_t (&rsel)[4], uint32_t *ow)
{
    const int4 *m4 = reinterpret_cast<const int4 *>(cm);
    const longlong2 *c2 = reinterpret_cast<const longlong2 *>(cC);
#pragma unroll
    for (int q = 0; q < kGroups; ++q)
        ow[q] = requant4_fast<kRes>(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3], m4[q],
                                    c2[2 * q], c2[2 * q + 1], kRes ? rw[q] : 0u, rsel, mr2);
}

// Exact all-32-bit form, used when the shortcut multiplier is a multiple of
// 2^(S-1) (m_r = k * 2^(S-1)) and the CTA's constants allow it.  With
// s = 33 - S >= 0 and m' = m * 2^s, every term of t * 2^s except the product
// is a multiple of 2^32:
//     t * 2^s = (acc + bias) * m' + 2^32 * (1 + r*k),
// so y2 = floor(t * 2^s / 2^32) = hi32((acc + bias) * m') + 1 + r*k exactly
// (mad.hi), and floor(t / 2^S) = floor(y2 / 2); clamping y2 to [0, 255]
// before halving gives the [0, 127] clamp.  No 64-bit arithmetic.
template <bool kRes, bool kAddBias, bool kK1, int kGroups>
__device__ __forceinline__ void requant_hi32(const uint32_t *v, const int32_t *cm,
                                             const int32_t *cb, const uint32_t *rw, int k,
                                             const uint32_t (&rsel)[4], uint32_t *ow)
{
    const int4 *m4 = reinterpret_cast<const int4 *>(cm);
    const int4 *b4 = reinterpret_cast<const int4 *>(cb);
#pragma unroll
    for (int q = 0; q < kGroups; ++q)
        ow[q] = requant4_hi32<kRes, kAddBias, kK1>(v[4 * q], v[4 * q + 1], v[4 * q + 2],
                                              v[4 * q + 3], m4[q],
                                              kAddBias ? b4[q] : make_int4(0, 0, 0, 0),
                                              kRes ? rw[q] : 0u, rsel, k);
}

// Bias folded into the MMA: one extra K step of 32 columns adds
//   sum_c A[c] * D_n[c] = bias[n]
// to every row of the accumulator, with the constant A row
//   [1, 127 x 15, 1, 127 x 15]
// and per-channel int8 digits D_n: D_n[0] = bias mod 127 (centred), the other
// 30 digits (columns 1-15, 17-31) carry (bias - D_n[0]) / 127 in steps of at
// most 127 in magnitude, D_n[16] = 0.  Exact for |bias| <= 30*127*127 + 63;
// used for |bias| <= 2^18.  Because the two 16-byte halves of the A row are
// equal, the sum does not depend on which half of a 32-byte row the 32-byte
// swizzle presents first, so both tiles are written without swizzling.
constexpr int kBiasFoldMax = 1 << 18;

__device__ __forceinline__ void bias_digits(int bias, uint32_t (&w)[8])
{
    int8_t d[32];
    const int d0 = ((bias + 63) % 127 + 127) % 127 - 63;  // bias mod 127 in [-63, 63]
    int D = (bias - d0) / 127;
    d[0] = static_cast<int8_t>(d0);
    d[16] = 0;
#pragma unroll
    for (int c = 1; c < 32; ++c) {
        if (c == 16)
            continue;
        const int step = D > 127 ? 127 : (D < -127 ? -127 : D);
        d[c] = static_cast<int8_t>(step);
        D -= step;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
        w[i] = static_cast<uint32_t>(static_cast<uint8_t>(d[4 * i])) |
               static_cast<uint32_t>(static_cast<uint8_t>(d[4 * i + 1])) << 8 |
               static_cast<uint32_t>(static_cast<uint8_t>(d[4 * i + 2])) << 16 |
               static_cast<uint32_t>(static_cast<uint8_t>(d[4 * i + 3])) << 24;
}

// Layer-wide conditions of the all-32-bit form (per channel: hi32_ok).
__device__ __forceinline__ bool hi32_layer_ok(int m_r, int S, bool res)
{
    if (S < 2 || S > 33)
        return false;
    if (!res)
        return true;
    const long long q = 1ll << (S - 1);
    if (static_cast<long long>(m_r) % q != 0)
        return false;
    // y2 = h + 1 + r*k with -2^30 <= h <= 2^30 - 1 and r in [-128, 127]
    // stays inside int32 while -2^30 - 1 <= r*k <= 2^30 - 1: k = -2^23 with
    // r = -128 would reach 2^31, so the lower bound is exclusive.
    const long long k = static_cast<long long>(m_r) / q;
    return k > -(1ll << 23) && k <= (1ll << 23);
}

// Per-channel conditions: m * 2^(33-S) fits int32, and acc + bias cannot
// overflow int32 (|acc| <= K * 2^14).
__device__ __forceinline__ bool hi32_ok(long long m, long long bias, int S, int K)
{
    if (S < 2 || S > 33)
        return false;
    const long long mp = m * (1ll << (33 - S));
    if (mp < INT_MIN || mp > INT_MAX)
        return false;
    return (bias < 0 ? -bias : bias) + static_cast<long long>(K) * 16384 < (1ll << 31);
}

// Whether the fast form is exact for output channel o of a layer of fan-in K
// (every |x|, |w| <= 128, so |acc| <= K * 2^14).
__device__ __forceinline__ bool fast_form_ok(long long m, long long bias, int m_r, int S, int K,
                                             bool res)
{
    if (S > 32)
        return false;
    const int sh = 32 - S;
    const long long mp = m * (1ll << sh);
    if (mp < INT_MIN || mp > INT_MAX)
        return false;
    double bound = static_cast<double>(K) * 16384.0 * fabs(static_cast<double>(mp)) +
                   fabs(static_cast<double>(bias) * static_cast<double>(mp)) + 2147483648.0;
    if (res) {
        const int k8 = sh / 8 < 3 ? sh / 8 : 3;
        const long long mr2 = static_cast<long long>(m_r) * (1ll << (sh - 8 * k8));
        if (mr2 < INT_MIN || mr2 > INT_MAX)
            return false;
        bound += 128.0 * fabs(static_cast<double>(m_r)) * static_cast<double>(1ll << sh);
    }
    return bound < 4.0e18;  // < 2^62 with margin for the double rounding
}

}  // namespace x1cb
