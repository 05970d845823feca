/*
 * Plain CPU oracle for the fused INT8 bottleneck convolutions.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library calls this file: only the
 * tests, the smoke check and the benchmark's CPU-baseline leg load it.  It
 * shares no code, header, table or helper with the CUDA path; it has its own
 * layout index arithmetic and its own requantisation.  Everything is written
 * as the plain definition, slow and obvious, with 64-bit intermediates.
 *
 * What it computes (per output pixel (b,h,w) and output channel o):
 *
 *   acc = sum_{r,s,i} X[b, h+r-pad, w+s-pad, i] * Wt[o, i, r, s]
 *         (taps that fall outside the image contribute 0)
 *   t   = (acc + bias[o]) * m[o] + (residual ? R[b,h,w,o] * m_r : 0) + 2^(S-1)
 *   y   = floor(t / 2^S)
 *   out = min(max(y, 0), 127)
 *
 * Sources:
 *  - Inspur MLPerf v2.0 ResNet50 convolution-merge article
 *    (news.cnblogs.com/n/719672), section 2.2: Conv3 is followed by Bn, then
 *    the Shortcut Sum with the block input and a Relu; Conv1 and Conv2 are each
 *    followed by Bn and Relu.  Section 3.4: Bn+Sum+Relu is applied to every
 *    Conv3 result before the write-back.  Section 3.1: data, weight and output
 *    are int8.
 *  - The requantisation rule above (folded BN as an int32 bias and an int32
 *    per-channel multiplier, residual multiplier m_r, round-half-up through
 *    +2^(S-1), arithmetic right shift by S, ReLU and saturation to [0,127]) is
 *    this library's statement of the fused op; the pages name the steps but
 *    print no formula.
 *  - Section 3.1 of the same article defines the layouts: activations
 *    [B, C/32, H, W, 32] (NC/32HW32) and 1x1 weights [O1, I1, O2, I2] with
 *    O2 = 128 and I2 = 32.  The 3x3 weight layout [O1, R, S, I1, O2, I2] is
 *    this library's extension (the pages give none).
 *  - Didi Cloud IFX DAWNBench article (blog.csdn.net/didi_cloud), section on
 *    inference optimisation: CONV+BN+RELU as one fused unit (the 3x3 stage).
 *
 * Domain: 1 <= S <= 60, fan-in R*R*Ic <= 36864, so every intermediate fits in
 * int64 with room to spare.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* floor(t / 2^S), written with C's truncating division so that nothing relies
 * on the implementation-defined right shift of a negative value. */
static int64_t floor_div_pow2(int64_t t, int S)
{
    int64_t d = (int64_t)1 << S;
    int64_t q = t / d;
    if (t % d != 0 && t < 0)
        q -= 1;
    return q;
}

/* One output element of the epilogue: BN (bias, multiplier), optional
 * shortcut Sum, rounding shift, ReLU and saturation to int8. */
int8_t x1o_requant(int64_t acc, int32_t bias, int32_t m, int has_res, int32_t r,
                   int32_t m_r, int S)
{
    int64_t t = (acc + (int64_t)bias) * (int64_t)m;
    if (has_res)
        t += (int64_t)r * (int64_t)m_r;
    t += (int64_t)1 << (S - 1);
    int64_t y = floor_div_pow2(t, S);
    if (y < 0)
        y = 0;
    if (y > 127)
        y = 127;
    return (int8_t)y;
}

/* ---- layouts (section 3.1 of the Inspur article) ------------------------- */

/* NC/32HW32: element (b, c, h, w) of a [B, C/32, H, W, 32] tensor. */
static size_t nc32_index(int64_t b, int64_t c, int64_t h, int64_t w, int64_t C, int64_t H,
                         int64_t W)
{
    return (size_t)((((b * (C / 32) + c / 32) * H + h) * W + w) * 32 + c % 32);
}

/* NHWC: element (b, h, w, c). */
static size_t nhwc_index(int64_t b, int64_t h, int64_t w, int64_t c, int64_t H, int64_t W,
                         int64_t C)
{
    return (size_t)(((b * H + h) * W + w) * C + c);
}

/* Blocked weight [O1, R, S, I1, O2, I2=32]: element (o, i, r, s).  O2 = 128
 * (the article's block of output channels); a layer of fewer than 128 output
 * channels (64: the network's stem) is one block of O2 = Oc.  For R = S = 1
 * this is the article's [O1, I1, O2, I2]. */
static size_t wblk_index(int64_t o, int64_t i, int64_t r, int64_t s, int64_t Ic, int64_t R,
                         int64_t Oc)
{
    int64_t I1 = Ic / 32;
    int64_t O2 = Oc < 128 ? Oc : 128;
    return (size_t)((((((o / O2) * R + r) * R + s) * I1 + i / 32) * O2 + o % O2) * 32 + i % 32);
}

/* OIHW (PyTorch convolution weight order): element (o, i, r, s). */
static size_t oihw_index(int64_t o, int64_t i, int64_t r, int64_t s, int64_t Ic, int64_t R)
{
    return (size_t)(((o * Ic + i) * R + r) * R + s);
}

void x1o_pack_act(const int8_t *nhwc, int8_t *nc32, int B, int H, int W, int C)
{
    for (int64_t b = 0; b < B; ++b)
        for (int64_t h = 0; h < H; ++h)
            for (int64_t w = 0; w < W; ++w)
                for (int64_t c = 0; c < C; ++c)
                    nc32[nc32_index(b, c, h, w, C, H, W)] = nhwc[nhwc_index(b, h, w, c, H, W, C)];
}

void x1o_unpack_act(const int8_t *nc32, int8_t *nhwc, int B, int H, int W, int C)
{
    for (int64_t b = 0; b < B; ++b)
        for (int64_t h = 0; h < H; ++h)
            for (int64_t w = 0; w < W; ++w)
                for (int64_t c = 0; c < C; ++c)
                    nhwc[nhwc_index(b, h, w, c, H, W, C)] = nc32[nc32_index(b, c, h, w, C, H, W)];
}

void x1o_pack_weight(const int8_t *oihw, int8_t *blk, int Oc, int Ic, int R)
{
    for (int64_t o = 0; o < Oc; ++o)
        for (int64_t i = 0; i < Ic; ++i)
            for (int64_t r = 0; r < R; ++r)
                for (int64_t s = 0; s < R; ++s)
                    blk[wblk_index(o, i, r, s, Ic, R, Oc)] = oihw[oihw_index(o, i, r, s, Ic, R)];
}

void x1o_unpack_weight(const int8_t *blk, int8_t *oihw, int Oc, int Ic, int R)
{
    for (int64_t o = 0; o < Oc; ++o)
        for (int64_t i = 0; i < Ic; ++i)
            for (int64_t r = 0; r < R; ++r)
                for (int64_t s = 0; s < R; ++s)
                    oihw[oihw_index(o, i, r, s, Ic, R)] = blk[wblk_index(o, i, r, s, Ic, R, Oc)];
}

/* ---- the fused convolution ---------------------------------------------- */

/* All Oc outputs of one pixel.  x is NHWC, wt is OIHW, r (may be NULL) and
 * the result row are indexed by channel. */
static void conv_pixel(const int8_t *x, const int8_t *wt, const int32_t *bias, const int32_t *m,
                       int S, const int8_t *r_row, int32_t m_r, int8_t *out_row, int64_t b,
                       int64_t h, int64_t w, int H, int W, int Ic, int Oc, int R, int pad)
{
    for (int64_t o = 0; o < Oc; ++o) {
        int64_t acc = 0;
        for (int64_t rr = 0; rr < R; ++rr) {
            int64_t hi = h + rr - pad;
            if (hi < 0 || hi >= H)
                continue;
            for (int64_t ss = 0; ss < R; ++ss) {
                int64_t wi = w + ss - pad;
                if (wi < 0 || wi >= W)
                    continue;
                const int8_t *xp = x + nhwc_index(b, hi, wi, 0, H, W, Ic);
                for (int64_t i = 0; i < Ic; ++i)
                    acc += (int64_t)xp[i] * (int64_t)wt[oihw_index(o, i, rr, ss, Ic, R)];
            }
        }
        out_row[o] = x1o_requant(acc, bias[o], m[o], r_row != NULL, r_row ? r_row[o] : 0, m_r, S);
    }
}

/* Full-tensor fused convolution, stride 1, zero padding `pad`, output H x W.
 * x: [B,H,W,Ic] NHWC.  wt: [Oc,Ic,R,R].  r: [B,H,W,Oc] or NULL.
 * out: [B,H,W,Oc]. */
void x1o_conv(const int8_t *x, const int8_t *wt, const int32_t *bias, const int32_t *m, int S,
              const int8_t *r, int32_t m_r, int8_t *out, int B, int H, int W, int Ic, int Oc,
              int R, int pad)
{
    int64_t rows = (int64_t)B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < rows; ++bh) {
        int64_t b = bh / H, h = bh % H;
        for (int64_t w = 0; w < W; ++w) {
            size_t p = nhwc_index(b, h, w, 0, H, W, Oc);
            conv_pixel(x, wt, bias, m, S, r ? r + p : NULL, m_r, out + p, b, h, w, H, W, Ic, Oc,
                       R, pad);
        }
    }
}

/* The same convolution evaluated only at `n` chosen pixels.  pix[k] is the
 * flattened index (b*H + h)*W + w; out_rows is [n, Oc]. */
void x1o_conv_pixels(const int8_t *x, const int8_t *wt, const int32_t *bias, const int32_t *m,
                     int S, const int8_t *r, int32_t m_r, const int64_t *pix, int64_t n,
                     int8_t *out_rows, int B, int H, int W, int Ic, int Oc, int R, int pad)
{
    (void)B;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t k = 0; k < n; ++k) {
        int64_t p = pix[k];
        int64_t b = p / ((int64_t)H * W), h = (p / W) % H, w = p % W;
        conv_pixel(x, wt, bias, m, S, r ? r + (size_t)p * Oc : NULL, m_r,
                   out_rows + (size_t)k * Oc, b, h, w, H, W, Ic, Oc, R, pad);
    }
}

/* Res3.x bottleneck block (section 2.2 of the Inspur article): conv1 1x1
 * Cin->Cmid +Bn+Relu, conv2 3x3 pad 1 Cmid->Cmid +Bn+Relu, conv3 1x1
 * Cmid->Cin +Bn + Sum with the block input + Relu.  All three stages use the
 * same shift S; only conv3 has the residual term. */
void x1o_bottleneck(const int8_t *x, const int8_t *w1, const int32_t *b1, const int32_t *m1,
                    const int8_t *w2, const int32_t *b2, const int32_t *m2, const int8_t *w3,
                    const int32_t *b3, const int32_t *m3, int32_t m_r, int S, int8_t *out, int B,
                    int H, int W, int Cin, int Cmid)
{
    size_t mid = (size_t)B * H * W * Cmid;
    int8_t *y1 = (int8_t *)malloc(mid);
    int8_t *y2 = (int8_t *)malloc(mid);
    x1o_conv(x, w1, b1, m1, S, NULL, 0, y1, B, H, W, Cin, Cmid, 1, 0);
    x1o_conv(y1, w2, b2, m2, S, NULL, 0, y2, B, H, W, Cmid, Cmid, 3, 1);
    x1o_conv(y2, w3, b3, m3, S, x, m_r, out, B, H, W, Cmid, Cin, 1, 0);
    free(y1);
    free(y2);
}

/* The block evaluated only at `n` chosen output pixels: conv1 is evaluated on
 * the 3x3 neighbourhood the pixel's conv2 needs, then conv2 and conv3 at the
 * pixel itself.  out_rows is [n, Cin]. */
void x1o_bottleneck_pixels(const int8_t *x, const int8_t *w1, const int32_t *b1,
                           const int32_t *m1, const int8_t *w2, const int32_t *b2,
                           const int32_t *m2, const int8_t *w3, const int32_t *b3,
                           const int32_t *m3, int32_t m_r, int S, const int64_t *pix, int64_t n,
                           int8_t *out_rows, int B, int H, int W, int Cin, int Cmid)
{
    (void)B;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t k = 0; k < n; ++k) {
        int64_t p = pix[k];
        int64_t b = p / ((int64_t)H * W), h = (p / W) % H, w = p % W;
        /* conv1 outputs on a 3x3 window stored as a tiny NHWC image. */
        int8_t *win = (int8_t *)calloc((size_t)9 * Cmid, 1);
        int8_t *y2 = (int8_t *)malloc((size_t)Cmid);
        for (int64_t dr = 0; dr < 3; ++dr)
            for (int64_t ds = 0; ds < 3; ++ds) {
                int64_t hh = h + dr - 1, ww = w + ds - 1;
                if (hh < 0 || hh >= H || ww < 0 || ww >= W)
                    continue; /* zero padding of conv2's input */
                conv_pixel(x, w1, b1, m1, S, NULL, 0, win + (dr * 3 + ds) * Cmid, b, hh, ww, H,
                           W, Cin, Cmid, 1, 0);
            }
        /* conv2 at the window centre.  Out-of-image taps were left at zero,
         * which is exactly the zero padding, so the window is treated as a
         * 3x3 image with no further padding. */
        for (int64_t o = 0; o < Cmid; ++o) {
            int64_t acc = 0;
            for (int64_t rr = 0; rr < 3; ++rr)
                for (int64_t ss = 0; ss < 3; ++ss)
                    for (int64_t i = 0; i < Cmid; ++i)
                        acc += (int64_t)win[(rr * 3 + ss) * Cmid + i] *
                               (int64_t)w2[oihw_index(o, i, rr, ss, Cmid, 3)];
            y2[o] = x1o_requant(acc, b2[o], m2[o], 0, 0, 0, S);
        }
        /* conv3 at the pixel with the block input as the shortcut. */
        const int8_t *r_row = x + (size_t)p * Cin;
        for (int64_t o = 0; o < Cin; ++o) {
            int64_t acc = 0;
            for (int64_t i = 0; i < Cmid; ++i)
                acc += (int64_t)y2[i] * (int64_t)w3[oihw_index(o, i, 0, 0, Cmid, 1)];
            out_rows[(size_t)k * Cin + o] = x1o_requant(acc, b3[o], m3[o], 1, r_row[o], m_r, S);
        }
        free(win);
        free(y2);
    }
}

/* ---- strided convolution and the projection block (Res3.1) ------------------
 *
 * The pages describe Res3.2-Res3.4 and say only that Res3.1's output feeds
 * Res3.2 (Inspur article, section 2.2).  Res3.1 is the stage's first block:
 * it halves the image and widens the channels, so its shortcut is a 1x1
 * projection convolution of stride 2 instead of the identity.  Read here as
 * in the MLPerf ResNet50 (v1.5) network: conv1 1x1 stride 1, conv2 3x3 pad 1
 * stride 2, conv3 1x1; shortcut 1x1 stride 2 on the block input.  The
 * projection's folded BN shares Conv3's per-channel multiplier (its relative
 * scale folded into its int8 weights), so the two products are summed into
 * one accumulator before the common bias, multiplier, rounding and ReLU:
 *
 *   acc = sum_i Y[b,h,w,i] * W3[o,i] + sum_j X[b, 2h, 2w, j] * WP[o,j]
 *   out = min(max(floor(((acc + bias[o]) * m[o] + 2^(S-1)) / 2^S), 0), 127)
 */

/* Output extent of a convolution along one axis. */
static int64_t conv_out_extent(int64_t in, int64_t R, int64_t pad, int64_t stride)
{
    return (in + 2 * pad - R) / stride + 1;
}

/* Fused convolution of any stride: output pixel (b, ho, wo) reads input
 * pixels (ho*stride + r - pad, wo*stride + s - pad); taps outside the image
 * contribute 0.  x: [B,H,W,Ic]; wt: [Oc,Ic,R,R]; r: [B,Ho,Wo,Oc] or NULL;
 * out: [B,Ho,Wo,Oc]. */
void x1o_conv_strided(const int8_t *x, const int8_t *wt, const int32_t *bias, const int32_t *m,
                      int S, const int8_t *r, int32_t m_r, int8_t *out, int B, int H, int W,
                      int Ic, int Oc, int R, int pad, int stride)
{
    int64_t Ho = conv_out_extent(H, R, pad, stride), Wo = conv_out_extent(W, R, pad, stride);
    int64_t rows = (int64_t)B * Ho;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < rows; ++bh) {
        int64_t b = bh / Ho, ho = bh % Ho;
        for (int64_t wo = 0; wo < Wo; ++wo) {
            size_t q = (size_t)((b * Ho + ho) * Wo + wo) * Oc;
            for (int64_t o = 0; o < Oc; ++o) {
                int64_t acc = 0;
                for (int64_t rr = 0; rr < R; ++rr) {
                    int64_t hi = ho * stride + rr - pad;
                    if (hi < 0 || hi >= H)
                        continue;
                    for (int64_t ss = 0; ss < R; ++ss) {
                        int64_t wi = wo * stride + ss - pad;
                        if (wi < 0 || wi >= W)
                            continue;
                        const int8_t *xp = x + nhwc_index(b, hi, wi, 0, H, W, Ic);
                        for (int64_t i = 0; i < Ic; ++i)
                            acc += (int64_t)xp[i] * (int64_t)wt[oihw_index(o, i, rr, ss, Ic, R)];
                    }
                }
                out[q + o] = x1o_requant(acc, bias[o], m[o], r != NULL, r ? r[q + o] : 0, m_r, S);
            }
        }
    }
}

/* Conv3 of the projection block with its shortcut in the same accumulator.
 * y: [B,H,W,Cy] (Conv2's output); w3: [Oc,Cy] (1x1, OIHW with R = 1);
 * x: [B,Hx,Wx,Cx] (the block input), sampled at (stride*h, stride*w);
 * wp: [Oc,Cx]; out: [B,H,W,Oc]. */
void x1o_conv_proj(const int8_t *y, const int8_t *w3, const int8_t *x, const int8_t *wp,
                   const int32_t *bias, const int32_t *m, int S, int8_t *out, int B, int H, int W,
                   int Cy, int Cx, int Oc, int Hx, int Wx, int stride)
{
    int64_t rows = (int64_t)B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < rows; ++bh) {
        int64_t b = bh / H, h = bh % H;
        for (int64_t w = 0; w < W; ++w) {
            const int8_t *yp = y + nhwc_index(b, h, w, 0, H, W, Cy);
            const int8_t *xp = x + nhwc_index(b, h * stride, w * stride, 0, Hx, Wx, Cx);
            size_t q = (size_t)nhwc_index(b, h, w, 0, H, W, Oc);
            for (int64_t o = 0; o < Oc; ++o) {
                int64_t acc = 0;
                for (int64_t i = 0; i < Cy; ++i)
                    acc += (int64_t)yp[i] * (int64_t)w3[o * Cy + i];
                for (int64_t j = 0; j < Cx; ++j)
                    acc += (int64_t)xp[j] * (int64_t)wp[o * Cx + j];
                out[q + o] = x1o_requant(acc, bias[o], m[o], 0, 0, 0, S);
            }
        }
    }
}

/* Res3.1 projection block: conv1 1x1 Cin->Cmid +Bn+Relu (H x W), conv2 3x3
 * pad 1 stride 2 Cmid->Cmid +Bn+Relu (-> Ho x Wo), conv3 1x1 Cmid->Cout plus
 * the stride-2 1x1 projection Cin->Cout of the block input in one
 * accumulator, +Bn+Relu.  x: [B,H,W,Cin]; out: [B,Ho,Wo,Cout]. */
void x1o_bottleneck_proj(const int8_t *x, const int8_t *w1, const int32_t *b1, const int32_t *m1,
                         const int8_t *w2, const int32_t *b2, const int32_t *m2,
                         const int8_t *w3, const int8_t *wp, const int32_t *b3,
                         const int32_t *m3, int S, int8_t *out, int B, int H, int W, int Cin,
                         int Cmid, int Cout)
{
    int64_t Ho = conv_out_extent(H, 3, 1, 2), Wo = conv_out_extent(W, 3, 1, 2);
    int8_t *y1 = (int8_t *)malloc((size_t)B * H * W * Cmid);
    int8_t *y2 = (int8_t *)malloc((size_t)B * Ho * Wo * Cmid);
    x1o_conv_strided(x, w1, b1, m1, S, NULL, 0, y1, B, H, W, Cin, Cmid, 1, 0, 1);
    x1o_conv_strided(y1, w2, b2, m2, S, NULL, 0, y2, B, H, W, Cmid, Cmid, 3, 1, 2);
    x1o_conv_proj(y2, w3, x, wp, b3, m3, S, out, B, (int)Ho, (int)Wo, Cmid, Cin, Cout, H, W, 2);
    free(y1);
    free(y2);
}

/* ---- the stem: convolution + BN + ReLU + max pooling --------------------------
 *
 * The Didi Cloud IFX article (inference-optimisation section) fuses
 * CONV+BN+RELU+MAXPOOL into one function; in ResNet50 that is the stem: the
 * 7x7 stride-2 convolution (pad 3) of the image, its BN and ReLU, then a 3x3
 * stride-2 max pooling (pad 1).  Max pooling takes, per channel, the largest
 * value of the window's in-image pixels (padding never wins).
 */

/* y: [B,H,W,C]; out: [B,Ho,Wo,C] with Ho = (H - 1)/2 + 1, Wo = (W - 1)/2 + 1:
 * out[b,i,j,c] = max of y[b, 2i+r-1, 2j+s-1, c] over r, s in 0..2 inside. */
void x1o_maxpool3s2(const int8_t *y, int8_t *out, int B, int H, int W, int C)
{
    int64_t Ho = conv_out_extent(H, 3, 1, 2), Wo = conv_out_extent(W, 3, 1, 2);
    for (int64_t b = 0; b < B; ++b)
        for (int64_t i = 0; i < Ho; ++i)
            for (int64_t j = 0; j < Wo; ++j)
                for (int64_t c = 0; c < C; ++c) {
                    int best = -129; /* below every int8 */
                    for (int64_t r = 0; r < 3; ++r)
                        for (int64_t s = 0; s < 3; ++s) {
                            int64_t h = 2 * i + r - 1, w = 2 * j + s - 1;
                            if (h < 0 || h >= H || w < 0 || w >= W)
                                continue;
                            int v = y[nhwc_index(b, h, w, c, H, W, C)];
                            if (v > best)
                                best = v;
                        }
                    out[nhwc_index(b, i, j, c, Ho, Wo, C)] = (int8_t)best;
                }
}

/* Stem: x1o_conv_strided (R x R, pad, stride) + BN + ReLU, then
 * x1o_maxpool3s2.  x: [B,H,W,Ic]; out: [B,Hp,Wp,Oc]. */
void x1o_conv_pool(const int8_t *x, const int8_t *wt, const int32_t *bias, const int32_t *m,
                   int S, int8_t *out, int B, int H, int W, int Ic, int Oc, int R, int pad,
                   int stride)
{
    int64_t Hc = conv_out_extent(H, R, pad, stride), Wc = conv_out_extent(W, R, pad, stride);
    int8_t *y = (int8_t *)malloc((size_t)B * Hc * Wc * Oc);
    x1o_conv_strided(x, wt, bias, m, S, NULL, 0, y, B, H, W, Ic, Oc, R, pad, stride);
    x1o_maxpool3s2(y, out, B, (int)Hc, (int)Wc, Oc);
    free(y);
}

int x1o_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}
