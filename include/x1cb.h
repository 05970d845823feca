/*
 * x1cb: fused INT8 ResNet bottleneck convolutions for NVIDIA B200 (sm_100a).
 *
 * C ABI.  Plain pointers and sizes only; no CUDA or framework types appear in
 * the signatures (a stream is passed as `void *`, the value of a
 * cudaStream_t; NULL means the legacy default stream).
 *
 * Conventions shared by every call
 * --------------------------------
 * Layouts (Inspur MLPerf v2.0 ResNet50 convolution-merge article,
 * news.cnblogs.com/n/719672, section 3.1):
 *   activations  NC/32HW32 = [B, C/32, H, W, 32] int8: element (b, c, h, w) at
 *                (((b*C/32 + c/32)*H + h)*W + w)*32 + c%32.
 *   1x1 weights  [O1, I1, O2, I2] = [Oc/128, Ic/32, 128, 32] int8: element
 *                (o, i) at (((o/128)*Ic/32 + i/32)*128 + o%128)*32 + i%32.
 *   3x3 weights  [O1, R, S, I1, O2, I2] = [Oc/128, 3, 3, Ic/32, 128, 32] int8
 *                (this library's extension of the same blocking; the pages
 *                give no 3x3 layout).
 *   bias, m      [Oc] int32 each (folded BN: per-channel bias and fixed-point
 *                multiplier).
 * Requantisation of every output element (the article names Bn, Sum and Relu
 * after Conv3 in sections 2.2 and 3.4 and int8 data in section 3.1; this is
 * the exact integer rule the library implements):
 *   t   = (acc + bias[o]) * m[o] + r * m_r + 2^(S-1)   (64-bit, exact)
 *   out = min(max(t >> S, 0), 127)                      (>> = floor division)
 * where acc is the exact int32 sum of x*w over the receptive field and the
 * r*m_r term is present only when a residual tensor is passed.
 *
 * Memory: every pointer is DEVICE memory of the CURRENT device (cudaSetDevice),
 * owned by the caller, 16-byte aligned (bias and multipliers: 4-byte).
 * Inputs and outputs must not overlap.  Every call checks where its operands
 * live (cudaPointerGetAttributes) and returns X1CB_ERR_DEVICE for host memory
 * or another GPU's memory.  The library never allocates device memory in any
 * call.  Calls are thread-safe: host-side caches are locked, and per-device
 * state (the kernels' shared-memory opt-in) is set once per device.
 * Execution: every call only enqueues work on `stream` and returns after the
 * argument checks and the launch; results are ready when the stream is
 * synchronised.  A bounded-wait timeout inside a kernel (which never happens
 * in normal operation) is recorded in a sticky device status word, read with
 * x1cb_last_device_error().
 * Limits: stride 1 (the stride-2 entry points below excepted); 1 <= S <= 60; Ic and Oc multiples of 32 and 128 with
 * Ic <= 4096; the weights of 128 output channels (R*R*Ic*128 bytes) must fit
 * in shared memory beside the rings (Ic <= 1120 for 1x1 with a residual,
 * Ic <= 1376 for 1x1 without, Ic <= 128 for 3x3); other shapes return
 * X1CB_ERR_SHAPE;
 * requires an sm_100 device.
 * Errors: a negative X1CB_ERR_* status; nothing is launched in that case.
 */
#ifndef X1CB_H
#define X1CB_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define X1CB_OK 0
#define X1CB_ERR_NULL (-1)      /* a required pointer is NULL */
#define X1CB_ERR_SHAPE (-2)     /* a size or parameter is outside the limits above */
#define X1CB_ERR_ALIGN (-3)     /* a pointer is not 16-byte aligned */
#define X1CB_ERR_ARCH (-4)      /* no sm_100 device is current */
#define X1CB_ERR_CUDA (-5)      /* a CUDA runtime/driver call failed */
#define X1CB_ERR_TIMEOUT (-6)   /* a kernel gave up a bounded wait */
#define X1CB_ERR_WORKSPACE (-7) /* workspace missing or too small */
#define X1CB_ERR_OVERLAP (-8)   /* an output overlaps an input */
#define X1CB_ERR_DEVICE (-9)    /* an operand is not memory of the current device */

/*
 * Fused 1x1 Conv3 + folded BN + shortcut Sum + ReLU + int8 requantisation
 * (the merged Conv3+Bn+Sum+Relu kernel of the Inspur article, sections 2.2,
 * 3.3 and 3.4: the 1x1 convolution is the GEMM out[M,N] = x[M,K].w[N,K]^T
 * with M = B*H*W, N = Oc, K = Ic, and Bn+Sum+Relu is applied to the
 * accumulator before the single write-back).
 *   x    [B, Ic/32, H, W, 32]   input activations (read)
 *   w    [Oc/128, Ic/32, 128, 32] blocked weights (read)
 *   bias [Oc], m [Oc]           folded BN (read)
 *   m_r, S                      residual multiplier and shift
 *   r    [B, Oc/32, H, W, 32]   shortcut (read); may be NULL for no Sum term
 *   out  [B, Oc/32, H, W, 32]   result (written)
 * Returns X1CB_OK or a negative X1CB_ERR_*.
 */
int conv1x1_bn_add_relu_i8(const int8_t *x, const int8_t *w, const int32_t *bias,
                           const int32_t *m, int32_t m_r, int32_t S, const int8_t *r,
                           int8_t *out, int B, int H, int W, int Ic, int Oc, void *stream);

/*
 * Fused 3x3 convolution (stride 1, zero padding `pad`, which must be 1) +
 * folded BN + ReLU + int8 requantisation, no shortcut (Conv2 of the Res3.x
 * block, Inspur article section 2.2; the CONV+BN+RELU fusion of the Didi
 * Cloud IFX DAWNBench article, inference-optimisation section).
 *   x [B, Ic/32, H, W, 32]; w [Oc/128, 3, 3, Ic/32, 128, 32];
 *   bias, m [Oc]; out [B, Oc/32, H, W, 32].
 */
int conv3x3_bn_relu_i8(const int8_t *x, const int8_t *w, const int32_t *bias, const int32_t *m,
                       int32_t S, int8_t *out, int B, int H, int W, int Ic, int Oc, int pad,
                       void *stream);

/*
 * Conv2 -> Conv3 of the Res3.x bottleneck as one launch (the merge of two
 * consecutive convolutions, Inspur article section 2.1): the 3x3 pad-1
 * convolution of y1 + BN + ReLU, requantised to int8, stays on chip as the A
 * operand of the 1x1 convolution + BN + shortcut Sum with r + ReLU.  Runs on
 * pairs of SMs sharing each MMA (both weight sets on chip).
 *   y1  [B, Cmid/32, H, W, 32] (Conv1's output); w2 [Cmid/128, 3, 3, Cmid/32, 128, 32]
 *   b2, m2 [Cmid]; w3 [Cout/128, Cmid/32, 128, 32]; b3, m3 [Cout]; m_r, S
 *   r   [B, Cout/32, H, W, 32] shortcut; out [B, Cout/32, H, W, 32]
 * Requires Cmid = 128, Cout a multiple of 128 up to 1024, W <= 126 and
 * (W % 4 == 0 or W <= 64); otherwise X1CB_ERR_SHAPE (use the two separate
 * calls).  Bit-identical to conv3x3_bn_relu_i8 followed by
 * conv1x1_bn_add_relu_i8.
 */
int conv3x3_conv1x1_bn_add_relu_i8(const int8_t *y1, const int8_t *w2, const int32_t *b2,
                                   const int32_t *m2, const int8_t *w3, const int32_t *b3,
                                   const int32_t *m3, int32_t m_r, int32_t S, const int8_t *r,
                                   int8_t *out, int B, int H, int W, int Cmid, int Cout,
                                   void *stream);

/*
 * Fused 3x3 convolution of stride 2 (zero padding 1) + folded BN + ReLU +
 * int8 requantisation: Conv2 of a downsampling (projection) block such as
 * Res3.1.  The Inspur article (section 2.2) says only that Res3.1's output
 * feeds Res3.2; the block's layers are read as in the MLPerf ResNet50 (v1.5)
 * network, whose stride-2 step is this 3x3.
 *   x   [B, Ic/32, H, W, 32]        input (read)
 *   w   [Oc/128, 3, 3, Ic/32, 128, 32]
 *   out [B, Oc/32, Ho, Wo, 32] with Ho = (H - 1)/2 + 1, Wo = (W - 1)/2 + 1;
 *       output pixel (h, w) reads input rows 2h-1..2h+1, columns 2w-1..2w+1.
 * Same requantisation as above without the r term.
 */
int conv3x3s2_bn_relu_i8(const int8_t *x, const int8_t *w, const int32_t *bias,
                         const int32_t *m, int32_t S, int8_t *out, int B, int H, int W, int Ic,
                         int Oc, void *stream);

/*
 * Conv3 of a projection block with its shortcut fused in: the 1x1 Conv3 of
 * y and the stride-2 1x1 projection of the block input x are accumulated into
 * the same int32 accumulator (the projection's folded BN shares Conv3's
 * multiplier, its relative scale folded into its int8 weights), then BN, ReLU
 * and requantisation as above (no separate r term):
 *   acc = sum_i y[b,h,w,i]*w3[o,i] + sum_j x[b,2h,2w,j]*wp[o,j]
 *   y   [B, Cy/32, H, W, 32]; w3 [Oc/128, Cy/32, 128, 32]
 *   x   [B, Cx/32, Hx, Wx, 32] with 2(H-1) < Hx and 2(W-1) < Wx
 *   wp  [Oc/128, Cx/32, 128, 32]; bias, m [Oc]; out [B, Oc/32, H, W, 32]
 * The shared-memory limit applies to the combined weights (Cy + Cx per output
 * channel).
 */
int conv1x1_proj_bn_relu_i8(const int8_t *y, const int8_t *w3, const int8_t *x,
                            const int8_t *wp, const int32_t *bias, const int32_t *m, int32_t S,
                            int8_t *out, int B, int H, int W, int Cy, int Hx, int Wx, int Cx,
                            int Oc, void *stream);

/*
 * The stem's CONV+BN+RELU+MAXPOOL as one launch (the fusion the Didi Cloud
 * IFX article's inference-optimisation section lists): an R x R convolution
 * (R in {1, 3, 5, 7}, zero padding (R-1)/2, stride 1 or 2) + folded BN + ReLU,
 * requantised as above (no r term), then 3x3 stride-2 max pooling (pad 1;
 * padding never wins) -- ResNet50's 7x7 stride-2 stem with R = 7, stride = 2.
 *   x   [B, Ic/32, H, W, 32]: an image of fewer channels (3) is given as one
 *       32-channel block with the unused channels zero
 *   w   [1, R, R, Ic/32, 64, 32] (x1cb_pack_weight of [64, Ic, R, R])
 *   out [B, 2, Hp, Wp, 32]: Hc = (H + 2*((R-1)/2) - R)/stride + 1 conv rows,
 *       Hp = (Hc - 1)/2 + 1 pooled rows (likewise W)
 * Oc must be 64 (the stem's width).  Each CTA computes a tile of
 * (2pw+1) x (2ph+1) conv pixels and pools it to pw x ph; neighbouring tiles
 * recompute one shared conv row or column.
 */
int conv_bn_relu_maxpool_i8(const int8_t *x, const int8_t *w, const int32_t *bias,
                            const int32_t *m, int32_t S, int8_t *out, int B, int H, int W, int Ic,
                            int Oc, int R, int stride, void *stream);

/*
 * The same stem with the image width-folded (the layout step
 * x1cb_pack_stem): each pixel of the folded tensor carries, for one output
 * column, its filter row's R taps x Cin channels in its 32-channel block, so
 * the R x R stride-2 convolution is an R x 1 convolution (rows at stride 2,
 * columns at stride 1) with R*Cin useful channels per K step instead of Cin
 * (21 of 32 for ResNet50's 7x7 over RGB, against 3 of 32 unfolded: 7x fewer
 * MMAs for the same result).  Pad (R-1)/2, 64 outputs, then 3x3 stride-2 max
 * pooling; bit-identical to conv_bn_relu_maxpool_i8 on the unfolded image.
 * H, W are the image's dims; Wc = (W + 2*((R-1)/2) - R)/2 + 1.
 *   folded [B, 1, H, Wc, 32] (x1cb_pack_stem); wf [1, R, 1, 1, 64, 32]
 *   (x1cb_pack_stem_weight); bias, m [64]; out [B, 2, Hp, Wp, 32] as above.
 * Each CTA tile loads one box of 2*16 + R - 2 folded rows x 8 columns and
 * computes 8 x 16 conv pixels, pooled to 3 x 7.
 */
int stem_conv_bn_relu_maxpool_i8(const int8_t *folded, const int8_t *wf, const int32_t *bias,
                                 const int32_t *m, int32_t S, int8_t *out, int B, int H, int W,
                                 int R, void *stream);

/* Bytes of device workspace bottleneck_proj_i8 needs for an H x W input:
 * [B, Cmid/32, H, W, 32] and [B, Cmid/32, Ho, Wo, 32]. */
size_t bottleneck_proj_i8_workspace_size(int B, int H, int W, int Cmid);

/*
 * Projection bottleneck block (Res3.1 of ResNet50 in the MLPerf v1.5 form):
 * conv1 1x1 Cin->Cmid +BN+ReLU on H x W; conv2 3x3 stride 2 Cmid->Cmid
 * +BN+ReLU to Ho x Wo; conv3 1x1 Cmid->Cout plus the stride-2 1x1 projection
 * Cin->Cout of the block input in one accumulator, +BN+ReLU.  Three launches
 * on `stream`.
 *   x  [B, Cin/32, H, W, 32]; out [B, Cout/32, Ho, Wo, 32]
 *   w1 [Cmid/128, Cin/32, 128, 32]; w2 [Cmid/128, 3, 3, Cmid/32, 128, 32];
 *   w3 [Cout/128, Cmid/32, 128, 32]; wp [Cout/128, Cin/32, 128, 32];
 *   b1, m1, b2, m2 [Cmid]; b3, m3 [Cout] (shared by Conv3 and the projection)
 *   workspace: caller-owned, >= bottleneck_proj_i8_workspace_size() bytes
 */
int bottleneck_proj_i8(const int8_t *x, const int8_t *w1, const int32_t *b1, const int32_t *m1,
                       const int8_t *w2, const int32_t *b2, const int32_t *m2, const int8_t *w3,
                       const int8_t *wp, const int32_t *b3, const int32_t *m3, int32_t S,
                       int8_t *out, void *workspace, size_t ws_bytes, int B, int H, int W,
                       int Cin, int Cmid, int Cout, void *stream);

/* Bytes of device workspace bottleneck_i8 needs: two [B, Cmid/32, H, W, 32]
 * intermediates. */
size_t bottleneck_i8_workspace_size(int B, int H, int W, int Cmid);

/*
 * Res3.x bottleneck block (Inspur article section 2.2): conv1 1x1 Cin->Cmid
 * +BN+ReLU, conv2 3x3 pad 1 Cmid->Cmid +BN+ReLU, conv3 1x1 Cmid->Cin +BN +
 * Sum with the block input + ReLU.  With Cmid = 128, Cin <= 1024 and W <= 126
 * conv2 and conv3 run as one kernel on pairs of SMs (the merge of two
 * consecutive convolutions of the article's section 2.1): conv2's output
 * stays on chip, so the block is two launches and only conv1's output goes
 * through the workspace.  Other shapes take three launches.  No host
 * synchronisation between launches.
 *   x   [B, Cin/32, H, W, 32] block input, also the shortcut (read)
 *   w1  [Cmid/128, Cin/32, 128, 32]; w2 [Cmid/128, 3, 3, Cmid/32, 128, 32];
 *   w3  [Cin/128, Cmid/32, 128, 32]; b*, m* [Cmid], [Cmid], [Cin]
 *   m_r, S                 residual multiplier of conv3; S is shared by all
 *   out [B, Cin/32, H, W, 32] (written)
 *   workspace              caller-owned device memory of at least
 *                          bottleneck_i8_workspace_size() bytes
 */
int bottleneck_i8(const int8_t *x, const int8_t *w1, const int32_t *b1, const int32_t *m1,
                  const int8_t *w2, const int32_t *b2, const int32_t *m2, const int8_t *w3,
                  const int32_t *b3, const int32_t *m3, int32_t m_r, int32_t S, int8_t *out,
                  void *workspace, size_t ws_bytes, int B, int H, int W, int Cin, int Cmid,
                  void *stream);

/*
 * bottleneck_i8 for callers that cannot allocate device memory.  The pages
 * have no counterpart to this entry point; it exists for callers with no way
 * to pass a workspace, such as an inference engine's plugin whose execution
 * step must not allocate (allocation can synchronise the device or fail under
 * memory pressure mid-request) or a runtime that fixes all device memory at
 * start-up.  Same arguments and result as bottleneck_i8 without the
 * workspace: the two intermediates live in a 32 MiB array built into the
 * library (a file-scope __device__ array held by every GPU that loads the
 * library until the process exits).  No allocator is called.
 *   Limit: bottleneck_i8_workspace_size(B, H, W, Cmid) <= 32 MiB (for the
 *   Res3.2 block, 28x28 with Cmid = 128: B <= 167); larger problems return
 *   X1CB_ERR_WORKSPACE before anything is launched.
 *   The first call with a given device current looks up the array's device
 *   address (cudaGetSymbolAddress) and caches it; make that first call before
 *   any stream capture.
 *   Every call uses the same array, so calls that overlap on the GPU (other
 *   streams, other threads) race with each other: serialise them.  Nothing in
 *   the array needs to start at zero; its contents after a call are those of
 *   that call's intermediates.
 */
int bottleneck_i8_noalloc(const int8_t *x, const int8_t *w1, const int32_t *b1, const int32_t *m1,
                          const int8_t *w2, const int32_t *b2, const int32_t *m2,
                          const int8_t *w3, const int32_t *b3, const int32_t *m3, int32_t m_r,
                          int32_t S, int8_t *out, int B, int H, int W, int Cin, int Cmid,
                          void *stream);

/* Layout conversions on the device (offline steps of the article's section
 * 3.1).  nhwc [B, H, W, C] <-> nc32 [B, C/32, H, W, 32]; C % 32 == 0. */
int x1cb_pack_act(const int8_t *nhwc, int8_t *nc32, int B, int H, int W, int C, void *stream);
int x1cb_unpack_act(const int8_t *nc32, int8_t *nhwc, int B, int H, int W, int C, void *stream);

/* oihw [Oc, Ic, R, R] (the usual convolution weight order) -> blocked
 * [Oc/O2, R, R, Ic/32, O2, 32] with O2 = 128 (O2 = 64 for a 64-channel
 * layer); R in {1, 3, 5, 7}. */
int x1cb_pack_weight(const int8_t *oihw, int8_t *blocked, int Oc, int Ic, int R, void *stream);

/* Width-folded stem input: nhwc [B, H, W, Cin] image -> folded
 * [B, 1, H, Wc, 32], Wc = (W + 2*((R-1)/2) - R)/2 + 1 (the stride-2 output
 * columns), with channel ds*Cin + ci of pixel (h, c) = channel ci of image
 * pixel (h, 2c - (R-1)/2 + ds), zero outside the image and from R*Cin on;
 * needs R*Cin <= 32. */
int x1cb_pack_stem(const int8_t *nhwc, int8_t *folded, int B, int H, int W, int Cin, int R,
                   void *stream);

/* Folded stem weights: oihw [64, Cin, R, R] -> [1, R, 1, 1, 64, 32] with entry
 * (dr, o, ds*Cin + ci) = w[o, ci, dr, ds], zero from R*Cin on. */
int x1cb_pack_stem_weight(const int8_t *oihw, int8_t *blocked, int Oc, int Cin, int R,
                          void *stream);

/* Human-readable name of a status code (static storage). */
const char *x1cb_status_string(int status);

/* Synchronises the current device, then returns X1CB_ERR_TIMEOUT if any
 * kernel since the last clear gave up a bounded wait, else X1CB_OK (or
 * X1CB_ERR_CUDA if the device cannot be read).  The raw bits go to *bits
 * when bits is not NULL.  clear != 0 resets the word. */
int x1cb_last_device_error(unsigned int *bits, int clear);

/* Synchronises the current device, then writes to *bits which exact
 * epilogue forms the kernels launched since the last clear ran (bit 0: the
 * generic 64-bit definition, 1: the 64-bit high-word form, 2: the all-32-bit
 * form, 3: the all-32-bit form with the bias added by the tensor core).  Every
 * form gives the same bytes; this only shows which arithmetic a shape and its
 * constants reached.  clear != 0 resets the record.  Returns X1CB_OK or an
 * error. */
int x1cb_last_epilogue_forms(unsigned int *bits, int clear);

/* Timeline trace of the kernels' pipeline roles, present only in a library
 * built with -DX1CB_TRACE (the default build returns 0 and copies nothing).
 * Synchronises the current device, copies up to `words` 64-bit entries of the
 * trace table to host memory `host` and, with clear != 0, zeroes the table.
 * Layout: [cta 0..3][event 0..15][n 0..1023] of SM clock values (0: not
 * recorded); the events of each kernel are listed where it records them.
 * Returns the number of entries copied, or a negative X1CB_ERR_* code. */
long long x1cb_trace_copy(unsigned long long *host, long long words, int clear);

/* enable = 1 makes bottleneck_i8 (and bottleneck_i8_noalloc) run conv2 and
 * conv3 as one launch (the fused conv2 -> conv3 kernel on CTA pairs) where
 * that form applies; 0 (the default) runs them as two launches, which
 * measured faster on B200 for the Res3.2 block (B = 1024: 419 against
 * 443 us per block).  Same results either way. */
void x1cb_set_block_fusion(int enable);

/* Limit of every in-kernel wait, in nanoseconds (default 2 s; 0 restores the
 * default).  Applies to launches made after the call. */
void x1cb_set_wait_limit_ns(unsigned long long ns);

/* Test hook: mode 1 makes the next launches' MMA warp wait on a barrier that
 * nothing arrives on, so the bounded-wait path runs out and reports
 * X1CB_ERR_TIMEOUT without hanging; mode 0 restores normal operation. */
void x1cb_debug_inject(int mode);

/* Describes the launch plan chosen for a convolution shape into buf (a
 * short text of key=value fields), for tests and benchmarks: cta_pair=1
 * marks a shortcut layer that runs on clusters of two CTAs sharing each MMA,
 * and a trailing "pair=1 pair_..." group gives the plan of a 128 -> 128 3x3
 * (stride 1 or 2), which runs on CTA pairs instead of the single-CTA plan
 * before it.  Returns X1CB_OK or an error. */
int x1cb_describe_plan(int B, int H, int W, int Ic, int Oc, int R, int has_res, char *buf,
                       size_t len);

/* As x1cb_describe_plan for an Hin x Win input at `stride` (pad (R-1)/2),
 * optionally with a projection source of Ic2 channels (1x1, stride 2, over a
 * 2H x 2W image; R = 1 and stride = 1 then) or with max pooling (pool != 0;
 * Oc = 64). */
int x1cb_describe_plan_ex(int B, int Hin, int Win, int Ic, int Oc, int R, int stride, int Ic2,
                          int has_res, int pool, char *buf, size_t len);

/* Describes the fused conv2 -> conv3 plan of a bottleneck block (tiles, ring
 * depths, shared memory, and the clusters of two CTAs the current device can
 * hold at once; 0 without a device).  X1CB_ERR_SHAPE when the block has no
 * fused form. */
int x1cb_describe_chain(int B, int H, int W, int Cmid, int Cout, char *buf, size_t len);

/* Library version, e.g. "x1cb 0.2.0 sm_100a". */
const char *x1cb_version(void);

#ifdef __cplusplus
}
#endif
#endif /* X1CB_H */
