// Internal host-side interfaces between the API layer and the kernels.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/x1cb.h"
#include "x1cb_plan.h"

namespace x1cb {

void choose_tile(int B, int Wp, int Hp, int kb, int &tw, int &th, int &tg);
void choose_halo_tile(int B, int H, int W, int &th, int &tg);
int encode_map(CUtensorMap *m, const void *base, int rank, const uint64_t *dims,
               const uint64_t *strides_bytes, const uint32_t *box, CUtensorMapSwizzle swz,
               CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_UINT8,
               const uint32_t *elem_strides = nullptr);
int opt_in_smem(const void *kern, int which);
int plan_conv(ConvPlan &p, int B, int H, int W, int Ic, int Oc, int R, int has_res, int S,
              int m_r, int num_sms);
// Geometry beyond the plain stride-1 layer: the input image is Hin x Win and
// the stride `stride` (output H x W); optionally a second 1x1 source of Ic2
// channels at stride `stride2` over a Hin2 x Win2 image, accumulated into the
// same outputs (Ic2 = 0: none).
struct ConvGeom {
    int stride = 1, Hin = 0, Win = 0;
    int Ic2 = 0, stride2 = 1, Hin2 = 0, Win2 = 0;
    int pool = 0;  // 3x3 stride-2 max pooling after the ReLU (64-channel layers)
    int Rw = 0;    // filter width when it differs from the height (0: square)
    int stride_w = 0;  // column stride when it differs from the row stride (0: same)
};
int plan_conv_ex(ConvPlan &p, int B, int H, int W, int Ic, int Oc, int R, int has_res, int S,
                 int m_r, int num_sms, const ConvGeom &g);
int launch_conv(const ConvPlan &p, const int8_t *x, const int8_t *w, const int32_t *bias,
                const int32_t *mult, const int8_t *r, int8_t *out, cudaStream_t stream,
                const int8_t *x2 = nullptr, const int8_t *w2 = nullptr);
// Fused Conv2 -> Conv3: plan (X1CB_ERR_SHAPE when the shape has no fused
// form) and launch.  y1 [B, Cm/32, H, W, 32] is Conv1's output, x the block
// input (the shortcut), out the block output.
int plan_chain(ChainPlan &p, int B, int H, int W, int Cm, int Cout, int S, int m_r);
int plan_conv2_pair(ChainPlan &p, int B, int H, int W, int S, int stride = 1, int Hin = 0,
                    int Win = 0);
int resident_clusters(int smem, int &clusters, bool c3 = true);
int launch_chain(const ChainPlan &p, const int8_t *y1, const int8_t *w2, const int32_t *b2,
                 const int32_t *m2, const int8_t *w3, const int32_t *b3, const int32_t *m3,
                 const int8_t *x, int8_t *out, cudaStream_t stream);

// Device addresses of the sticky status word and the epilogue-forms word of
// the current device (for kernels outside the convolution's translation unit).
int device_words(unsigned int **status, unsigned int **forms);
unsigned int read_and_clear_dev_status(bool clear);
// Timeline table of trace builds (null in the default build); copy_trace
// copies up to `words` of it to the host (returns the words copied).
unsigned long long *trace_table();
long long copy_trace(unsigned long long *host, long long words, bool clear);
unsigned int read_and_clear_dev_forms(bool clear);

// The bottleneck chain behind bottleneck_i8 and bottleneck_i8_noalloc.
// ws_checked: the workspace was supplied by the library itself (its own
// device array), so its residency is not re-checked.
int bottleneck_chain(const int8_t *x, const int8_t *w1, const int32_t *b1, const int32_t *m1,
                     const int8_t *w2, const int32_t *b2, const int32_t *m2, const int8_t *w3,
                     const int32_t *b3, const int32_t *m3, int32_t m_r, int32_t S, int8_t *out,
                     void *workspace, size_t ws_bytes, int B, int H, int W, int Cin, int Cmid,
                     void *stream, bool ws_trusted);

int launch_pack_act(const int8_t *nhwc, int8_t *nc32, int B, int H, int W, int C,
                    cudaStream_t s);
int launch_unpack_act(const int8_t *nc32, int8_t *nhwc, int B, int H, int W, int C,
                      cudaStream_t s);
int launch_pack_weight(const int8_t *oihw, int8_t *blk, int Oc, int Ic, int R, cudaStream_t s);
int launch_pack_stem(const int8_t *nhwc, int8_t *folded, int B, int H, int W, int Cin, int R,
                     cudaStream_t s);
int launch_pack_stem_weight(const int8_t *oihw, int8_t *blk, int Oc, int Cin, int R,
                            cudaStream_t s);

}  // namespace x1cb
