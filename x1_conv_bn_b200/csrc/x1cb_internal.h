// Internal host-side interfaces between the API layer and the kernels.
#pragma once
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/x1cb.h"
#include "x1cb_plan.h"

namespace x1cb {

void choose_tile(int B, int Wp, int Hp, int &tw, int &th, int &tg);
int plan_conv(ConvPlan &p, int B, int H, int W, int Ic, int Oc, int R, int has_res, int S,
              int m_r, int num_sms);
int launch_conv(const ConvPlan &p, const int8_t *x, const int8_t *w, const int32_t *bias,
                const int32_t *mult, const int8_t *r, int8_t *out, cudaStream_t stream);
unsigned int read_and_clear_dev_status(bool clear);

int launch_pack_act(const int8_t *nhwc, int8_t *nc32, int B, int H, int W, int C,
                    cudaStream_t s);
int launch_unpack_act(const int8_t *nc32, int8_t *nhwc, int B, int H, int W, int C,
                      cudaStream_t s);
int launch_pack_weight(const int8_t *oihw, int8_t *blk, int Oc, int Ic, int R, cudaStream_t s);

}  // namespace x1cb
