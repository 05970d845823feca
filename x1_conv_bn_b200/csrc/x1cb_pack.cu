// Layout conversions (Inspur MLPerf ResNet50 convolution-merge article,
// news.cnblogs.com/n/719672, section 3.1): NHWC <-> NC/32HW32 activations and
// OIHW -> blocked [O1, R, S, I1, O2, I2=32] weights (O2 = 128, or Oc below 128).  These are the
// article's offline preparation steps; they move 32-byte channel chunks with
// 16-byte vector accesses.
#include <cuda_runtime.h>

#include <cstdint>

#include "x1cb_internal.h"

namespace x1cb {
namespace {

// One thread per (image, channel block, pixel): consecutive threads take
// consecutive pixels of one channel block, so the NC/32HW32 side is fully
// contiguous and the NHWC side reads whole 32-byte sectors.
__global__ void pack_act_kernel(const int8_t *__restrict__ nhwc, int8_t *__restrict__ nc32,
                                long long B, long long HW, long long C)
{
    const long long C1 = C / 32;
    const long long n = B * C1 * HW;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long hw = i % HW;
        const long long c1 = (i / HW) % C1;
        const long long b = i / (HW * C1);
        const uint4 *src = reinterpret_cast<const uint4 *>(nhwc + (b * HW + hw) * C + c1 * 32);
        uint4 *dst = reinterpret_cast<uint4 *>(nc32 + i * 32);
        const uint4 a = src[0], c = src[1];
        dst[0] = a;
        dst[1] = c;
    }
}

__global__ void unpack_act_kernel(const int8_t *__restrict__ nc32, int8_t *__restrict__ nhwc,
                                  long long B, long long HW, long long C)
{
    const long long C1 = C / 32;
    const long long n = B * C1 * HW;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long hw = i % HW;
        const long long c1 = (i / HW) % C1;
        const long long b = i / (HW * C1);
        const uint4 *src = reinterpret_cast<const uint4 *>(nc32 + i * 32);
        uint4 *dst = reinterpret_cast<uint4 *>(nhwc + (b * HW + hw) * C + c1 * 32);
        const uint4 a = src[0], c = src[1];
        dst[0] = a;
        dst[1] = c;
    }
}

// One thread per destination byte (weights are small).
__global__ void pack_weight_kernel(const int8_t *__restrict__ oihw, int8_t *__restrict__ blk,
                                   int Oc, int Ic, int R)
{
    const long long n = static_cast<long long>(Oc) * Ic * R * R;
    const int I1 = Ic / 32;
    const int O2 = Oc < 128 ? Oc : 128;  // a 64-channel layer is one block of 64
    for (long long d = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; d < n;
         d += static_cast<long long>(gridDim.x) * blockDim.x) {
        // d = ((((ob*R + r)*R + s)*I1 + i1)*O2 + o2)*32 + i2
        long long t = d;
        const int i2 = static_cast<int>(t % 32);
        t /= 32;
        const int o2 = static_cast<int>(t % O2);
        t /= O2;
        const int i1 = static_cast<int>(t % I1);
        t /= I1;
        const int s = static_cast<int>(t % R);
        t /= R;
        const int r = static_cast<int>(t % R);
        const int ob = static_cast<int>(t / R);
        const long long o = static_cast<long long>(ob) * O2 + o2;
        const long long i = static_cast<long long>(i1) * 32 + i2;
        blk[d] = oihw[((o * Ic + i) * R + r) * R + s];
    }
}

// The stem's width-folded image: pixel (h, c) of the folded tensor
// [B, 1, H, Wc, 32] (Wc output columns of the stride-2 convolution) holds, in
// channel ds*Cin + ci, channel ci of image pixel (h, 2c - pad + ds) for the R
// taps ds of a filter row (zero outside the image; channels from R*Cin on are
// zero).  The R x R stride-2 convolution of the image then is an R x 1
// convolution of the folded tensor, stride 2 along rows and 1 along columns.
// One thread per folded pixel.
__global__ void pack_stem_kernel(const int8_t *__restrict__ nhwc, int8_t *__restrict__ folded,
                                 int B, int H, int W, int Wc, int Cin, int R)
{
    const long long n = static_cast<long long>(B) * H * Wc;
    const int pad = (R - 1) / 2;
    for (long long q = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; q < n;
         q += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int c = static_cast<int>(q % Wc);
        const long long bh = q / Wc;  // b * H + h
        uint32_t words[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        for (int ds = 0; ds < R; ++ds) {
            const int w = 2 * c - pad + ds;
            if (w < 0 || w >= W)
                continue;
            const int8_t *src = nhwc + (bh * W + w) * Cin;
            for (int ci = 0; ci < Cin; ++ci) {
                const int k = ds * Cin + ci;
                words[k >> 2] |= static_cast<uint32_t>(static_cast<uint8_t>(src[ci]))
                                  << (8 * (k & 3));
            }
        }
        uint4 *dst = reinterpret_cast<uint4 *>(folded + q * 32);
        dst[0] = make_uint4(words[0], words[1], words[2], words[3]);
        dst[1] = make_uint4(words[4], words[5], words[6], words[7]);
    }
}

// Folded stem weights: [1, R, 1, 1, Oc, 32] with entry (dr, o, ds*Cin + ci) =
// w[o, ci, dr, ds] of the OIHW weight [Oc, Cin, R, R] (zero from R*Cin on).
__global__ void pack_stem_weight_kernel(const int8_t *__restrict__ oihw,
                                        int8_t *__restrict__ blk, int Oc, int Cin, int R)
{
    const long long n = static_cast<long long>(R) * Oc * 32;
    for (long long d = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; d < n;
         d += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int c = static_cast<int>(d % 32);
        const int o = static_cast<int>((d / 32) % Oc);
        const int dr = static_cast<int>(d / (32LL * Oc));
        int8_t v = 0;
        if (c < R * Cin) {
            const int ds = c / Cin, ci = c % Cin;
            v = oihw[((static_cast<long long>(o) * Cin + ci) * R + dr) * R + ds];
        }
        blk[d] = v;
    }
}

int grid_for(long long n, int threads)
{
    long long g = (n + threads - 1) / threads;
    if (g > 148LL * 64)
        g = 148LL * 64;
    return static_cast<int>(g < 1 ? 1 : g);
}

}  // namespace

int launch_pack_act(const int8_t *nhwc, int8_t *nc32, int B, int H, int W, int C, cudaStream_t s)
{
    const long long n = static_cast<long long>(B) * H * W * (C / 32);
    if (n == 0)
        return X1CB_OK;
    pack_act_kernel<<<grid_for(n, 256), 256, 0, s>>>(nhwc, nc32, B, static_cast<long long>(H) * W,
                                                      C);
    return cudaGetLastError() == cudaSuccess ? X1CB_OK : X1CB_ERR_CUDA;
}

int launch_unpack_act(const int8_t *nc32, int8_t *nhwc, int B, int H, int W, int C, cudaStream_t s)
{
    const long long n = static_cast<long long>(B) * H * W * (C / 32);
    if (n == 0)
        return X1CB_OK;
    unpack_act_kernel<<<grid_for(n, 256), 256, 0, s>>>(nc32, nhwc, B,
                                                        static_cast<long long>(H) * W, C);
    return cudaGetLastError() == cudaSuccess ? X1CB_OK : X1CB_ERR_CUDA;
}

int launch_pack_weight(const int8_t *oihw, int8_t *blk, int Oc, int Ic, int R, cudaStream_t s)
{
    const long long n = static_cast<long long>(Oc) * Ic * R * R;
    if (n == 0)
        return X1CB_OK;
    pack_weight_kernel<<<grid_for(n, 256), 256, 0, s>>>(oihw, blk, Oc, Ic, R);
    return cudaGetLastError() == cudaSuccess ? X1CB_OK : X1CB_ERR_CUDA;
}

}  // namespace x1cb

namespace x1cb {

int launch_pack_stem(const int8_t *nhwc, int8_t *folded, int B, int H, int W, int Cin, int R,
                     cudaStream_t s)
{
    const int pad = (R - 1) / 2;
    const int Wc = W + 2 * pad >= R ? (W + 2 * pad - R) / 2 + 1 : 0;
    const long long n = static_cast<long long>(B) * H * Wc;
    pack_stem_kernel<<<grid_for(n, 256), 256, 0, s>>>(nhwc, folded, B, H, W, Wc, Cin, R);
    return cudaGetLastError() == cudaSuccess ? X1CB_OK : X1CB_ERR_CUDA;
}

int launch_pack_stem_weight(const int8_t *oihw, int8_t *blk, int Oc, int Cin, int R,
                            cudaStream_t s)
{
    const long long n = static_cast<long long>(R) * Oc * 32;
    pack_stem_weight_kernel<<<grid_for(n, 256), 256, 0, s>>>(oihw, blk, Oc, Cin, R);
    return cudaGetLastError() == cudaSuccess ? X1CB_OK : X1CB_ERR_CUDA;
}

}  // namespace x1cb
