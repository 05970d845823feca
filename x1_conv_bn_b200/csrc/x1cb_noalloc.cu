// bottleneck_i8_noalloc: the Res3.x bottleneck chain for callers that cannot
// allocate device memory.
//
// Some callers have no way to hand the library a workspace: an inference
// engine's plugin whose execution step must not allocate (an allocation there
// can synchronise the device or fail under memory pressure in the middle of
// a request), or a runtime that fixes every byte of device memory when it
// starts.  For them this variant keeps the two intermediate activations of
// the chain in a fixed-size array that is part of the library image itself:
// it calls no allocator, neither CUDA's nor any framework's.
//
// The array is a file-scope __device__ variable, so every GPU on which the
// library is loaded holds it until the process exits.  Host code cannot use
// its name as a device address; the address is looked up once per device
// with cudaGetSymbolAddress (on the first call made with that device
// current) and handed to the kernels as an ordinary pointer.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "x1cb_internal.h"

namespace x1cb {
namespace {

constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(32) << 20;  // 32 MiB

static __device__ __align__(256) int8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch for the current device, looked up on
// the first call per device and cached.
int scratch_address(void **out)
{
    static std::mutex mu;
    static void *addr[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return X1CB_ERR_CUDA;
    std::lock_guard<std::mutex> lk(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();  // reset the (non-sticky) error state for later calls
            return X1CB_ERR_CUDA;
        }
        addr[dev] = p;
    }
    *out = addr[dev];
    return X1CB_OK;
}

}  // namespace
}  // namespace x1cb

extern "C" int bottleneck_i8_noalloc(const int8_t *x, const int8_t *w1, const int32_t *b1,
                                     const int32_t *m1, const int8_t *w2, const int32_t *b2,
                                     const int32_t *m2, const int8_t *w3, const int32_t *b3,
                                     const int32_t *m3, int32_t m_r, int32_t S, int8_t *out,
                                     int B, int H, int W, int Cin, int Cmid, void *stream)
{
    if (B < 0 || H < 0 || W < 0 || Cmid < 0)
        return X1CB_ERR_SHAPE;
    const size_t need = bottleneck_i8_workspace_size(B, H, W, Cmid);
    if (need > x1cb::kNoAllocScratchBytes)
        return X1CB_ERR_WORKSPACE;  // the two intermediates do not fit the built-in scratch
    if (need == 0)
        return x1cb::bottleneck_chain(x, w1, b1, m1, w2, b2, m2, w3, b3, m3, m_r, S, out,
                                      nullptr, 0, B, H, W, Cin, Cmid, stream, true);
    void *scratch = nullptr;
    if (int e = x1cb::scratch_address(&scratch))
        return e;
    // The intermediates are written in full by conv1 and conv2 before they are
    // read, so nothing in the scratch has to start at zero.
    return x1cb::bottleneck_chain(x, w1, b1, m1, w2, b2, m2, w3, b3, m3, m_r, S, out, scratch,
                                  x1cb::kNoAllocScratchBytes, B, H, W, Cin, Cmid, stream, true);
}
