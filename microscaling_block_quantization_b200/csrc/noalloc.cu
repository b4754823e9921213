// mx_quantize_noalloc: mx_quantize for callers that cannot allocate device
// memory -- plain C callers that link only this library and hold no device
// allocator, code that runs while a CUDA graph is being captured (where
// cudaMalloc is not allowed), or services that reserved all of HBM for
// weights and caches up front.  The scratch space mx_quantize takes from the
// caller (tensor-amax word and per-CTA statistics records) lives instead in a
// fixed array of this library's device image.
#include <cuda_runtime.h>
#include <mutex>
#include <stdint.h>

#include "mx.h"
#include "mx_internal.h"

namespace {

// Largest scratch mx_quantize can need: a 256-byte header plus one 64-byte
// record for each of at most 4096 CTAs (262,400 bytes).  Every GPU that loads
// the library holds this array until the process exits.
constexpr int64_t kScratchBytes = mxk::kWorkspaceBytes;
static __device__ __align__(256) uint8_t g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void *g_scratch_ptr[kMaxDevices];
std::mutex g_mu;

// Device address of g_scratch on the current device, resolved once per device
// (host code only sees a host-side stand-in under that name).
int scratch_for_current_device(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MX_ERR_NO_DEVICE;
    if (dev < 0 || dev >= kMaxDevices) return MX_ERR_NO_DEVICE;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return MX_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return MX_OK;
}

}  // namespace

extern "C" int mx_quantize_noalloc(const mx_config *cfg, const void *x, int32_t x_dtype, int64_t rows,
                                   int64_t cols, void *codes, uint8_t *scales, float *tensor_scale,
                                   uint8_t *macro_scales, uint16_t *offsets, double *stats,
                                   void *stream)
{
    mx_sizes s;
    int rc = mx_query_sizes(cfg, rows, cols, &s);
    if (rc != MX_OK) return rc;
    // a given amax lives in a caller's workspace, which this entry has none
    // of; rotation (mx_hadamard_quantize) is a separate entry point
    if (cfg->tensor_scale == MX_TS_AMAX || cfg->hadamard) return MX_ERR_UNSUPPORTED;
    if (s.workspace_bytes > kScratchBytes) return MX_ERR_WORKSPACE;
    void *scratch = nullptr;
    rc = scratch_for_current_device(&scratch);
    if (rc != MX_OK) return rc;
    // The scratch needs no clearing: its control words are zero at load and
    // every call leaves them zero, and every statistics record a call reads is
    // written earlier in the same call.
    rc = mx_quantize(cfg, x, x_dtype, rows, cols, codes, scales, tensor_scale, macro_scales, offsets,
                     stats, scratch, kScratchBytes, stream);
    // A launch that failed after an earlier one of the same call was queued
    // (the tensor-amax pass, an MSE round) can leave a control word set, and
    // unlike a caller's workspace nobody else can clear this one: queue a
    // reset of the 256-byte header behind whatever did run (a memset node,
    // no allocation).
    if (rc == MX_ERR_CUDA)
        (void)cudaMemsetAsync(scratch, 0, mxk::kWsHeader, static_cast<cudaStream_t>(stream));
    return rc;
}
