// Internal launch parameters shared by the library's translation units.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "mx_device.cuh"

namespace mxk {

// Upper bound on the CTAs of a reducing launch: each CTA writes one partial
// record of kPartialDoubles doubles into the caller's workspace.
constexpr int kMaxPartials = 4096;
// tensors of one grouped quantizer launch
constexpr int kFastGroupMax = 4;
constexpr int kPartialDoubles = 8;
// workspace: [0, 256) control words, then the partials.  Control words: the
// tensor-amax accumulator at byte 0, the launch ticket at byte 64.  Both are
// zero before a launch and the launch's last CTA leaves them zero.
constexpr int64_t kWsHeader = 256;
// Largest tensor a call takes (elements, exclusive): the kernels index
// elements, 8-element code words and blocks in 32 bits.
constexpr int64_t kMaxElements = INT64_C(1) << 32;
constexpr int64_t kWsTicket = 64;
// the MSE rule's tensor scale of each alternation round (floats, cleared by
// the call that used them)
constexpr int64_t kWsMseChain = 192;
constexpr int64_t kWorkspaceBytes = kWsHeader + (int64_t)kMaxPartials * kPartialDoubles * 8;

struct QParams {
    const void *x;
    int64_t rows, cols;
    void *codes;
    uint8_t *scales;
    float *tensor_scale;     // device; read when ts_mode != TS_NONE
    uint8_t *macro;
    uint16_t *offsets;
    float *rotated;          // y output (fp32), or null
    double *partials;        // per-CTA stats records, or null (no stats)
    unsigned int *amax_word; // tensor-amax accumulator (AMAX launches)
    unsigned int *ticket;    // CTAs finished (stats or a computed tensor scale), or null
    double *stats;           // MX_STATS_LEN doubles, written by the last CTA
    double count;            // elements
    ElemDesc ed;
    ScaleDesc sd;
    int block;               // B
    int lanes_per_block;     // row axis: B / 8
    int round_mode;
    int asym;
    int mbs;                 // 0 / 128
    int had;                 // 0 / 16 / 32
    int ts_mode;
    int sf_gemm;             // scales in the tcgen05 chunk layout (row axis)
    uint64_t seed;
};

struct DParams {
    const void *codes;
    const uint8_t *scales;
    const float *tensor_scale;
    const uint8_t *macro;
    const uint16_t *offsets;
    int64_t rows, cols;
    void *out;
    int out_fp32;
    ElemDesc ed;
    ScaleDesc sd;
    int block, axis, asym, mbs, had, ts_mode, sf_gemm;
};

struct SParams {
    const void *x;
    const void *xh;
    int x_fp32, xh_fp32;
    int64_t rows, cols;
    int block, axis;
    float *per_block_mse;
    double *partials;
};

// per-launch helpers implemented in the .cu files
int launch_quantize(const QParams &p, int axis, int in_fp32, int fast, cudaStream_t st,
                    int *grid_out);
int launch_tensor_amax(const QParams &p, int axis, int in_fp32, cudaStream_t st);
int launch_dequantize(const DParams &p, cudaStream_t st);
int launch_qsnr(const SParams &p, cudaStream_t st, int *grid_out);
int launch_finalize_stats(const double *partials, int nparts, double count, double *stats,
                          cudaStream_t st);
int device_sm_count();
// Resident CTAs per SM of a kernel at a block size and dynamic shared memory
// size, queried once per (kernel, threads, smem) and cached (the query and
// the shared-memory attribute are host work that would otherwise sit between
// short kernels); raises the kernel's dynamic shared-memory limit as needed.
int cached_occupancy(const void *kernel, int threads, size_t smem);

// Programmatic dependent launch: a CTA lets the next launch on the stream
// start (its CTAs take SMs as this grid's CTAs retire) and, before its first
// global access, waits until the preceding grid has completed with its
// memory visible.  Both are no-ops for a kernel launched without the
// programmatic-serialization attribute.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Launch with programmatic stream serialization (the kernel pairs it with
// pdl_trigger / pdl_wait): the launch may begin while the previous kernel on
// the stream drains.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem,
                              cudaStream_t st, Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args &&>(args)...);
}
int launch_quantize_col(const QParams &p, int axis, int in_fp32, int fast, cudaStream_t st,
                        int *grid_out);
int launch_amax_col(const QParams &p, int in_fp32, cudaStream_t st);
// E2M1 round-to-nearest-even, symmetric, row axis, no macro scale, rotation
// or rotated output: the TMA-fed persistent quantizer.
int launch_quantize_fast(const QParams &p, int in_fp32, cudaStream_t st, int *grid_out);
// CTAs of a grouped launch over n tensors with work[i] units each (a CTA
// takes at least one unit): one CTA per tensor, then one at a time to the
// tensor with the most units per CTA; cta0 gets the prefix (n + 1 entries)
inline void split_ctas(const uint64_t *work, int n, uint64_t total, uint32_t *cta0)
{
    uint64_t c[kFastGroupMax], sum = 0;
    for (int i = 0; i < n; ++i) {
        c[i] = 1;
        sum += work[i];
    }
    if (total > sum) total = sum;
    for (uint64_t k = n; k < total; ++k) {
        int best = -1;
        for (int i = 0; i < n; ++i)
            if (c[i] < work[i] && (best < 0 || work[i] * c[best] > work[best] * c[i])) best = i;
        if (best < 0) break;
        ++c[best];
    }
    cta0[0] = 0;
    for (int i = 0; i < n; ++i) cta0[i + 1] = cta0[i] + (uint32_t)c[i];
}

// one launch over ps[0..n) (n <= kFastGroupMax, one configuration, every tensor
// non-empty and eligible for launch_quantize_fast)
int launch_quantize_fast_group(const QParams *ps, int n, int in_fp32, cudaStream_t st);
// one launch of the double-buffered column / 2D quantizer over ps[0..n)
// (bf16 input, E2M1 round-to-nearest-even, symmetric, no macro scale, no
// rotation; n <= kFastGroupMax, every tensor non-empty)
int launch_quantize_colx_group(const QParams *ps, int n, int axis, cudaStream_t st);
// the tensor-amax pre-pass of ps[0..n) without rotation, one launch
int launch_tensor_amax_group(const QParams *ps, int n, int in_fp32, cudaStream_t st);
// Other element types / rounding modes / offsets, row axis, blocks of 32, no
// macro scale, rotation or rotated output: the TMA-fed persistent quantizer.
int launch_quantize_gen(const QParams &p, int in_fp32, cudaStream_t st, int *grid_out);
// Read and clear the status words of the two persistent quantizers'
// bounded waits (synchronise st); 0 when no wait gave up.
int launch_stats_refinalize(double *stats, cudaStream_t st);
int launch_quantize_mse(const QParams &p, double *records, float *chain, int in_fp32, cudaStream_t st);
int take_status_fast(cudaStream_t st, int *v);
int take_status_gen(cudaStream_t st, int *v);

}  // namespace mxk
