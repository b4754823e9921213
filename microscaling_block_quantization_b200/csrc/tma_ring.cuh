// Shared-memory ring fed by TMA for the persistent row-axis quantizers.
//
// The flat tensor is viewed as rows of one 32-element chunk (64 bytes of bf16
// or 128 of fp32).  One producer lane streams tiles of 256 chunks into a ring
// of stages with 2-D TMA copies (64- / 128-byte swizzle, so that every
// consumer lane's 16-byte reads of its own chunk are bank-conflict free); the
// eight consumer warps quantize one chunk per lane and per tile and release
// the stage.  Every mbarrier wait is bounded by the global timer: on timeout
// the wait records a code in this translation unit's status word (read and
// cleared through take_ring_status) and the kernel leaves its loop.
#pragma once
#include <cuda.h>

#include "quant_common.cuh"

namespace mxk {
namespace {

constexpr int kRingConsumers = 256;                    // 8 warps, one chunk per lane
constexpr int kRingThreads = kRingConsumers + 32;      // + producer warp
constexpr uint64_t kRingWaitNs = 2000000000ull;

__device__ int g_ring_status;

__device__ __forceinline__ uint32_t ring_saddr(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ uint64_t ring_now_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ bool ring_try(uint64_t *bar, uint32_t phase)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(ring_saddr(bar)), "r"(phase) : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool ring_wait(uint64_t *bar, uint32_t phase, int where)
{
    if (ring_try(bar, phase)) return true;
    const uint64_t t0 = ring_now_ns();
    while (!ring_try(bar, phase))
        if (ring_now_ns() - t0 > kRingWaitNs) {
            atomicCAS(&g_ring_status, 0, where);
            return false;
        }
    return true;
}

template <typename InT>
struct RingCfg {
    static constexpr int kChunkBytes = 32 * (int)sizeof(InT);
    static constexpr int kTileBytes = kRingConsumers * kChunkBytes;   // 16 KB / 32 KB
    static constexpr int kStages = sizeof(InT) == 2 ? 4 : 3;
    static constexpr int kSmem = 1024 + kStages * kTileBytes + 256;
};

// Ring layout in dynamic shared memory (1024-byte aligned for the swizzle).
template <typename InT>
struct Ring {
    uint8_t *stage0;
    uint64_t *full, *empty;
    __device__ __forceinline__ explicit Ring(uint8_t *smem_raw)
    {
        stage0 = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
        full = reinterpret_cast<uint64_t *>(stage0 + RingCfg<InT>::kStages * RingCfg<InT>::kTileBytes);
        empty = full + RingCfg<InT>::kStages;
    }
    __device__ __forceinline__ uint8_t *stage(uint32_t s) const { return stage0 + s * RingCfg<InT>::kTileBytes; }
    // thread 0; the caller synchronises the CTA afterwards
    __device__ __forceinline__ void init() const
    {
        for (int s = 0; s < RingCfg<InT>::kStages; ++s) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(ring_saddr(&full[s])), "r"(1));
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(ring_saddr(&empty[s])), "r"(kRingConsumers / 32));
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    // producer lane: the CTA's tiles first, first + stride, ...
    __device__ __forceinline__ void produce(const CUtensorMap *tm, uint32_t ntiles, int where, uint32_t first,
                                            uint32_t stride) const
    {
        constexpr uint32_t S = RingCfg<InT>::kStages;
        // the quantizer reads each input line once: mark it first to evict,
        // so that it does not displace lines other launches still need
        uint64_t pol;
        asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
        uint32_t i = 0;
        for (uint32_t tile = first; tile < ntiles; tile += stride, ++i) {
            const uint32_t s = i % S;
            if (i >= S && !ring_wait(&empty[s], ((i / S) - 1) & 1, where)) break;
            asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                         ::"r"(ring_saddr(&full[s])), "r"(RingCfg<InT>::kTileBytes) : "memory");
            asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
                         " [%0], [%1, {%3, %4}], [%2], %5;"
                         ::"r"(ring_saddr(stage(s))), "l"((uint64_t)tm), "r"(ring_saddr(&full[s])),
                           "r"(0), "r"((int)(tile * kRingConsumers)), "l"(pol)
                         : "memory");
        }
    }
    // consumer: wait for the i-th tile of this CTA
    __device__ __forceinline__ bool acquire(uint32_t i, int where) const
    {
        constexpr uint32_t S = RingCfg<InT>::kStages;
        return ring_wait(&full[i % S], (i / S) & 1, where);
    }
    // consumer warp: every lane has read its chunk of the i-th tile.  The
    // slot's next fill is an async-proxy (TMA) write, so each lane's
    // generic-proxy reads are ordered before it by a proxy fence ahead of the
    // arrive.
    __device__ __forceinline__ void release(uint32_t i) const
    {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if ((threadIdx.x & 31) == 0)
            asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];"
                         ::"r"(ring_saddr(&empty[i % RingCfg<InT>::kStages])) : "memory");
    }
};

// Lane t's chunk (row t of the stage) out of the swizzled tile.
__device__ __forceinline__ void ring_read_chunk(const uint8_t *stage, int t, const __nv_bfloat16 *, float y[32])
{
    const uint8_t *row = stage + 64 * t;
    const int sw = (t >> 1) & 3;                       // 64-byte swizzle
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint4 u = *reinterpret_cast<const uint4 *>(row + 16 * (k ^ sw));
        unpack_bf16x2(u.x, y[8 * k + 0], y[8 * k + 1]);
        unpack_bf16x2(u.y, y[8 * k + 2], y[8 * k + 3]);
        unpack_bf16x2(u.z, y[8 * k + 4], y[8 * k + 5]);
        unpack_bf16x2(u.w, y[8 * k + 6], y[8 * k + 7]);
    }
}
__device__ __forceinline__ void ring_read_chunk(const uint8_t *stage, int t, const float *, float y[32])
{
    const uint8_t *row = stage + 128 * t;
    const int sw = t & 7;                              // 128-byte swizzle
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const float4 u = *reinterpret_cast<const float4 *>(row + 16 * (k ^ sw));
        y[4 * k + 0] = u.x; y[4 * k + 1] = u.y; y[4 * k + 2] = u.z; y[4 * k + 3] = u.w;
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

inline EncodeTiledFn ring_encoder()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<EncodeTiledFn>(f);
    }
    return fn;
}

// Tensor map of x viewed as nch rows of one chunk; box = one tile.
template <typename InT>
inline int ring_map(CUtensorMap *tm, const void *x, uint64_t nch)
{
    using RC = RingCfg<InT>;
    EncodeTiledFn enc = ring_encoder();
    if (!enc) return -1;
    const cuuint64_t dims[2] = {(cuuint64_t)RC::kChunkBytes, (cuuint64_t)nch};
    const cuuint64_t strides[1] = {(cuuint64_t)RC::kChunkBytes};
    const cuuint32_t box[2] = {(cuuint32_t)RC::kChunkBytes, (cuuint32_t)kRingConsumers};
    const cuuint32_t estr[2] = {1, 1};
    return enc(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(x), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE,
               sizeof(InT) == 2 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS
               ? 0 : -1;
}

// Persistent grid: resident CTAs on every SM, no more than tiles or partial
// records.
inline unsigned ring_grid(const void *kernel, int smem, uint64_t nch)
{
    const int occ = cached_occupancy(kernel, kRingThreads, smem);
    const uint64_t ntiles = (nch + kRingConsumers - 1) / kRingConsumers;
    uint64_t g = (uint64_t)device_sm_count() * occ;
    if (g > ntiles) g = ntiles;
    if (g > (uint64_t)kMaxPartials) g = kMaxPartials;
    if (g < 1) g = 1;
    return (unsigned)g;
}

// Reads and clears this translation unit's status word (synchronises st).
inline int take_ring_status(cudaStream_t st, int *v)
{
    *v = 0;
    if (cudaMemcpyFromSymbolAsync(v, g_ring_status, sizeof(int), 0, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return -1;
    if (cudaStreamSynchronize(st) != cudaSuccess) return -1;
    if (*v == 0) return 0;
    const int zero = 0;
    if (cudaMemcpyToSymbolAsync(g_ring_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st) != cudaSuccess)
        return -1;
    return cudaStreamSynchronize(st) == cudaSuccess ? 0 : -1;
}

}  // namespace
}  // namespace mxk
