// Block-scaled FP4 GEMM on the sm_100a 5th-generation tensor cores, and the
// post-operation QSNR of "Unveiling the Potential of Quantization with MXFP4"
// (Sec.3 Eq. (2)); the product is the A B^T of the same page's Fig. 5 (MBS
// matrix multiply), the Blackwell FP4 GEMM of "Bridging the Gap ...
// Microscaling FP4 Quantization" (sec. 2.3).
//
// One CTA computes a 128 x 128 tile of C = A^Q (B^Q)^T with FP32 accumulation
// in tensor memory:
//   warp 0       TMA producer: 2-D tensor copies of the packed E2M1 (or bf16)
//                tiles with 128-byte swizzle, 1-D bulk copies of the scale
//                chunks (512-byte 128-row x 4-scale chunks, written in that
//                layout by the quantizer), one mbarrier per stage;
//   warp 1       tensor memory owner and MMA issuer: tcgen05.cp of the scale
//                chunks into tensor memory, tcgen05.mma kind::mxf4 (E8M0,
//                32-element blocks) / kind::mxf4nvf4 (UE4M3, 16-element
//                blocks) / kind::f16 (bf16), tcgen05.commit to free stages;
//   warps 2..5   epilogue: tcgen05.ld of the accumulator lanes of their
//                quadrant, per-tensor scales, the C store.
// The persistent 128 x 256 kernel (k_gemm_p) and the fused QSNR(AB) kernel
// (k_gemm_qsnr_f: both products of one output tile in turn, the error sums
// reduced in the epilogue, C never written) follow below.
// Every TMA load targets its own CTA only; every wait on an mbarrier is bounded and sets a
// device status word instead of hanging.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "mx.h"
#include "mx_internal.h"

namespace mxg {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int kStages = 3;
constexpr int kThreads = 192;
constexpr int kTmemCols = 256;
constexpr int kTileBytes = BM * 128;              // one operand tile: 128 rows x 128 bytes
constexpr uint64_t kWaitNs = 2000000000ull;       // bound of one mbarrier wait: 2 s

enum { KIND_BF16 = 0, KIND_MXF4 = 1, KIND_NVF4 = 2, KIND_MXF6 = 3 };
constexpr uint32_t kFmtE2M1 = 5;     // E2M1 in the kind::mxf8f6f4 instruction descriptor
enum { EPI_BF16 = 0, EPI_F32 = 1 };

// device status word of the bounded waits (read and cleared by mx_device_status)
__device__ int g_status;

struct GParams {
    int M, N, K;
    const uint8_t *sfa, *sfb;    // scale chunks (FP4 kinds)
    const float *tsA, *tsB;      // per-tensor scales or null
    void *C;                     // EPI_BF16 / EPI_F32 output, row-major M x N
    double *partials;            // QSNR(AB): per-CTA [sum C_ref^2, sum (C_ref - C_q)^2]
    double *stats;               // QSNR(AB): [sum C_ref^2, sum (C_ref - C_q)^2, dB]
    uint32_t ab_fmt;             // KIND_MXF6: A / B element formats of the instruction descriptor
    uint32_t stage_tx;           // KIND_MXF6: bytes the TMA brings per stage (A, B and scales)
};

template <int KIND>
struct Kind {
    static constexpr int kChunks = KIND == KIND_MXF4 ? 2 : KIND == KIND_NVF4 ? 4 : 0;  // per stage
    static constexpr int kSfBytes = kChunks * 512;                                    // per operand
    static constexpr int kKPerStage = KIND == KIND_BF16 ? 64 : 256;                   // elements
    static constexpr int kStageBytes = 2 * kTileBytes + 2 * kSfBytes;
    static constexpr int kSfCols = 2 * kChunks * 4;                                   // TMEM columns
};

// ------------------------------------------------------------ primitives --
__device__ __forceinline__ uint32_t saddr(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(saddr(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(saddr(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t *bar, uint32_t phase)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(saddr(bar)), "r"(phase) : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t now_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Bounded wait: false (and the status word set) once kWaitNs have passed.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t phase, int where)
{
    if (mbar_try(bar, phase)) return true;
    const uint64_t t0 = now_ns();
    while (true) {
        if (mbar_try(bar, phase)) return true;
        if (now_ns() - t0 > kWaitNs) break;
    }
    atomicCAS(&g_status, 0, where);
    return false;
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar, int x, int y)
{
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%3, %4}], [%2];"
                 ::"r"(saddr(dst)), "l"((uint64_t)map), "r"(saddr(bar)), "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(saddr(dst)), "l"(src), "r"(bytes), "r"(saddr(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(saddr(bar)) : "memory");
}

// K-major operand tile with 128-byte swizzle: 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr)
{
    uint64_t d = (uint64_t)((addr >> 4) & 0x3fffu);
    d |= (uint64_t)1 << 16;                  // leading byte offset (16 B units; unused by SW128 K-major)
    d |= (uint64_t)(1024 >> 4) << 32;        // stride byte offset: 8 rows x 128 B
    d |= (uint64_t)1 << 46;                  // descriptor version (sm100)
    d |= (uint64_t)2 << 61;                  // SWIZZLE_128B
    return d;
}
// 32 rows x 16 bytes, unswizzled (a scale chunk): 8-row groups 128 bytes apart.
__device__ __forceinline__ uint64_t desc_sf(uint32_t addr)
{
    uint64_t d = (uint64_t)((addr >> 4) & 0x3fffu);
    d |= (uint64_t)(128 >> 4) << 16;
    d |= (uint64_t)(128 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    return d;
}

// Instruction descriptors (M = 128, N = BN, K-major operands, FP32 accumulate).
template <int KIND>
__device__ __forceinline__ uint32_t idesc_base()
{
    uint32_t d = 0;
    if (KIND == KIND_BF16) {
        d |= 1u << 4;      // accumulator F32
        d |= 1u << 7;      // A bf16
        d |= 1u << 10;     // B bf16
    } else {
        d |= 1u << 7;      // A E2M1
        d |= 1u << 10;     // B E2M1
        if (KIND == KIND_MXF4) d |= 1u << 23;   // scales UE8M0 (UE4M3 = 0)
    }
    d |= (uint32_t)(BN >> 3) << 17;
    d |= (uint32_t)(BM >> 4) << 24;
    return d;
}

template <int KIND>
__device__ __forceinline__ void mma(uint32_t dt, uint64_t ad, uint64_t bd, uint32_t idesc, uint32_t sfa,
                                    uint32_t sfb, uint32_t acc)
{
    if constexpr (KIND == KIND_BF16) {
        asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                     "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
                     ::"r"(dt), "l"(ad), "l"(bd), "r"(idesc), "r"(acc), "r"(0), "r"(0), "r"(0), "r"(0));
        (void)sfa;
        (void)sfb;
    } else if constexpr (KIND == KIND_MXF4) {
        asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                     "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
                     ::"r"(dt), "l"(ad), "l"(bd), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb));
    } else if constexpr (KIND == KIND_MXF6) {
        asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                     "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
                     ::"r"(dt), "l"(ad), "l"(bd), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb));
    } else {
        asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                     "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
                     ::"r"(dt), "l"(ad), "l"(bd), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb));
    }
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float v[32])
{
    uint32_t r[32];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32"
                 " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15,"
                 " %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
                   "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
                   "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
                   "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
                   "=r"(r[31])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// ---------------------------------------------------------------- kernel --
template <int KIND, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    k_gemm(const GParams p, const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB)
{
    using KT = Kind<KIND>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *sA = smem;                                   // kStages x 16 KB
    uint8_t *sB = sA + kStages * kTileBytes;              // kStages x 16 KB
    uint8_t *sSFA = sB + kStages * kTileBytes;            // kStages x kSfBytes
    uint8_t *sSFB = sSFA + kStages * KT::kSfBytes;
    uint64_t *full = reinterpret_cast<uint64_t *>(sSFB + kStages * KT::kSfBytes);
    uint64_t *empty = full + kStages;
    uint64_t *accf = empty + kStages;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(accf + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    const int ktiles = p.K / KT::kKPerStage;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accf, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(saddr(tmem_holder)), "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_holder;
    const uint32_t tsf = tbase + BN;                      // scale-factor ring after the accumulator

    if (warp == 0) {
        if (lane == 0) {
            const int sfrow_chunks = (p.K / (KIND == KIND_MXF4 ? 32 : 16)) / 4;   // chunks per 128 rows
            for (int kt = 0; kt < ktiles; ++kt) {
                const int s = kt % kStages;
                if (kt >= kStages && !mbar_wait(&empty[s], ((kt / kStages) - 1) & 1, 1)) break;
                mbar_expect_tx(&full[s], KT::kStageBytes);
                const int kx = KIND == KIND_BF16 ? kt * 64 : kt * 128;    // elements (bf16) / bytes (FP4)
                tma_load_2d(sA + s * kTileBytes, &tmA, &full[s], kx, m0);
                tma_load_2d(sB + s * kTileBytes, &tmB, &full[s], kx, n0);
                if constexpr (KIND != KIND_BF16) {
                    const size_t ca = ((size_t)(m0 / 128) * sfrow_chunks + (size_t)kt * KT::kChunks) * 512;
                    const size_t cb = ((size_t)(n0 / 128) * sfrow_chunks + (size_t)kt * KT::kChunks) * 512;
                    bulk_load(sSFA + s * KT::kSfBytes, p.sfa + ca, KT::kSfBytes, &full[s]);
                    bulk_load(sSFB + s * KT::kSfBytes, p.sfb + cb, KT::kSfBytes, &full[s]);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc0 = idesc_base<KIND>();
            bool ok = true;
            for (int kt = 0; kt < ktiles; ++kt) {
                const int s = kt % kStages;
                if (!mbar_wait(&full[s], (kt / kStages) & 1, 2)) { ok = false; break; }
                tc_fence_after();
                const uint32_t sfa_t = tsf + s * KT::kSfCols;           // this stage's scale columns
                const uint32_t sfb_t = sfa_t + KT::kChunks * 4;
                if constexpr (KIND != KIND_BF16) {
#pragma unroll
                    for (int c = 0; c < KT::kChunks; ++c) {
                        asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;"
                                     ::"r"(sfa_t + 4 * c), "l"(desc_sf(saddr(sSFA + s * KT::kSfBytes + c * 512))));
                        asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;"
                                     ::"r"(sfb_t + 4 * c), "l"(desc_sf(saddr(sSFB + s * KT::kSfBytes + c * 512))));
                    }
                }
                const uint32_t a0 = saddr(sA + s * kTileBytes), b0 = saddr(sB + s * kTileBytes);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    // each MMA covers 32 bytes of the 128-byte row: K = 64 (FP4) or 16 (bf16)
                    uint32_t idesc = idesc0, sfa = 0, sfb = 0;
                    if constexpr (KIND == KIND_MXF4) {
                        const uint32_t id = (k & 1) * 2;                 // byte of the 4-scale word
                        idesc |= (id << 29) | (id << 4);
                        sfa = sfa_t + 4 * (k >> 1);
                        sfb = sfb_t + 4 * (k >> 1);
                    } else if constexpr (KIND == KIND_NVF4) {
                        sfa = sfa_t + 4 * k;
                        sfb = sfb_t + 4 * k;
                    }
                    mma<KIND>(tbase, desc_sw128(a0 + 32 * k), desc_sw128(b0 + 32 * k), idesc, sfa, sfb,
                              (kt > 0 || k > 0) ? 1u : 0u);
                }
                tc_commit(&empty[s]);
            }
            if (ok) tc_commit(accf);
        }
        __syncwarp();
    } else {
        // epilogue: warp w reads accumulator lanes 32 * (w % 4) .. + 31
        const int q = warp & 3;
        const int row = m0 + 32 * q + lane;
        const bool ready = mbar_wait(accf, 0, 3);
        tc_fence_after();
        float scale = 1.0f;
        if (p.tsA) scale = __fmul_rn(scale, *p.tsA);
        if (p.tsB) scale = __fmul_rn(scale, *p.tsB);
        if (ready) {
#pragma unroll 1
            for (int ch = 0; ch < BN / 32; ++ch) {
                float v[32];
                tmem_ld32(tbase + ((uint32_t)(32 * q) << 16) + ch * 32, v);
                const int col = n0 + ch * 32;
                if constexpr (EPI == EPI_BF16) {
                    __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(p.C) + (size_t)row * p.N + col;
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                        uint32_t w[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            w[j] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[i + 2 * j] * scale)) |
                                   ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[i + 2 * j + 1] * scale)) << 16);
                        *reinterpret_cast<uint4 *>(dst + i) = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                } else {
                    float *dst = static_cast<float *>(p.C) + (size_t)row * p.N + col;
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        *reinterpret_cast<float4 *>(dst + i) =
                            make_float4(v[i] * scale, v[i + 1] * scale, v[i + 2] * scale, v[i + 3] * scale);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tbase), "r"(kTmemCols));
    }
}

// ---------------------------------------------------------------------------
// Persistent 128 x 256 variant for the FP4 kinds: one CTA per SM walks its
// share of the output tiles; 4 stages of A (16 KB) + B (32 KB) + scales in
// shared memory; the accumulator (256 TMEM columns) is released as soon as the
// eight epilogue warps have moved it into registers, so the stores of tile i
// overlap the MMAs of tile i + 1, and the producer keeps loading across tiles.
constexpr int BNP = 256;
constexpr int kStagesP = 4;
constexpr int kThreadsP = 320;                 // producer, MMA, 8 epilogue warps
constexpr int kTmemColsP = 512;

template <int KIND>
struct KindP {
    // 4-scale chunks per stage: a stage is 128 bytes of every row, K = 256
    // E2M1 elements (MXF4: 8 blocks of 32, NVF4: 16 of 16) or K = 128 FP6
    // elements in byte containers (MXF6: 4 blocks of 32)
    // (an E2M1 operand of kind::mxf8f6f4 also takes one byte per element in
    // shared memory: the TMA expands each 8-byte group of 16 packed codes to
    // 16 bytes, the upper 8 left zero)
    static constexpr int kChunks = KIND == KIND_MXF4 ? 2 : KIND == KIND_MXF6 ? 1 : 4;
    static constexpr int kSfaBytes = kChunks * 512;                  // 128 rows of A
    static constexpr int kSfbBytes = 2 * kChunks * 512;              // 256 rows of B
    static constexpr int kABytes = BM * 128, kBBytes = BNP * 128;
    static constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
    static constexpr int kSfCols = kChunks * 4 + 2 * kChunks * 4;    // TMEM columns per stage
};

template <int KIND>
__device__ __forceinline__ uint32_t idesc_p(uint32_t ab_fmt)
{
    // A, B formats: E2M1 (kind::mxf4 / mxf4nvf4), or E2M3 = 3 / E3M2 = 4 (kind::mxf8f6f4)
    uint32_t d = KIND == KIND_MXF6 ? ab_fmt : (1u << 7) | (1u << 10);
    if (KIND != KIND_NVF4) d |= 1u << 23;        // UE8M0 scales
    d |= (uint32_t)(BNP >> 3) << 17;
    d |= (uint32_t)(BM >> 4) << 24;
    return d;
}

template <int KIND, int EPI>
__global__ void __launch_bounds__(kThreadsP, 1)
    k_gemm_p(const GParams p, const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB)
{
    using KT = KindP<KIND>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *sA = smem;
    uint8_t *sB = sA + kStagesP * KT::kABytes;
    uint8_t *sSFA = sB + kStagesP * KT::kBBytes;
    uint8_t *sSFB = sSFA + kStagesP * KT::kSfaBytes;
    uint64_t *full = reinterpret_cast<uint64_t *>(sSFB + kStagesP * KT::kSfbBytes);
    uint64_t *empty = full + kStagesP;
    uint64_t *accf = empty + kStagesP;            // accumulator full (MMA -> epilogue)
    uint64_t *acce = accf + 1;                    // accumulator free (epilogue -> MMA)
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(acce + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntn = p.N / BNP, ntm = p.M / BM;
    const int ntiles = ntn * ntm;
    const int ktiles = p.K / (KIND == KIND_MXF6 ? 128 : 256);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStagesP; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accf, 1);
        mbar_init(acce, 8);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(saddr(tmem_holder)), "r"(kTmemColsP));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_holder;
    const uint32_t tsf = tbase + BNP;

    if (warp == 0) {
        if (lane == 0) {
            const int sf_chunks_row = (p.K / (KIND == KIND_NVF4 ? 16 : 32)) / 4;
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
                const int m0 = (tile / ntn) * BM, n0 = (tile % ntn) * BNP;
                for (int kt = 0; kt < ktiles; ++kt, ++it) {
                    const int s = it % kStagesP;
                    if (it >= (uint32_t)kStagesP && !mbar_wait(&empty[s], ((it / kStagesP) - 1) & 1, 11)) { ok = false; break; }
                    mbar_expect_tx(&full[s], KIND == KIND_MXF6 ? p.stage_tx : (uint32_t)KT::kStageBytes);
                    tma_load_2d(sA + s * KT::kABytes, &tmA, &full[s], kt * 128, m0);
                    tma_load_2d(sB + s * KT::kBBytes, &tmB, &full[s], kt * 128, n0);
                    const size_t ca = ((size_t)(m0 / 128) * sf_chunks_row + (size_t)kt * KT::kChunks) * 512;
                    const size_t cb0 = ((size_t)(n0 / 128) * sf_chunks_row + (size_t)kt * KT::kChunks) * 512;
                    const size_t cb1 = ((size_t)(n0 / 128 + 1) * sf_chunks_row + (size_t)kt * KT::kChunks) * 512;
                    bulk_load(sSFA + s * KT::kSfaBytes, p.sfa + ca, KT::kSfaBytes, &full[s]);
                    bulk_load(sSFB + s * KT::kSfbBytes, p.sfb + cb0, KT::kChunks * 512, &full[s]);
                    bulk_load(sSFB + s * KT::kSfbBytes + KT::kChunks * 512, p.sfb + cb1, KT::kChunks * 512, &full[s]);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc0 = idesc_p<KIND>(p.ab_fmt);
            uint32_t it = 0, tcount = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++tcount) {
                // wait until the epilogue has drained the previous tile's accumulator
                if (tcount > 0 && !mbar_wait(acce, (tcount - 1) & 1, 12)) { ok = false; break; }
                tc_fence_after();
                for (int kt = 0; kt < ktiles; ++kt, ++it) {
                    const int s = it % kStagesP;
                    if (!mbar_wait(&full[s], (it / kStagesP) & 1, 13)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sfa_t = tsf + s * KT::kSfCols;
                    const uint32_t sfb_t = sfa_t + KT::kChunks * 4;
#pragma unroll
                    for (int c = 0; c < KT::kChunks; ++c) {
                        asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;"
                                     ::"r"(sfa_t + 4 * c), "l"(desc_sf(saddr(sSFA + s * KT::kSfaBytes + c * 512))));
                        // B rows 0..127 -> columns 8c..8c+3, rows 128..255 -> 8c+4..8c+7
                        asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;"
                                     ::"r"(sfb_t + 8 * c), "l"(desc_sf(saddr(sSFB + s * KT::kSfbBytes + c * 512))));
                        asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;"
                                     ::"r"(sfb_t + 8 * c + 4),
                                       "l"(desc_sf(saddr(sSFB + s * KT::kSfbBytes + KT::kChunks * 512 + c * 512))));
                    }
                    const uint32_t a0 = saddr(sA + s * KT::kABytes), b0 = saddr(sB + s * KT::kBBytes);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        uint32_t idesc = idesc0, sfa, sfb;
                        if constexpr (KIND == KIND_MXF4) {
                            // K = 64: two 32-blocks, scale bytes 0-1 or 2-3 of a chunk column
                            const uint32_t id = (k & 1) * 2;
                            idesc |= (id << 29) | (id << 4);
                            sfa = sfa_t + 4 * (k >> 1);
                            sfb = sfb_t + 8 * (k >> 1);
                        } else if constexpr (KIND == KIND_MXF6) {
                            // K = 32: one 32-block, scale byte k of the stage's chunk column
                            const uint32_t id = (uint32_t)k;
                            idesc |= (id << 29) | (id << 4);
                            sfa = sfa_t;
                            sfb = sfb_t;
                        } else {
                            sfa = sfa_t + 4 * k;
                            sfb = sfb_t + 8 * k;
                        }
                        mma<KIND>(tbase, desc_sw128(a0 + 32 * k), desc_sw128(b0 + 32 * k), idesc, sfa, sfb,
                                  (kt > 0 || k > 0) ? 1u : 0u);
                    }
                    tc_commit(&empty[s]);
                }
                if (ok) tc_commit(accf);
            }
        }
        __syncwarp();
    } else {
        // eight epilogue warps: quadrant q = warp % 4 (TMEM lanes), column half h
        const int q = warp & 3, h = (warp - 2) >> 2;
        float scale = 1.0f;
        if (p.tsA) scale = __fmul_rn(scale, *p.tsA);
        if (p.tsB) scale = __fmul_rn(scale, *p.tsB);
        uint32_t tcount = 0;
        for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++tcount) {
            const int m0 = (tile / ntn) * BM, n0 = (tile % ntn) * BNP;
            if (!mbar_wait(accf, tcount & 1, 14)) break;
            tc_fence_after();
            float v[128];
#pragma unroll
            for (int ch = 0; ch < 4; ++ch)
                tmem_ld32(tbase + ((uint32_t)(32 * q) << 16) + h * 128 + ch * 32, v + 32 * ch);
            // the accumulator is in registers: hand it back to the MMA warp
            tc_fence_before();
            __syncwarp();
            if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(saddr(acce)) : "memory");
            const int row = m0 + 32 * q + lane;
            const int col = n0 + h * 128;
            if constexpr (EPI == EPI_BF16) {
                __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(p.C) + (size_t)row * p.N + col;
#pragma unroll
                for (int i = 0; i < 128; i += 8) {
                    uint32_t w[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        __nv_bfloat162 t2 = __floats2bfloat162_rn(v[i + 2 * j] * scale, v[i + 2 * j + 1] * scale);
                        w[j] = *reinterpret_cast<uint32_t *>(&t2);
                    }
                    *reinterpret_cast<uint4 *>(dst + i) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            } else {
                float *dst = static_cast<float *>(p.C) + (size_t)row * p.N + col;
#pragma unroll
                for (int i = 0; i < 128; i += 4)
                    *reinterpret_cast<float4 *>(dst + i) =
                        make_float4(v[i] * scale, v[i + 1] * scale, v[i + 2] * scale, v[i + 3] * scale);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tbase), "r"(kTmemColsP));
    }
}

// ---------------------------------------------------------------------------
// Fused QSNR(AB) ("Unveiling the Potential of Quantization with MXFP4", Sec.3
// Eq. (2)): persistent, one CTA per SM, 128 x BNT output tiles.  For every
// tile the MMA warp forms C_q = A^Q (B^Q)^T with the block-scaled kind into
// the accumulator (BNT TMEM columns), the eight epilogue warps move it into
// registers (BNT / 2 floats a thread, times the tensor scales) and hand the
// columns back, the MMA warp then forms C_ref = A B^T with kind::f16 on the
// bf16 operands into the same columns, and the epilogue reduces
// sum C_ref^2 and sum (C_ref - C_q)^2 against the registers.  C is never
// written.  The producer streams both phases through one shared-memory ring:
// a block-scaled stage is 128 bytes of every row (plus the scale chunks), a
// bf16 stage 64 elements (also 128 bytes) of every row.  Tiles are walked in
// groups of kGroupM tile rows so that the A and B slices a wave of CTAs reads
// stay in L2 (the bf16 operands are four times the FP4 ones).
constexpr int kGroupM = 16;

template <int KIND, int BNT>
struct KindQ {
    static constexpr int kChunks = KindP<KIND>::kChunks;          // scale chunks per stage and 128 rows
    static constexpr int kBHalves = BNT / 128;                    // 128-row groups of B
    static constexpr int kSfaBytes = kChunks * 512;
    static constexpr int kSfbBytes = kBHalves * kChunks * 512;
    static constexpr int kABytes = BM * 128, kBBytes = BNT * 128;
    static constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
    static constexpr int kSfCols = kChunks * 4 + kBHalves * kChunks * 4;
    static constexpr int kSmem = 1024 + kStagesP * kStageBytes + 256;
};

// tile index -> (tile row, tile column): groups of kGroupM tile rows, walked
// column by column inside a group
__device__ __forceinline__ void qsnr_tile(int tile, int ntm, int ntn, int &mt, int &nt)
{
    const int per = kGroupM * ntn;
    const int g = tile / per, r = tile - g * per;
    const int gm = min(kGroupM, ntm - g * kGroupM);
    mt = g * kGroupM + r % gm;
    nt = r / gm;
}

template <int KIND, int BNT>
__global__ void __launch_bounds__(kThreadsP, 1)
    k_gemm_qsnr_f(const GParams p, const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmAr, const __grid_constant__ CUtensorMap tmBr)
{
    using KT = KindQ<KIND, BNT>;
    constexpr int HALF = BNT / 2;                 // columns per epilogue warp
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *sA = smem;
    uint8_t *sB = sA + kStagesP * KT::kABytes;
    uint8_t *sSFA = sB + kStagesP * KT::kBBytes;
    uint8_t *sSFB = sSFA + kStagesP * KT::kSfaBytes;
    uint64_t *full = reinterpret_cast<uint64_t *>(sSFB + kStagesP * KT::kSfbBytes);
    uint64_t *empty = full + kStagesP;
    uint64_t *accf = empty + kStagesP;            // accumulator full (MMA -> epilogue), once per product
    uint64_t *acce = accf + 1;                    // accumulator read out (epilogue -> MMA)
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(acce + 1);
    double *red = reinterpret_cast<double *>(tmem_holder + 4);      // 8 warps x 2 sums

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntn = p.N / BNT, ntm = p.M / BM;
    const int ntiles = ntn * ntm;
    const int kq = p.K / (KIND == KIND_MXF6 ? 128 : 256);      // block-scaled stages per tile
    const int kr = p.K / 64;                                     // bf16 stages per tile

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStagesP; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accf, 1);
        mbar_init(acce, 8);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(saddr(tmem_holder)), "r"(kTmemColsP));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_holder;
    const uint32_t tsf = tbase + BNT;

    if (warp == 0) {
        if (lane == 0) {
            const int sf_chunks_row = (p.K / (KIND == KIND_NVF4 ? 16 : 32)) / 4;
            const uint32_t tx_q = KIND == KIND_MXF6 ? p.stage_tx : (uint32_t)KT::kStageBytes;
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
                int mt, nt;
                qsnr_tile(tile, ntm, ntn, mt, nt);
                const int m0 = mt * BM, n0 = nt * BNT;
                for (int kt = 0; kt < kq + kr; ++kt, ++it) {
                    const int s = it % kStagesP;
                    if (it >= (uint32_t)kStagesP && !mbar_wait(&empty[s], ((it / kStagesP) - 1) & 1, 15)) { ok = false; break; }
                    if (kt < kq) {
                        mbar_expect_tx(&full[s], tx_q);
                        tma_load_2d(sA + s * KT::kABytes, &tmA, &full[s], kt * 128, m0);
                        tma_load_2d(sB + s * KT::kBBytes, &tmB, &full[s], kt * 128, n0);
                        const size_t ca = ((size_t)(m0 / 128) * sf_chunks_row + (size_t)kt * KT::kChunks) * 512;
                        bulk_load(sSFA + s * KT::kSfaBytes, p.sfa + ca, KT::kSfaBytes, &full[s]);
#pragma unroll
                        for (int hb = 0; hb < KT::kBHalves; ++hb) {
                            const size_t cb = ((size_t)(n0 / 128 + hb) * sf_chunks_row + (size_t)kt * KT::kChunks) * 512;
                            bulk_load(sSFB + s * KT::kSfbBytes + hb * KT::kChunks * 512, p.sfb + cb,
                                      KT::kChunks * 512, &full[s]);
                        }
                    } else {
                        const int kx = (kt - kq) * 64;                       // bf16 elements
                        mbar_expect_tx(&full[s], (uint32_t)(KT::kABytes + KT::kBBytes));
                        tma_load_2d(sA + s * KT::kABytes, &tmAr, &full[s], kx, m0);
                        tma_load_2d(sB + s * KT::kBBytes, &tmBr, &full[s], kx, n0);
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            // block-scaled kind (N = BNT) and kind::f16 on bf16 (N = BNT)
            uint32_t idq = KIND == KIND_MXF6 ? p.ab_fmt : (1u << 7) | (1u << 10);
            if (KIND != KIND_NVF4) idq |= 1u << 23;
            idq |= (uint32_t)(BNT >> 3) << 17;
            idq |= (uint32_t)(BM >> 4) << 24;
            const uint32_t idr = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BNT >> 3) << 17) |
                                 ((uint32_t)(BM >> 4) << 24);
            uint32_t it = 0, ph = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
                for (int part = 0; part < 2 && ok; ++part, ++ph) {
                    // the epilogue has read the previous product out of the accumulator
                    if (ph > 0 && !mbar_wait(acce, (ph - 1) & 1, 16)) { ok = false; break; }
                    tc_fence_after();
                    const int k0 = part == 0 ? 0 : kq, k1 = part == 0 ? kq : kq + kr;
                    for (int kt = k0; kt < k1; ++kt, ++it) {
                        const int s = it % kStagesP;
                        if (!mbar_wait(&full[s], (it / kStagesP) & 1, 17)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t a0 = saddr(sA + s * KT::kABytes), b0 = saddr(sB + s * KT::kBBytes);
                        const uint32_t acc0 = kt > k0 ? 1u : 0u;
                        if (part == 1) {
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                mma<KIND_BF16>(tbase, desc_sw128(a0 + 32 * k), desc_sw128(b0 + 32 * k), idr, 0, 0,
                                               (acc0 | (uint32_t)k) ? 1u : 0u);
                        } else {
                            const uint32_t sfa_t = tsf + s * KT::kSfCols;
                            const uint32_t sfb_t = sfa_t + KT::kChunks * 4;
#pragma unroll
                            for (int c = 0; c < KT::kChunks; ++c) {
                                asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;"
                                             ::"r"(sfa_t + 4 * c), "l"(desc_sf(saddr(sSFA + s * KT::kSfaBytes + c * 512))));
#pragma unroll
                                for (int hb = 0; hb < KT::kBHalves; ++hb)
                                    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;"
                                                 ::"r"(sfb_t + 4 * KT::kBHalves * c + 4 * hb),
                                                   "l"(desc_sf(saddr(sSFB + s * KT::kSfbBytes + hb * KT::kChunks * 512 + c * 512))));
                            }
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                uint32_t idesc = idq, sfa, sfb;
                                if constexpr (KIND == KIND_MXF4) {
                                    const uint32_t id = (k & 1) * 2;
                                    idesc |= (id << 29) | (id << 4);
                                    sfa = sfa_t + 4 * (k >> 1);
                                    sfb = sfb_t + 4 * KT::kBHalves * (k >> 1);
                                } else if constexpr (KIND == KIND_MXF6) {
                                    const uint32_t id = (uint32_t)k;
                                    idesc |= (id << 29) | (id << 4);
                                    sfa = sfa_t;
                                    sfb = sfb_t;
                                } else {
                                    sfa = sfa_t + 4 * k;
                                    sfb = sfb_t + 4 * KT::kBHalves * k;
                                }
                                mma<KIND>(tbase, desc_sw128(a0 + 32 * k), desc_sw128(b0 + 32 * k), idesc, sfa, sfb,
                                          (acc0 | (uint32_t)k) ? 1u : 0u);
                            }
                        }
                        tc_commit(&empty[s]);
                    }
                    if (ok) tc_commit(accf);
                }
            }
        }
        __syncwarp();
    } else {
        // eight epilogue warps: TMEM lane quadrant q = warp % 4, column half h
        const int q = warp & 3, h = (warp - 2) >> 2;
        float scale = 1.0f;
        if (p.tsA) scale = __fmul_rn(scale, *p.tsA);
        if (p.tsB) scale = __fmul_rn(scale, *p.tsB);
        const uint32_t tcol = tbase + ((uint32_t)(32 * q) << 16) + h * HALF;
        double s_ref = 0.0, s_err = 0.0;
        uint32_t ph = 0;
        for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
            // C_q of this thread's row and column half, into registers
            if (!mbar_wait(accf, ph & 1, 18)) break;
            tc_fence_after();
            float cq[HALF];
#pragma unroll
            for (int ch = 0; ch < HALF / 32; ++ch) tmem_ld32(tcol + ch * 32, cq + 32 * ch);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(saddr(acce)) : "memory");
            ++ph;
            // C_ref, 32 columns at a time, against the registers
            if (!mbar_wait(accf, ph & 1, 19)) break;
            tc_fence_after();
#pragma unroll
            for (int ch = 0; ch < HALF / 32; ++ch) {
                float v[32];
                tmem_ld32(tcol + ch * 32, v);
                if (ch == HALF / 32 - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(saddr(acce)) : "memory");
                }
                // 32 terms per chunk in binary32 (two chains), then binary64
                float r0 = 0.f, r1 = 0.f, e0 = 0.f, e1 = 0.f;
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    const float d0 = __fmaf_rn(-cq[32 * ch + i], scale, v[i]);
                    const float d1 = __fmaf_rn(-cq[32 * ch + i + 1], scale, v[i + 1]);
                    r0 = __fmaf_rn(v[i], v[i], r0);
                    r1 = __fmaf_rn(v[i + 1], v[i + 1], r1);
                    e0 = __fmaf_rn(d0, d0, e0);
                    e1 = __fmaf_rn(d1, d1, e1);
                }
                s_ref += (double)r0 + (double)r1;
                s_err += (double)e0 + (double)e1;
            }
            ++ph;
        }
        for (int o = 16; o > 0; o >>= 1) {
            s_ref += __shfl_down_sync(0xffffffffu, s_ref, o);
            s_err += __shfl_down_sync(0xffffffffu, s_err, o);
        }
        if (lane == 0) {
            red[2 * (warp - 2)] = s_ref;
            red[2 * (warp - 2) + 1] = s_err;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) {
        double a = 0.0, b = 0.0;
        for (int w = 0; w < 8; ++w) { a += red[2 * w]; b += red[2 * w + 1]; }
        p.partials[2 * blockIdx.x] = a;
        p.partials[2 * blockIdx.x + 1] = b;
    }
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tbase), "r"(kTmemColsP));
    }
}

// ---------------------------------------------------------------------------
// Tensor-core ceiling probe: every CTA (one per SM) issues `iters` stages of
// four 128 x 256 x K MMAs of a kind on operands resident in its shared memory
// (all-zero codes, unit scales), accumulating into tensor memory, with no
// global traffic; with `sf_copies` each stage first copies its scale chunks
// into tensor memory as the GEMM's stages do.  The launch time over the
// flops gives the kind's tensor throughput on this device.  Waits bounded.
template <int KIND>
__global__ void __launch_bounds__(128, 1) k_tc_peak(int64_t iters, int sf_copies)
{
    using KT = KindP<KIND>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *sA = smem, *sB = sA + KT::kABytes, *sSFA = sB + KT::kBBytes, *sSFB = sSFA + KT::kSfaBytes;
    uint64_t *done = reinterpret_cast<uint64_t *>(sSFB + KT::kSfbBytes);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(done + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // zero codes; unit scales (E8M0 127, UE4M3 0x38)
    const uint32_t one = KIND == KIND_NVF4 ? 0x38383838u : 0x7f7f7f7fu;
    for (int i = threadIdx.x; i < (KT::kABytes + KT::kBBytes) / 4; i += blockDim.x)
        reinterpret_cast<uint32_t *>(sA)[i] = 0u;
    for (int i = threadIdx.x; i < (KT::kSfaBytes + KT::kSfbBytes) / 4; i += blockDim.x)
        reinterpret_cast<uint32_t *>(sSFA)[i] = one;
    if (threadIdx.x == 0) {
        mbar_init(done, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(saddr(tmem_holder)), "r"(kTmemColsP));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_holder, tsf = tbase + BNP;
    if (warp == 0 && lane == 0) {
        const uint32_t idesc0 = idesc_p<KIND>((3u << 7) | (3u << 10));
        const uint32_t a0 = saddr(sA), b0 = saddr(sB);
        for (int64_t it = 0; it < iters; ++it) {
            // sf_copies 2: the copies rotate over four slots of scale columns,
            // as the GEMM's stages do; 1: one slot
            const uint32_t sfa_t = tsf + (sf_copies == 2 ? (uint32_t)(it & 3) * KT::kSfCols : 0u);
            if (sf_copies || it == 0) {
#pragma unroll
                for (int c = 0; c < KT::kChunks; ++c) {
                    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;"
                                 ::"r"(sfa_t + 4 * c), "l"(desc_sf(saddr(sSFA + c * 512))));
                    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;"
                                 ::"r"(sfa_t + KT::kChunks * 4 + 8 * c), "l"(desc_sf(saddr(sSFB + c * 512))));
                    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;"
                                 ::"r"(sfa_t + KT::kChunks * 4 + 8 * c + 4),
                                   "l"(desc_sf(saddr(sSFB + KT::kChunks * 512 + c * 512))));
                }
            }
            const uint32_t sfb_t = sfa_t + KT::kChunks * 4;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                uint32_t idesc = idesc0, sfa, sfb;
                if constexpr (KIND == KIND_MXF4) {
                    const uint32_t id = (k & 1) * 2;
                    idesc |= (id << 29) | (id << 4);
                    sfa = sfa_t + 4 * (k >> 1);
                    sfb = sfb_t + 8 * (k >> 1);
                } else if constexpr (KIND == KIND_MXF6) {
                    const uint32_t id = (uint32_t)k;
                    idesc |= (id << 29) | (id << 4);
                    sfa = sfa_t;
                    sfb = sfb_t;
                } else {
                    sfa = sfa_t + 4 * k;
                    sfb = sfb_t + 8 * k;
                }
                mma<KIND>(tbase, desc_sw128(a0 + 32 * k), desc_sw128(b0 + 32 * k), idesc, sfa, sfb,
                          (it > 0 || k > 0) ? 1u : 0u);
            }
        }
        tc_commit(done);
        mbar_wait(done, 0, 20);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tbase), "r"(kTmemColsP));
    }
}

template <int KIND>
int launch_tc_peak(int64_t iters, int sf_copies, cudaStream_t st)
{
    using KT = KindP<KIND>;
    const int smem = 1024 + KT::kABytes + KT::kBBytes + KT::kSfaBytes + KT::kSfbBytes + 64;
    auto k = k_tc_peak<KIND>;
    static bool attr = false;
    if (!attr) {
        if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return MX_ERR_CUDA;
        attr = true;
    }
    k<<<mxk::device_sm_count(), 128, smem, st>>>(iters, sf_copies);
    return cudaGetLastError() == cudaSuccess ? MX_OK : MX_ERR_CUDA;
}

// Sum the per-CTA records in a fixed order: [sum C_ref^2, sum err^2, QSNR dB].
__global__ void k_gemm_qsnr_finalize(const double *partials, int n, double *out)
{
    __shared__ double sh[256][2];
    double a = 0.0, b = 0.0;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        a += partials[2 * i];
        b += partials[2 * i + 1];
    }
    sh[threadIdx.x][0] = a;
    sh[threadIdx.x][1] = b;
    __syncthreads();
    for (int w = blockDim.x / 2; w > 0; w >>= 1) {
        if ((int)threadIdx.x < w) {
            sh[threadIdx.x][0] += sh[threadIdx.x + w][0];
            sh[threadIdx.x][1] += sh[threadIdx.x + w][1];
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        const double r = sh[0][0], e = sh[0][1];
        out[0] = r;
        out[1] = e;
        out[2] = (r == 0.0) ? __longlong_as_double(0x7ff8000000000000ll)
               : (e == 0.0) ? __longlong_as_double(0x7ff0000000000000ll)
                            : 10.0 * log10(r / e);
    }
}

// ------------------------------------------------------------------- host --
typedef CUresult (*EncodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                CUtensorMapFloatOOBfill);

EncodeTiled encoder()
{
    static EncodeTiled fn = nullptr;
    if (!fn) {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<EncodeTiled>(f);
    }
    return fn;
}

// rows x row_bytes operand, box of 128 rows x 128 bytes, 128-byte swizzle
// elem_bits: 16 (bf16), 4 (packed E2M1 bytes for kind::mxf4 / mxf4nvf4), or -4 / -6
// (packed E2M1 / dense FP6, widened to one byte per element for kind::mxf8f6f4)
bool make_map(CUtensorMap *m, const void *base, int rows, int K, int elem_bits, unsigned box_rows = 128)
{
    EncodeTiled enc = encoder();
    if (!enc) return false;
    if (elem_bits == -4 || elem_bits == -6) {
        // packed sub-byte codes read for kind::mxf8f6f4: a box of 128 elements
        // (64 bytes of E2M1, 96 of FP6) lands as 128 bytes in shared memory,
        // every group of 16 codes widened to 16 bytes (8 / 4 zero bytes added)
        const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
        const cuuint64_t strides[1] = {(cuuint64_t)K * (elem_bits == -4 ? 4 : 6) / 8};
        const cuuint32_t box[2] = {128u, box_rows};
        const cuuint32_t estr[2] = {1, 1};
        return enc(m, elem_bits == -4 ? CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B : CU_TENSOR_MAP_DATA_TYPE_16U6_ALIGN16B,
                   2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    }
    const bool bf16 = elem_bits == 16;
    const cuuint64_t row_bytes = (cuuint64_t)K * elem_bits / 8;
    const cuuint64_t inner = bf16 ? (cuuint64_t)K : row_bytes;
    const cuuint64_t dims[2] = {inner, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {bf16 ? 64u : 128u, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
               const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int KIND, int EPI>
int launch(const GParams &p, const void *A, const void *B, cudaStream_t st)
{
    CUtensorMap ta, tb;
    const int bits = KIND == KIND_BF16 ? 16 : 4;
    if (!make_map(&ta, A, p.M, p.K, bits) || !make_map(&tb, B, p.N, p.K, bits)) return MX_ERR_CUDA;
    using KT = Kind<KIND>;
    const int smem = 1024 + kStages * KT::kStageBytes + 256;
    auto k = k_gemm<KIND, EPI>;
    static bool attr = false;
    if (!attr) {
        if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return MX_ERR_CUDA;
        attr = true;
    }
    dim3 grid(p.N / BN, p.M / BM);
    k<<<grid, kThreads, smem, st>>>(p, ta, tb);
    return cudaGetLastError() == cudaSuccess ? MX_OK : MX_ERR_CUDA;
}


template <int KIND, int EPI>
int launch_p(const GParams &p, const void *A, const void *B, cudaStream_t st)
{
    CUtensorMap ta, tb;
    using KT = KindP<KIND>;
    int abits = 4, bbits = 4;
    GParams q = p;
    if (KIND == KIND_MXF6) {
        // per operand: dense FP6 (6 bits per code) or packed E2M1, both widened
        // to one byte per element by the TMA; the transaction counts the
        // packed bytes read
        const bool a4 = ((p.ab_fmt >> 7) & 7u) == kFmtE2M1, b4 = ((p.ab_fmt >> 10) & 7u) == kFmtE2M1;
        abits = a4 ? -4 : -6;
        bbits = b4 ? -4 : -6;
        q.stage_tx = (uint32_t)((a4 ? KT::kABytes / 2 : KT::kABytes / 4 * 3) +
                                (b4 ? KT::kBBytes / 2 : KT::kBBytes / 4 * 3) + KT::kSfaBytes + KT::kSfbBytes);
    }
    if (!make_map(&ta, A, p.M, p.K, abits, 128) || !make_map(&tb, B, p.N, p.K, bbits, 256)) return MX_ERR_CUDA;
    const int smem = 1024 + kStagesP * KT::kStageBytes + 256;
    auto k = k_gemm_p<KIND, EPI>;
    static bool attr = false;
    if (!attr) {
        if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return MX_ERR_CUDA;
        attr = true;
    }
    const int tiles = (p.M / BM) * (p.N / BNP);
    int grid = mxk::device_sm_count();
    if (grid > tiles) grid = tiles;
    k<<<grid, kThreadsP, smem, st>>>(q, ta, tb);
    return cudaGetLastError() == cudaSuccess ? MX_OK : MX_ERR_CUDA;
}

constexpr int kMaxQsnrCtas = 1024;     // per-CTA records of the fused QSNR(AB) kernel

template <int KIND, int BNT>
int launch_qsnr_f(const GParams &p, const void *Aq, const void *Bq, const void *A, const void *B,
                  cudaStream_t st)
{
    using KT = KindQ<KIND, BNT>;
    CUtensorMap ta, tb, tar, tbr;
    GParams q = p;
    int abits = 4, bbits = 4;
    if (KIND == KIND_MXF6) {
        const bool a4 = ((p.ab_fmt >> 7) & 7u) == kFmtE2M1, b4 = ((p.ab_fmt >> 10) & 7u) == kFmtE2M1;
        abits = a4 ? -4 : -6;
        bbits = b4 ? -4 : -6;
        q.stage_tx = (uint32_t)((a4 ? KT::kABytes / 2 : KT::kABytes / 4 * 3) +
                                (b4 ? KT::kBBytes / 2 : KT::kBBytes / 4 * 3) + KT::kSfaBytes + KT::kSfbBytes);
    }
    if (!make_map(&ta, Aq, p.M, p.K, abits, 128) || !make_map(&tb, Bq, p.N, p.K, bbits, BNT) ||
        !make_map(&tar, A, p.M, p.K, 16, 128) || !make_map(&tbr, B, p.N, p.K, 16, BNT))
        return MX_ERR_CUDA;
    auto k = k_gemm_qsnr_f<KIND, BNT>;
    static bool attr = false;
    if (!attr) {
        if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, KT::kSmem) != cudaSuccess)
            return MX_ERR_CUDA;
        attr = true;
    }
    const int tiles = (p.M / BM) * (p.N / BNT);
    int grid = mxk::device_sm_count();
    if (grid > tiles) grid = tiles;
    if (grid > kMaxQsnrCtas) grid = kMaxQsnrCtas;
    k<<<grid, kThreadsP, KT::kSmem, st>>>(q, ta, tb, tar, tbr);
    if (cudaGetLastError() != cudaSuccess) return MX_ERR_CUDA;
    k_gemm_qsnr_finalize<<<1, 256, 0, st>>>(p.partials, grid, p.stats);
    return cudaGetLastError() == cudaSuccess ? MX_OK : MX_ERR_CUDA;
}

template <int KIND>
int launch_qsnr_kind(const GParams &p, const void *Aq, const void *Bq, const void *A, const void *B,
                     cudaStream_t st)
{
    return p.N % BNP == 0 ? launch_qsnr_f<KIND, BNP>(p, Aq, Bq, A, B, st)
                          : launch_qsnr_f<KIND, BN>(p, Aq, Bq, A, B, st);
}

// MXFP4 (E2M1 + E8M0, block 32) or NVFP4 (E2M1 + UE4M3, block 16) operands
// quantized along K in the tcgen05 scale layout; returns the kind or -1.
int fp4_kind(const mx_config *a, const mx_config *b)
{
    if (!a || !b) return -1;
    // rotated operands are accepted when both carry the same rotation along
    // K: (A H)(B H)^T = A B^T for the orthonormal block Hadamard H
    auto layout = [](const mx_config *c) {
        return c->axis == MX_AXIS_ROW && c->sf_layout == 1 && !c->asymmetric && !c->macro_block;
    };
    if (!layout(a) || !layout(b) || a->hadamard != b->hadamard) return -1;
    auto fp6 = [](const mx_config *c) { return c->elem == MX_E2M3 || c->elem == MX_E3M2; };
    if (fp6(a) || fp6(b)) {
        // kind::mxf8f6f4: FP6 x FP6, or FP6 with an E2M1 operand (E8M0, blocks of 32)
        const bool elems = (fp6(a) || a->elem == MX_E2M1) && (fp6(b) || b->elem == MX_E2M1);
        if (elems && a->scale_fmt == MX_SCALE_E8M0 && b->scale_fmt == MX_SCALE_E8M0 && a->block == 32 &&
            b->block == 32)
            return KIND_MXF6;
        return -1;
    }
    if (a->elem != MX_E2M1 || b->elem != MX_E2M1) return -1;
    if (a->scale_fmt == MX_SCALE_E8M0 && b->scale_fmt == MX_SCALE_E8M0 && a->block == 32 && b->block == 32)
        return KIND_MXF4;
    // (UE4M3 scales chosen by the nearest or the MSE rule alike)
    auto near = [](const mx_config *c) { return c->rule == MX_RULE_NEAREST || c->rule == MX_RULE_MSE; };
    if (a->scale_fmt == MX_SCALE_UE4M3 && b->scale_fmt == MX_SCALE_UE4M3 && near(a) && near(b) &&
        a->block == 16 && b->block == 16)
        return KIND_NVF4;
    return -1;
}

// kind::mxf8f6f4 operand formats (instruction descriptor bits 7-9 and 10-12):
// E2M3 = 3, E3M2 = 4, E2M1 = 5
uint32_t fp6_formats(const mx_config *a, const mx_config *b)
{
    auto f = [](const mx_config *c) { return c->elem == MX_E2M3 ? 3u : c->elem == MX_E3M2 ? 4u : kFmtE2M1; };
    return (f(a) << 7) | (f(b) << 10);
}

bool shapes_ok(int64_t M, int64_t N, int64_t K)
{
    return M > 0 && N > 0 && K > 0 && M % BM == 0 && N % BN == 0 && K % 256 == 0 && M < (1 << 30) &&
           N < (1 << 30) && K < (1 << 30);
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace mxg

using namespace mxg;

extern "C" {

int64_t mx_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K)
{
    (void)K;
    if (M <= 0 || N <= 0) return 0;
    // one record of two binary64 sums per CTA of the fused kernel
    return 256 + (int64_t)kMaxQsnrCtas * 16;
}

int mx_gemm(const mx_config *ca, const mx_config *cb, const void *Aq, const uint8_t *Asf,
            const void *Bq, const uint8_t *Bsf, const float *tsA, const float *tsB, int64_t M,
            int64_t N, int64_t K, void *C, int32_t c_dtype, void *stream)
{
    const int kind = fp4_kind(ca, cb);
    if (kind < 0) return MX_ERR_UNSUPPORTED;
    if (!shapes_ok(M, N, K)) return MX_ERR_INVALID;
    if (!Aq || !Bq || !Asf || !Bsf || !C) return MX_ERR_INVALID;
    if (c_dtype != MX_DT_BF16 && c_dtype != MX_DT_FP32) return MX_ERR_INVALID;
    if (!aligned16(Aq) || !aligned16(Bq) || !aligned16(Asf) || !aligned16(Bsf) || !aligned16(C))
        return MX_ERR_ALIGN;
    GParams p;
    memset(&p, 0, sizeof(p));
    p.M = (int)M;
    p.N = (int)N;
    p.K = (int)K;
    p.sfa = Asf;
    p.sfb = Bsf;
    if (kind == KIND_NVF4) {
        p.tsA = ca->tensor_scale != MX_TS_NONE ? tsA : nullptr;
        p.tsB = cb->tensor_scale != MX_TS_NONE ? tsB : nullptr;
    }
    p.C = C;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (kind == KIND_MXF6) {
        // MXFP6 (and FP6 x E2M1): the persistent 128 x 256 kernel only
        if (N % BNP) return MX_ERR_UNSUPPORTED;
        // the widening TMA types want 32-byte aligned operands
        if (((uintptr_t)Aq & 31u) || ((uintptr_t)Bq & 31u)) return MX_ERR_ALIGN;
        p.ab_fmt = fp6_formats(ca, cb);
        return c_dtype == MX_DT_BF16 ? launch_p<KIND_MXF6, EPI_BF16>(p, Aq, Bq, st)
                                     : launch_p<KIND_MXF6, EPI_F32>(p, Aq, Bq, st);
    }
    if (N % BNP == 0) {
        if (kind == KIND_MXF4)
            return c_dtype == MX_DT_BF16 ? launch_p<KIND_MXF4, EPI_BF16>(p, Aq, Bq, st)
                                         : launch_p<KIND_MXF4, EPI_F32>(p, Aq, Bq, st);
        return c_dtype == MX_DT_BF16 ? launch_p<KIND_NVF4, EPI_BF16>(p, Aq, Bq, st)
                                     : launch_p<KIND_NVF4, EPI_F32>(p, Aq, Bq, st);
    }
    if (kind == KIND_MXF4)
        return c_dtype == MX_DT_BF16 ? launch<KIND_MXF4, EPI_BF16>(p, Aq, Bq, st)
                                     : launch<KIND_MXF4, EPI_F32>(p, Aq, Bq, st);
    return c_dtype == MX_DT_BF16 ? launch<KIND_NVF4, EPI_BF16>(p, Aq, Bq, st)
                                 : launch<KIND_NVF4, EPI_F32>(p, Aq, Bq, st);
}

int mx_gemm_qsnr(const mx_config *ca, const mx_config *cb, const void *A, const void *B, int64_t M,
                 int64_t N, int64_t K, const void *Aq, const uint8_t *Asf, const void *Bq,
                 const uint8_t *Bsf, const float *tsA, const float *tsB, double *stats,
                 void *workspace, int64_t workspace_bytes, void *stream)
{
    const int kind = fp4_kind(ca, cb);
    if (kind < 0) return MX_ERR_UNSUPPORTED;
    if (!shapes_ok(M, N, K)) return MX_ERR_INVALID;
    if (!A || !B || !stats || !Aq || !Bq || !Asf || !Bsf) return MX_ERR_INVALID;
    if (!workspace || workspace_bytes < mx_gemm_workspace_bytes(M, N, K)) return MX_ERR_WORKSPACE;
    if (!aligned16(A) || !aligned16(B) || !aligned16(Aq) || !aligned16(Bq) || !aligned16(Asf) ||
        !aligned16(Bsf) || !aligned16(workspace) || ((uintptr_t)stats & 7u))
        return MX_ERR_ALIGN;
    GParams p;
    memset(&p, 0, sizeof(p));
    p.M = (int)M;
    p.N = (int)N;
    p.K = (int)K;
    p.sfa = Asf;
    p.sfb = Bsf;
    if (kind == KIND_NVF4) {
        p.tsA = ca->tensor_scale != MX_TS_NONE ? tsA : nullptr;
        p.tsB = cb->tensor_scale != MX_TS_NONE ? tsB : nullptr;
    }
    p.partials = reinterpret_cast<double *>(static_cast<uint8_t *>(workspace) + 256);
    p.stats = stats;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // both products of every output tile in one persistent kernel, the sums
    // reduced in its epilogue (C is not written), then the per-CTA records
    // summed in a fixed order
    if (kind == KIND_MXF6) {
        if (N % BNP) return MX_ERR_UNSUPPORTED;
        if (((uintptr_t)Aq & 31u) || ((uintptr_t)Bq & 31u)) return MX_ERR_ALIGN;
        p.ab_fmt = fp6_formats(ca, cb);
        return launch_qsnr_f<KIND_MXF6, BNP>(p, Aq, Bq, A, B, st);
    }
    if (kind == KIND_MXF4) return launch_qsnr_kind<KIND_MXF4>(p, Aq, Bq, A, B, st);
    return launch_qsnr_kind<KIND_NVF4>(p, Aq, Bq, A, B, st);
}

int mx_gemm_qsnr_finalize(double *stats, void *stream)
{
    if (!stats) return MX_ERR_INVALID;
    if ((uintptr_t)stats & 7u) return MX_ERR_ALIGN;
    // one record: the buffer's own two sums, read before the three entries are written
    k_gemm_qsnr_finalize<<<1, 256, 0, static_cast<cudaStream_t>(stream)>>>(stats, 1, stats);
    return cudaGetLastError() == cudaSuccess ? MX_OK : MX_ERR_CUDA;
}

int mx_tensor_peak(int32_t kind, int64_t iters, int32_t sf_copies, double *flops, void *stream)
{
    // at most 2^22 stages: well under a second at any clock (the bounded
    // waits give up after two)
    if (iters <= 0 || iters > (INT64_C(1) << 22) || !flops || (kind < KIND_MXF4 || kind > KIND_MXF6))
        return MX_ERR_INVALID;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // flops of the launch: CTAs x stages x four MMAs of 128 x 256 x K
    const double k_mma = kind == KIND_MXF6 ? 32.0 : 64.0;
    *flops = (double)mxk::device_sm_count() * (double)iters * 4.0 * 2.0 * BM * BNP * k_mma;
    switch (kind) {
    case KIND_MXF4: return launch_tc_peak<KIND_MXF4>(iters, sf_copies, st);
    case KIND_NVF4: return launch_tc_peak<KIND_NVF4>(iters, sf_copies, st);
    default: return launch_tc_peak<KIND_MXF6>(iters, sf_copies, st);
    }
}

int mx_device_status(void *stream, int32_t *status)
{
    if (!status) return MX_ERR_INVALID;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int v = 0;
    if (cudaMemcpyFromSymbolAsync(&v, g_status, sizeof(int), 0, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return MX_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return MX_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbolAsync(g_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st) != cudaSuccess)
        return MX_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return MX_ERR_CUDA;
    int vf = 0, vg = 0;
    if (mxk::take_status_fast(st, &vf) || mxk::take_status_gen(st, &vg)) return MX_ERR_CUDA;
    *status = v ? v : vf ? vf : vg;
    return MX_OK;
}

}  // extern "C"
