// sm_100a E2M1 round-to-nearest-even quantizer fed by TMA ("MXFP4" and
// "NVFP4" of "Unveiling the Potential of Quantization with MXFP4", Sec.2; any
// block size of "Is Finer Better?"; E8M0 floor / ceil / OAS or UE4M3 / UE5M3
// nearest scales, with the fused fidelity sums of Sec.3 Eq. (1)).
//
// Persistent CTAs, one producer warp and eight consumer warps.  The flat
// tensor is viewed as rows of one 32-element chunk (64 bytes of bf16 or 128
// of fp32); the producer streams tiles of 256 chunks into a shared-memory ring
// with 2-D TMA copies (64 / 128-byte swizzle, so that every lane's 16-byte
// reads of its own chunk are bank-conflict free), each consumer lane
// quantizes one chunk per tile: all of HBM's latency is covered by the ring,
// and the registers hold no load buffers.  Every mbarrier wait is bounded.
#include <cuda.h>

#include "quant_common.cuh"

namespace mxk {

namespace {

constexpr int kConsumers = 256;                     // 8 warps, one chunk per lane
constexpr int kFastThreads = kConsumers + 32;       // + producer warp
constexpr uint64_t kWaitNs = 2000000000ull;

__device__ int g_fast_status;

__device__ __forceinline__ uint32_t saddr(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ uint64_t now_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ bool mbar_try(uint64_t *bar, uint32_t phase)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(saddr(bar)), "r"(phase) : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t phase)
{
    if (mbar_try(bar, phase)) return true;
    const uint64_t t0 = now_ns();
    while (!mbar_try(bar, phase))
        if (now_ns() - t0 > kWaitNs) {
            atomicCAS(&g_fast_status, 0, 1);
            return false;
        }
    return true;
}

__device__ __forceinline__ float fmax_nan(float a, float b)
{
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

// number of zero-magnitude E2M1 codes among the 8 nibbles of w: a nibble's
// magnitude m (0..7) plus 7 sets bit 3 exactly when m != 0, with no carry out
__device__ __forceinline__ int zero_codes8(uint32_t w)
{
    return 8 - __popc(((w & 0x77777777u) + 0x77777777u) & 0x88888888u);
}

// Lane t's chunk (row t of the stage) out of the swizzled tile.
__device__ __forceinline__ void read_chunk(const uint8_t *stage, int t, const __nv_bfloat16 *, float y[32])
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
__device__ __forceinline__ void read_chunk(const uint8_t *stage, int t, const float *, float y[32])
{
    const uint8_t *row = stage + 128 * t;
    const int sw = t & 7;                              // 128-byte swizzle
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const float4 u = *reinterpret_cast<const float4 *>(row + 16 * (k ^ sw));
        y[4 * k + 0] = u.x; y[4 * k + 1] = u.y; y[4 * k + 2] = u.z; y[4 * k + 3] = u.w;
    }
}

template <typename InT>
struct FastCfg {
    static constexpr int kChunkBytes = 32 * (int)sizeof(InT);
    static constexpr int kTileBytes = kConsumers * kChunkBytes;      // 16 KB / 32 KB
    static constexpr int kStages = sizeof(InT) == 2 ? 4 : 3;
    static constexpr int kSmem = 1024 + kStages * kTileBytes + 256;
};

// in-lane block Hadamard on the 32-element chunk: groups of n (16 or 32)
__device__ __forceinline__ void hadamard32(float y[32], int n)
{
#pragma unroll
    for (int h = 1; h < 32; h <<= 1) {
        if (h >= n) break;
#pragma unroll
        for (int i = 0; i < 32; i += 2 * h)
#pragma unroll
            for (int j = i; j < i + h; ++j) {
                const float a = y[j], b = y[j + h];
                y[j] = __fadd_rn(a, b);
                y[j + h] = __fsub_rn(a, b);
            }
    }
    const float c = hadamard_scale(n);
#pragma unroll
    for (int j = 0; j < 32; ++j) y[j] = __fmul_rn(y[j], c);
}

// HAD: block rotation before quantization; MBS: 1 x 128 macro scale over the
// 4 lanes of a macro block (consecutive chunks of a tile are consecutive lanes).
template <typename InT, int B, bool STATS, bool HAD, bool MBS>
__global__ void __launch_bounds__(kFastThreads, (HAD || MBS) ? 2 : 3) k_quant_fast(const QParams p, const __grid_constant__ CUtensorMap tm)
{
    using FC = FastCfg<InT>;
    constexpr int NB = B <= 32 ? 32 / B : 1;
    constexpr int G = B <= 32 ? 1 : B / 32;
    constexpr int L = B <= 32 ? B : 32;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *ring = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t *full = reinterpret_cast<uint64_t *>(ring + FC::kStages * FC::kTileBytes);
    uint64_t *empty = full + FC::kStages;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t nch = (uint32_t)(p.rows * p.cols / 32);
    const uint32_t ntiles = (nch + kConsumers - 1) / kConsumers;

    if (threadIdx.x == 0) {
        for (int s = 0; s < FC::kStages; ++s) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(saddr(&full[s])), "r"(1));
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(saddr(&empty[s])), "r"(kConsumers / 32));
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    __syncthreads();

    Acc acc = {0, 0, 0, 0, 0};
    if (warp == kConsumers / 32) {
        // producer: one lane streams the CTA's tiles through the ring
        if (lane == 0) {
            uint32_t i = 0;
            for (uint32_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++i) {
                const uint32_t s = i % FC::kStages;
                if (i >= (uint32_t)FC::kStages && !mbar_wait(&empty[s], ((i / FC::kStages) - 1) & 1)) break;
                asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                             ::"r"(saddr(&full[s])), "r"(FC::kTileBytes) : "memory");
                asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
                             " [%0], [%1, {%3, %4}], [%2];"
                             ::"r"(saddr(ring + s * FC::kTileBytes)), "l"((uint64_t)&tm), "r"(saddr(&full[s])),
                               "r"(0), "r"((int)(tile * kConsumers))
                             : "memory");
            }
        }
        __syncwarp();
    } else {
        const float sT = (p.ts_mode != TS_NONE) ? *p.tensor_scale : 1.0f;
        const bool nearest = p.sd.fmt != S_E8M0 && p.sd.rule == R_NEAREST;
        const uint32_t S = (uint32_t)(p.cols / B);
        const int t = threadIdx.x;
        uint32_t i = 0;
        for (uint32_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++i) {
            const uint32_t s = i % FC::kStages;
            if (!mbar_wait(&full[s], (i / FC::kStages) & 1)) break;
            float ys[MBS ? 32 : 1];         // pre-macro-scale values (statistics reference)
            float y[32];
            read_chunk(ring + s * FC::kTileBytes, t, static_cast<const InT *>(nullptr), y);
            if constexpr (HAD) hadamard32(y, p.had);
            // macro-block scale: y' = y * (1 / S_M), x_hat = (q X) S_M
            float sm = 1.0f;
            if constexpr (MBS) {
                float m = 0.0f;
#pragma unroll
                for (int j = 0; j < 32; ++j) m = fmax_nan(m, fabsf(y[j]));
                int mbad = !(m <= FLT_MAX);
                float mm = grp_max(mbad ? 0.0f : m, 4);
                mbad = grp_or(mbad, 4);
                const uint32_t mcode = macro_code(p.ed, mm, mbad);
                sm = e4m3_value(mcode);
                const float invm = __fdiv_rn(1.0f, sm);
                if ((t & 3) == 0 && tile * kConsumers + t < nch) p.macro[(tile * kConsumers + t) >> 2] = (uint8_t)mcode;
                // keep y for the statistics: scale a copy below
#pragma unroll
                for (int j = 0; j < 32; ++j) ys[j] = y[j];
#pragma unroll
                for (int j = 0; j < 32; ++j) y[j] = __fmul_rn(y[j], invm);
            }

            const uint32_t c = tile * kConsumers + t;
            const bool ok = c < nch;
            uint32_t words[4];
            uint32_t scode[NB];
            // packed two-lane binary32 arithmetic (each lane rounded as a scalar op)
            float2 sx2 = make_float2(0.f, 0.f), se2 = sx2, sb2 = sx2;
            int nzc = 0, ftzc = 0;
#pragma unroll
            for (int k = 0; k < NB; ++k) {
                const int j0 = k * L;
                float a = 0.0f, mabs = FLT_MAX;
#pragma unroll
                for (int j = j0; j < j0 + L; ++j) {
                    a = fmax_nan(a, fabsf(y[j]));
                    if (STATS) mabs = fminf(mabs, fabsf(MBS ? ys[MBS ? j : 0] : y[j]));
                }
                int bad = !(a <= FLT_MAX);
                if (G > 1) {
                    a = grp_max(bad ? 0.0f : a, G);
                    bad = grp_or(bad, G);
                }
                const BlockScale bs = block_scale(p.ed, p.sd, bad ? 0.0f : a, bad, sT);
                scode[k] = bs.code;
                float deqT = bs.nan ? __uint_as_float(0x7fc00000u) : nearest ? __fmul_rn(bs.deq, sT) : bs.deq;
                if (MBS) deqT = __fmul_rn(deqT, sm);       // X * S_M is exact (power of two times E4M3)
                const float2 inv2 = make_float2(bs.inv, bs.inv);
                const float2 nq2 = make_float2(-deqT, -deqT);
                int qz = 0;
#pragma unroll
                for (int w = 0; w < L / 8; ++w) {
                    const int jb = j0 + 8 * w;
                    float s8[8];
#pragma unroll
                    for (int e = 0; e < 8; e += 2) {
                        const float2 v = __fmul2_rn(make_float2(y[jb + e], y[jb + e + 1]), inv2);
                        s8[e] = v.x;
                        s8[e + 1] = v.y;
                    }
                    const uint32_t word = bs.zero ? 0u : cvt_e2m1x8(s8);
                    words[jb >> 3] = word;
                    if (STATS) {
                        float q[8];
                        e2m1x8_values(word, q);
#pragma unroll
                        for (int e = 0; e < 8; e += 2) {
                            const float2 yv = MBS ? make_float2(ys[MBS ? jb + e : 0], ys[MBS ? jb + e + 1 : 0])
                                                  : make_float2(y[jb + e], y[jb + e + 1]);
                            const float2 d = __ffma2_rn(make_float2(q[e], q[e + 1]), nq2, yv);   // y - q deq
                            se2 = __ffma2_rn(d, d, se2);
                            sx2 = __ffma2_rn(yv, yv, sx2);
                            sb2 = __fadd2_rn(sb2, d);
                        }
                        qz += zero_codes8(word);
                    }
                }
                if (STATS) {
                    int xz = 0;
                    if (mabs == 0.0f)                      // rare: count exact zeros
#pragma unroll
                        for (int j = j0; j < j0 + L; ++j) xz += ((MBS ? ys[MBS ? j : 0] : y[j]) == 0.0f);
                    nzc += L - xz;
                    if (!bs.nan) ftzc += qz - xz;
                }
            }
            const float sx = sx2.x + sx2.y, se = se2.x + se2.y, sb = -(sb2.x + sb2.y);
            // every lane of the warp has consumed its chunk: release the stage
            __syncwarp();
            if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(saddr(&empty[s])) : "memory");
            if (ok) {
                reinterpret_cast<uint4 *>(p.codes)[c] = make_uint4(words[0], words[1], words[2], words[3]);
                if (G == 1 || (lane & (G - 1)) == 0) {
                    const uint32_t b0 = (G == 1) ? c * NB : c / G;
                    if (p.sf_gemm) {
                        const uint32_t r = b0 / S, j = b0 - r * S;
#pragma unroll
                        for (int k = 0; k < NB; ++k) p.scales[sf_chunk_index(r, j + k, S)] = (uint8_t)scode[k];
                    } else if (NB == 4) {
                        *reinterpret_cast<uint32_t *>(p.scales + b0) =
                            scode[0] | (scode[NB > 1 ? 1 : 0] << 8) | (scode[NB > 2 ? 2 : 0] << 16) |
                            (scode[NB > 3 ? 3 : 0] << 24);
                    } else if (NB == 2) {
                        *reinterpret_cast<uint16_t *>(p.scales + b0) = (uint16_t)(scode[0] | (scode[NB > 1 ? 1 : 0] << 8));
                    } else {
                        p.scales[b0] = (uint8_t)scode[0];
                    }
                }
                if (STATS) {
                    acc.x2 += (double)sx;
                    acc.e2 += (double)se;
                    acc.e += (double)sb;
                    acc.nz += (double)nzc;
                    acc.ftz += (double)ftzc;
                }
            }
        }
    }
    if (STATS) write_partials(p.partials, acc);
}

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

template <typename InT, int B, bool STATS, bool HAD, bool MBS>
int launch_fast_b(const QParams &p, cudaStream_t st, int *grid_out)
{
    using FC = FastCfg<InT>;
    EncodeTiled enc = encoder();
    if (!enc) return -1;
    const uint64_t nch = (uint64_t)(p.rows * p.cols / 32);
    CUtensorMap tm;
    const cuuint64_t dims[2] = {(cuuint64_t)FC::kChunkBytes, (cuuint64_t)nch};
    const cuuint64_t strides[1] = {(cuuint64_t)FC::kChunkBytes};
    const cuuint32_t box[2] = {(cuuint32_t)FC::kChunkBytes, (cuuint32_t)kConsumers};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(p.x), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE,
            sizeof(InT) == 2 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return -1;
    auto k = k_quant_fast<InT, B, STATS, HAD, MBS>;
    const int occ = cached_occupancy(reinterpret_cast<const void *>(k), kFastThreads, FC::kSmem);
    const uint64_t ntiles = (nch + kConsumers - 1) / kConsumers;
    uint64_t g = (uint64_t)device_sm_count() * occ;
    if (g > ntiles) g = ntiles;
    if (g > (uint64_t)kMaxPartials) g = kMaxPartials;
    if (g < 1) g = 1;
    k<<<(unsigned)g, kFastThreads, FC::kSmem, st>>>(p, tm);
    *grid_out = (int)g;
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

template <typename InT, int B, bool HAD, bool MBS>
int launch_fast_s(const QParams &p, cudaStream_t st, int *grid_out)
{
    return p.partials ? launch_fast_b<InT, B, true, HAD, MBS>(p, st, grid_out)
                      : launch_fast_b<InT, B, false, HAD, MBS>(p, st, grid_out);
}

template <typename InT>
int launch_fast_t(const QParams &p, cudaStream_t st, int *grid_out)
{
    if (p.had || p.mbs) {
        // rotation and / or macro scale: blocks of 16 and 32
        const bool h = p.had != 0, m = p.mbs != 0;
        if (p.block == 32) {
            if (h && m) return launch_fast_s<InT, 32, true, true>(p, st, grid_out);
            if (h) return launch_fast_s<InT, 32, true, false>(p, st, grid_out);
            return launch_fast_s<InT, 32, false, true>(p, st, grid_out);
        }
        if (h && m) return launch_fast_s<InT, 16, true, true>(p, st, grid_out);
        if (h) return launch_fast_s<InT, 16, true, false>(p, st, grid_out);
        return launch_fast_s<InT, 16, false, true>(p, st, grid_out);
    }
    switch (p.block) {
    case 8: return launch_fast_s<InT, 8, false, false>(p, st, grid_out);
    case 16: return launch_fast_s<InT, 16, false, false>(p, st, grid_out);
    case 32: return launch_fast_s<InT, 32, false, false>(p, st, grid_out);
    case 64: return launch_fast_s<InT, 64, false, false>(p, st, grid_out);
    case 128: return launch_fast_s<InT, 128, false, false>(p, st, grid_out);
    case 256: return launch_fast_s<InT, 256, false, false>(p, st, grid_out);
    default: return -1;
    }
}

}  // namespace

// E2M1 / RTNE / symmetric, row axis, no rotated output; rotation and macro
// scale only with blocks of 16 or 32.
int launch_quantize_fast(const QParams &p, int in_fp32, cudaStream_t st, int *grid_out)
{
    return in_fp32 ? launch_fast_t<float>(p, st, grid_out) : launch_fast_t<__nv_bfloat16>(p, st, grid_out);
}

}  // namespace mxk
