// sm_100a block quantizer kernels, row axis (the contiguous dimension).
//
// One pass over HBM per tensor: 128-bit vector loads, optional block
// Hadamard rotation, optional macro-block scale, optional offset, block
// statistic by warp shuffles, shared scale, element rounding, nibble packing
// and the fidelity sums of the dequantized values, all in registers.
//
// Method: "Unveiling the Potential of Quantization with MXFP4" (Sec.2 formats,
// Sec.4 OAS and MBS); "Is Finer Better?" (UE4M3/UE5M3 scales, per-tensor
// scale); "Bridging the Gap ... Microscaling FP4 Quantization" (sec. 2.2-2.3,
// rotation fused with quantization); fmread summary of Yang et al. (rounding
// modes, asymmetric scaling, row / column / 2D blocks).
#include <mutex>
#include <string.h>

#include "quant_common.cuh"

namespace mxk {

// ================================================================ row axis ==
// Thread = 32 consecutive elements of a row (four 16-byte loads in flight for
// bf16, eight for fp32).  A block of B <= 32 elements lies inside the thread
// (32 / B blocks per thread); a block of B > 32 spans B / 32 consecutive lanes.
// A 1 x 128 macro block spans 4 lanes; a 16- or 32-point rotation group lies
// inside the thread.


__device__ __forceinline__ void load32(const __nv_bfloat16 *x, int64_t e, float v[32])
{
    const uint4 *p = reinterpret_cast<const uint4 *>(x + e);
    uint4 u[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) u[i] = __ldg(p + i);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        unpack_bf16x2(u[i].x, v[8 * i + 0], v[8 * i + 1]);
        unpack_bf16x2(u[i].y, v[8 * i + 2], v[8 * i + 3]);
        unpack_bf16x2(u[i].z, v[8 * i + 4], v[8 * i + 5]);
        unpack_bf16x2(u[i].w, v[8 * i + 6], v[8 * i + 7]);
    }
}
__device__ __forceinline__ void load32(const float *x, int64_t e, float v[32])
{
    const float4 *p = reinterpret_cast<const float4 *>(x + e);
    float4 u[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) u[i] = __ldg(p + i);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        v[4 * i + 0] = u[i].x; v[4 * i + 1] = u[i].y; v[4 * i + 2] = u[i].z; v[4 * i + 3] = u[i].w;
    }
}

// in-thread block Hadamard on 32 elements: groups of n (16 or 32)
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

// number of zero-magnitude E2M1 codes among the 8 nibbles of w
__device__ __forceinline__ int zero_codes8(uint32_t w)
{
    const uint32_t m = w & 0x77777777u;
    const uint32_t t = (m | (m >> 1) | (m >> 2)) & 0x11111111u;
    return 8 - __popc(t);
}

template <typename InT, int B, bool FAST>
__global__ void __launch_bounds__(kThreads) k_quant_row(const QParams p)
{
    constexpr int NB = B <= 32 ? 32 / B : 1;    // blocks per thread
    constexpr int G = B <= 32 ? 1 : B / 32;     // lanes per block
    constexpr int L = B <= 32 ? B : 32;         // elements of a block held by the thread
    const InT *x = static_cast<const InT *>(p.x);
    const int lane = threadIdx.x & 31;
    const uint32_t nch = (uint32_t)(p.rows * p.cols / 32);
    const uint32_t gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t nw = (gridDim.x * blockDim.x) >> 5;
    const bool stats = p.partials != nullptr;
    const float sT = launch_tensor_scale(p);
    const bool nearest = p.sd.fmt != S_E8M0 && p.sd.rule == R_NEAREST;
    const uint32_t S = (uint32_t)(p.cols / B);  // scales per row
    Acc acc = {0, 0, 0, 0, 0};

    for (uint32_t c0 = gw * 32; c0 < nch; c0 += nw * 32) {
        const uint32_t c = c0 + lane;
        const bool ok = c < nch;
        const int64_t e0 = (int64_t)c * 32;
        float y[32];
        if (ok) load32(x, e0, y);
        else
#pragma unroll
            for (int j = 0; j < 32; ++j) y[j] = 0.0f;

        if (p.had) hadamard32(y, p.had);
        if (p.rotated && ok)
#pragma unroll
            for (int j = 0; j < 32; j += 4)
                *reinterpret_cast<float4 *>(p.rotated + e0 + j) = make_float4(y[j], y[j + 1], y[j + 2], y[j + 3]);

        // macro-block scale (MBS) over 4 lanes
        float sm = 1.0f, invm = 1.0f;
        if (p.mbs) {
            float m = 0.0f;
#pragma unroll
            for (int j = 0; j < 32; ++j) m = fmax_nan(m, fabsf(y[j]));
            int bad = !(m <= FLT_MAX);
            float mm = bad ? 0.0f : m;
            mm = grp_max(mm, 4);
            bad = grp_or(bad, 4);
            const uint32_t code = macro_code(p.ed, mm, bad);
            sm = e4m3_value(code);
            invm = __fdiv_rn(1.0f, sm);
            if (ok && (lane & 3) == 0) p.macro[c >> 2] = (uint8_t)code;
        }
        auto xq = [&](int j) -> float { return p.mbs ? __fmul_rn(y[j], invm) : y[j]; };

        uint32_t words[FAST ? 4 : 8];   // 4-bit: 4 words of 8 nibbles; FP6: 8 words of 4 bytes
#pragma unroll
        for (int i = 0; i < (FAST ? 4 : 8); ++i) words[i] = 0;
        uint32_t scode[NB];
        uint16_t obits[NB];

#pragma unroll
        for (int k = 0; k < NB; ++k) {
            const int j0 = k * L;
            float a = 0.0f, mn = FLT_MAX, mx = -FLT_MAX;
#pragma unroll
            for (int j = j0; j < j0 + L; ++j) {
                const float v = xq(j);
                a = fmax_nan(a, fabsf(v));
                if (!FAST && p.asym) { mn = fminf(mn, v); mx = fmaxf(mx, v); }
            }
            int bad = !(a <= FLT_MAX);
            if (G > 1) {
                a = grp_max(bad ? 0.0f : a, G);
                bad = grp_or(bad, G);
                if (!FAST && p.asym) { mn = grp_min(mn, G); mx = grp_max(mx, G); }
            }
            float o = 0.0f;
            if (!FAST && p.asym) {
                if (!bad) o = p.ed.is_int ? bf16_round(mn) : bf16_round(__fmul_rn(__fadd_rn(mx, mn), 0.5f));
                float ra = 0.0f;
#pragma unroll
                for (int j = j0; j < j0 + L; ++j) {
                    const float d = __fsub_rn(xq(j), o);
                    ra = fmaxf(ra, p.ed.is_int ? d : fabsf(d));
                }
                if (G > 1) ra = grp_max(ra, G);
                a = ra;
            }
            const BlockScale bs = block_scale(p.ed, p.sd, bad ? 0.0f : a, bad, sT);
            scode[k] = bs.code;
            obits[k] = (!FAST && p.asym) ? __bfloat16_as_ushort(__float2bfloat16_rn(o)) : (uint16_t)0;

            if constexpr (FAST) {
                // E2M1, RTNE: conversion instruction, 8 elements per word
                float deqT = bs.nan ? __uint_as_float(0x7fc00000u)
                           : nearest ? __fmul_rn(bs.deq, sT) : bs.deq;
                if (p.mbs) deqT = __fmul_rn(deqT, sm);
                float sx = 0.f, se = 0.f, sb = 0.f;
                int xz = 0, qz = 0;
#pragma unroll
                for (int w = 0; w < L / 8; ++w) {
                    const int jb = j0 + 8 * w;
                    float s8[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) s8[i] = __fmul_rn(xq(jb + i), bs.inv);
                    const uint32_t word = bs.zero ? 0u : cvt_e2m1x8(s8);
                    words[jb >> 3] = word;
                    if (stats) {
                        float q[8];
                        e2m1x8_values(word, q);
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const float yv = y[jb + i];
                            const float d = fmaf(-q[i], deqT, yv);
                            se = fmaf(d, d, se);
                            sx = fmaf(yv, yv, sx);
                            sb -= d;
                            xz += (yv == 0.0f);
                        }
                        qz += zero_codes8(word);
                    }
                }
                if (stats && ok) {
                    acc.x2 += (double)sx;
                    acc.e2 += (double)se;
                    acc.e += (double)sb;
                    acc.nz += (double)(L - xz);
                    acc.ftz += bs.nan ? 0.0 : (double)(qz - xz);
                }
            } else {
                uint4 rw = make_uint4(0, 0, 0, 0);
                float yv[L], xh[L];
#pragma unroll
                for (int j = j0; j < j0 + L; ++j) {
                    if (p.round_mode == RD_SR && (j & 3) == 0)
                        rw = element_words(p.seed, ((uint64_t)e0 + j) >> 2);
                    float q = 0.0f;
                    uint32_t code = 0;
                    if (!bs.zero) {
                        float v = xq(j);
                        if (p.asym) v = __fsub_rn(v, o);
                        code = encode_elem(p.ed, p.round_mode, __fmul_rn(v, bs.inv), word_of(rw, j & 3), q);
                    }
                    if (p.ed.code_bits == 4) words[j >> 3] |= code << (4 * (j & 7));
                    else words[j >> 2] |= code << (8 * (j & 3));
                    yv[j - j0] = y[j];
                    xh[j - j0] = deq_value(p, q, bs, sm, o, sT);
                }
                if (stats && ok) acc_add<L>(acc, yv, xh);
            }
        }

        if (ok) {
            // codes: 16 bytes (4-bit) or 32 bytes (FP6) per thread
            if (FAST || p.ed.code_bits == 4) {
                reinterpret_cast<uint4 *>(p.codes)[c] = make_uint4(words[0], words[1], words[2], words[3]);
            } else {
                uint4 *dst = reinterpret_cast<uint4 *>(p.codes) + 2 * (size_t)c;
                if (p.sf_gemm) {                    // dense tensor-core operand form, 24 bytes
                    fp6_store_dense(static_cast<uint8_t *>(p.codes) + 24 * (size_t)c,
                                    fp6_group_pack(words[0], words[1], words[2], words[3]),
                                    fp6_group_pack(words[FAST ? 0 : 4], words[FAST ? 0 : 5], words[FAST ? 0 : 6],
                                                   words[FAST ? 0 : 7]));
                } else {
                    dst[0] = make_uint4(words[0], words[1], words[2], words[3]);
                    dst[1] = make_uint4(words[FAST ? 0 : 4], words[FAST ? 0 : 5], words[FAST ? 0 : 6],
                                        words[FAST ? 0 : 7]);
                }
            }
            // scales (and offsets): NB per thread, or one per G lanes
            if (G == 1 || (lane & (G - 1)) == 0) {
                const uint32_t b0 = (G == 1) ? c * NB : c / G;
                if (p.sf_gemm) {
                    const uint32_t r = b0 / S, j = b0 - r * S;
#pragma unroll
                    for (int k = 0; k < NB; ++k) p.scales[sf_chunk_index(r, j + k, S)] = (uint8_t)scode[k];
                } else if (NB == 4) {
                    *reinterpret_cast<uint32_t *>(p.scales + b0) =
                        scode[0] | (scode[NB > 1 ? 1 : 0] << 8) | (scode[NB > 2 ? 2 : 0] << 16) | (scode[NB > 3 ? 3 : 0] << 24);
                } else if (NB == 2) {
                    *reinterpret_cast<uint16_t *>(p.scales + b0) = (uint16_t)(scode[0] | (scode[NB > 1 ? 1 : 0] << 8));
                } else {
                    p.scales[b0] = (uint8_t)scode[0];
                }
                if (!FAST && p.asym)
#pragma unroll
                    for (int k = 0; k < NB; ++k) p.offsets[b0 + k] = obits[k];
            }
        }
    }
    finish_launch(p, acc);
}

// Tensor absmax of y (NaN skipped) for the per-tensor scale, row chunks
// (rotation along rows: row and 2D layouts).
template <typename InT>
__global__ void __launch_bounds__(kThreads) k_amax_row(const QParams p)
{
    const InT *x = static_cast<const InT *>(p.x);
    const int lane = threadIdx.x & 31;
    const uint32_t nch = (uint32_t)(p.rows * p.cols / 32);
    const uint32_t gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t nw = (gridDim.x * blockDim.x) >> 5;
    float m = 0.0f;
    for (uint32_t c0 = gw * 32; c0 < nch; c0 += nw * 32) {
        const uint32_t c = c0 + lane;
        float v[32];
        if (c < nch) load32(x, (int64_t)c * 32, v);
        else
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = 0.0f;
        if (p.had) hadamard32(v, p.had);
#pragma unroll
        for (int j = 0; j < 32; ++j) m = fmaxf(m, fabsf(v[j]));
    }
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
    if (lane == 0 && m > 0.0f) atomicMax(p.amax_word, __float_as_uint(m));
}

// Tensor absmax without rotation (any block axis), of up to kFastGroupMax
// tensors in one launch (the CTAs split among them in proportion to their
// sizes): consecutive lanes read consecutive 16-byte vectors, four in flight
// per thread, NaN skipped.  Each tensor is walked from its end towards its
// start, so that the quantizer's forward walk that follows first meets the
// lines this pass touched last (still in L2 when the tensor is not much
// larger than L2).
struct AmaxGroup {
    const void *x[kFastGroupMax];
    uint64_t nv[kFastGroupMax];             // 16-byte vectors
    unsigned int *word[kFastGroupMax];
    uint32_t cta0[kFastGroupMax + 1];
    int n;
};

template <typename InT>
__global__ void __launch_bounds__(kThreads) k_amax_vec(const __grid_constant__ AmaxGroup g)
{
    constexpr int U = 4;
    int item = 0;
    while (item + 1 < g.n && blockIdx.x >= g.cta0[item + 1]) ++item;
    const uint4 *x = static_cast<const uint4 *>(g.x[item]);
    const uint64_t nv = g.nv[item];
    const uint64_t cta = blockIdx.x - g.cta0[item];
    const uint64_t T = (uint64_t)(g.cta0[item + 1] - g.cta0[item]) * blockDim.x;
    pdl_trigger();
    pdl_wait();
    float m = 0.0f;
    __nv_bfloat162 m2 = __float2bfloat162_rn(0.0f);
    for (uint64_t i = cta * blockDim.x + threadIdx.x; i < nv; i += U * T) {
        uint4 u[U];
#pragma unroll
        for (int k = 0; k < U; ++k) {
            const uint64_t j = i + k * T;
            u[k] = j < nv ? __ldg(x + (nv - 1 - j)) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int k = 0; k < U; ++k) {
            if constexpr (sizeof(InT) == 2) {
                const uint32_t w[4] = {u[k].x, u[k].y, u[k].z, u[k].w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    m2 = __hmax2(m2, __habs2(*reinterpret_cast<const __nv_bfloat162 *>(&w[e])));
            } else {
                m = fmaxf(m, fmaxf(fmaxf(fabsf(__uint_as_float(u[k].x)), fabsf(__uint_as_float(u[k].y))),
                                   fmaxf(fabsf(__uint_as_float(u[k].z)), fabsf(__uint_as_float(u[k].w)))));
            }
        }
    }
    if constexpr (sizeof(InT) == 2) {
        const float2 f = __bfloat1622float2(m2);
        m = fmaxf(f.x, f.y);
    }
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
    if ((threadIdx.x & 31) == 0 && m > 0.0f) atomicMax(g.word[item], __float_as_uint(m));
}

template <typename InT>
int launch_amax_vec(const QParams *ps, int n, cudaStream_t st)
{
    AmaxGroup g;
    memset(&g, 0, sizeof(g));
    uint64_t warps[kFastGroupMax], sum = 0;
    for (int i = 0; i < n; ++i) {
        g.x[i] = ps[i].x;
        g.nv[i] = (uint64_t)(ps[i].rows * ps[i].cols) * sizeof(InT) / 16;
        g.word[i] = ps[i].amax_word;
        warps[i] = (g.nv[i] / 4 + 31) / 32;
        sum += warps[i];
    }
    g.n = n;
    // the one-tensor grid for the sum of the tensors, then a share of it per
    // tensor in proportion to its vectors (at least one CTA each)
    const int total = grid_for(k_amax_vec<InT>, (int64_t)sum);
    g.cta0[0] = 0;
    uint64_t given = 0, acc = 0;
    for (int i = 0; i < n; ++i) {
        acc += warps[i];
        uint64_t upto = sum ? (uint64_t)total * acc / sum : (uint64_t)i + 1;
        if (upto < given + 1) upto = given + 1;
        g.cta0[i + 1] = (uint32_t)upto;
        given = upto;
    }
    return launch_pdl(k_amax_vec<InT>, g.cta0[n], kThreads, 0, st, g) == cudaSuccess ? 0 : -1;
}

int launch_tensor_amax_group(const QParams *ps, int n, int in_fp32, cudaStream_t st)
{
    if (n < 1 || n > kFastGroupMax) return -1;
    return in_fp32 ? launch_amax_vec<float>(ps, n, st) : launch_amax_vec<__nv_bfloat16>(ps, n, st);
}

// Sum the per-CTA records in a fixed order and derive MSE, R-MSE, QSNR (Eq. (1)),
// bias and the flush-to-zero share.
// derived statistics recomputed from the sums and the count already in
// `stats` (after the sums of several calls were added together)
__global__ void k_refinalize_stats(double *stats)
{
    const double s[5] = {stats[0], stats[1], stats[2], stats[3], stats[4]};
    store_stats(stats, s, stats[10]);
}

__global__ void k_finalize_stats(const double *partials, int nparts, double count, double *stats)
{
    __shared__ double sh[256][5];
    double s[5] = {0, 0, 0, 0, 0};
    for (int i = threadIdx.x; i < nparts; i += blockDim.x)
        for (int k = 0; k < 5; ++k) s[k] += partials[(int64_t)i * kPartialDoubles + k];
    for (int k = 0; k < 5; ++k) sh[threadIdx.x][k] = s[k];
    __syncthreads();
    for (int w = blockDim.x / 2; w > 0; w >>= 1) {
        if ((int)threadIdx.x < w)
            for (int k = 0; k < 5; ++k) sh[threadIdx.x][k] += sh[threadIdx.x + w][k];
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        const double t[5] = {sh[0][0], sh[0][1], sh[0][2], sh[0][3], sh[0][4]};
        store_stats(stats, t, count);
    }
}

// ============================================================== launches ===
int cached_occupancy(const void *kernel, int threads, size_t smem)
{
    struct Entry { const void *k; int threads; size_t smem; int occ; };
    static Entry table[64];
    static int used = 0;
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i)
        if (table[i].k == kernel && table[i].threads == threads && table[i].smem == smem) return table[i].occ;
    if (smem > 48 * 1024) cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    int occ = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, threads, smem) != cudaSuccess || occ < 1) occ = 1;
    if (used < 64) table[used++] = Entry{kernel, threads, smem, occ};
    return occ;
}

static int g_sms = 0;
int device_sm_count()
{
    if (g_sms == 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess) return 148;
        if (cudaDeviceGetAttribute(&g_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) g_sms = 148;
    }
    return g_sms;
}

template <typename InT, int B>
static int launch_row_b(const QParams &p, int fast, cudaStream_t st, int *grid_out)
{
    const int64_t warps = (p.rows * p.cols / 32 + 31) / 32;
    if (fast) {
        const int g = grid_for(k_quant_row<InT, B, true>, warps);
        k_quant_row<InT, B, true><<<g, kThreads, 0, st>>>(p);
        *grid_out = g;
    } else {
        const int g = grid_for(k_quant_row<InT, B, false>, warps);
        k_quant_row<InT, B, false><<<g, kThreads, 0, st>>>(p);
        *grid_out = g;
    }
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

template <typename InT>
static int launch_row(const QParams &p, int fast, cudaStream_t st, int *grid_out)
{
    switch (p.block) {
    case 8: return launch_row_b<InT, 8>(p, fast, st, grid_out);
    case 16: return launch_row_b<InT, 16>(p, fast, st, grid_out);
    case 32: return launch_row_b<InT, 32>(p, fast, st, grid_out);
    case 64: return launch_row_b<InT, 64>(p, fast, st, grid_out);
    case 128: return launch_row_b<InT, 128>(p, fast, st, grid_out);
    case 256: return launch_row_b<InT, 256>(p, fast, st, grid_out);
    default: return -1;
    }
}

int launch_quantize(const QParams &p, int axis, int in_fp32, int fast, cudaStream_t st, int *grid_out)
{
    if (axis == AX_ROW && fast && !p.rotated &&
        ((!p.mbs && !p.had) || p.block == 16 || p.block == 32))
        return launch_quantize_fast(p, in_fp32, st, grid_out);
    if (axis == AX_ROW && !fast && !p.rotated && !p.mbs && !p.had && p.block == 32)
        return launch_quantize_gen(p, in_fp32, st, grid_out);
    if (axis == AX_ROW)
        return in_fp32 ? launch_row<float>(p, fast, st, grid_out)
                       : launch_row<__nv_bfloat16>(p, fast, st, grid_out);
    return launch_quantize_col(p, axis, in_fp32, fast, st, grid_out);
}

int launch_tensor_amax(const QParams &p, int axis, int in_fp32, cudaStream_t st)
{
    cudaError_t e = cudaSuccess;
    if (axis == AX_COL && p.had) {
        if (launch_amax_col(p, in_fp32, st)) return -1;
    } else if (!p.had) {
        if (launch_tensor_amax_group(&p, 1, in_fp32, st)) return -1;
    } else {
        const int64_t tiles = (p.rows * p.cols / 32 + 31) / 32;
        if (in_fp32) {
            const int g = grid_for(k_amax_row<float>, tiles);
            k_amax_row<float><<<g, kThreads, 0, st>>>(p);
        } else {
            const int g = grid_for(k_amax_row<__nv_bfloat16>, tiles);
            k_amax_row<__nv_bfloat16><<<g, kThreads, 0, st>>>(p);
        }
    }
    return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? 0 : -1;
}

int launch_finalize_stats(const double *partials, int nparts, double count, double *stats,
                          cudaStream_t st)
{
    k_finalize_stats<<<1, 256, 0, st>>>(partials, nparts, count, stats);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

int launch_stats_refinalize(double *stats, cudaStream_t st)
{
    k_refinalize_stats<<<1, 1, 0, st>>>(stats);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace mxk
