// sm_100a dequantization and fidelity-reduction kernels.
//
// Dequantization is the fake-quantization half of the fmread summary of Yang
// et al. (quantize, then return to high precision); the reductions are the
// tensor QSNR of "Unveiling the Potential of Quantization with MXFP4", Sec.3
// Eq. (1), the R-MSE of the same summary, and the per-block MSE of "Is Finer
// Better?" (error decomposition per block and per tensor).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <float.h>
#include <stdint.h>

#include "mx_device.cuh"
#include "mx_internal.h"

namespace mxk {

namespace {
constexpr unsigned kFull = 0xffffffffu;
constexpr int kThreads = 256;

__device__ __forceinline__ float qnan() { return __uint_as_float(0x7fc00000u); }

// block-scale value of a stored byte
__device__ __forceinline__ float scale_value(const ScaleDesc &sd, uint32_t code)
{
    if (sd.fmt == S_E8M0) return code == 0xffu ? qnan() : exp2i((int)code - 127);
    return ue_value(sd, code);
}

__device__ __forceinline__ float deq_one(const DParams &p, uint32_t code, uint32_t scode,
                                         float sT, float sm, float o)
{
    const float s = scale_value(p.sd, scode);
    if (s != s) return qnan();
    const float q = decode_elem(p.ed, code);
    if (p.sd.fmt != S_E8M0 && p.sd.rule == R_NEAREST) return __fmul_rn(__fmul_rn(q, s), sT);
    float v = __fmul_rn(q, s);
    if (p.mbs) v = __fmul_rn(v, sm);
    if (p.asym) v = __fadd_rn(v, o);
    return v;
}

__device__ __forceinline__ void hadamard8(float y[8], int n, int lane)
{
#pragma unroll
    for (int h = 1; h < 8; h <<= 1)
#pragma unroll
        for (int i = 0; i < 8; i += 2 * h)
#pragma unroll
            for (int j = i; j < i + h; ++j) {
                float a = y[j], b = y[j + h];
                y[j] = __fadd_rn(a, b);
                y[j + h] = __fsub_rn(a, b);
            }
    for (int m = 1; m < n / 8; m <<= 1) {
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float w = __shfl_xor_sync(kFull, y[j], m);
            y[j] = upper ? __fsub_rn(w, y[j]) : __fadd_rn(y[j], w);
        }
    }
    const float c = hadamard_scale(n);
#pragma unroll
    for (int j = 0; j < 8; ++j) y[j] = __fmul_rn(y[j], c);
}

__device__ __forceinline__ void store8(void *out, bool f32, int64_t e, const float v[8])
{
    if (f32) {
        float *o = static_cast<float *>(out) + e;
        reinterpret_cast<float4 *>(o)[0] = make_float4(v[0], v[1], v[2], v[3]);
        reinterpret_cast<float4 *>(o)[1] = make_float4(v[4], v[5], v[6], v[7]);
    } else {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            w[i] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[2 * i])) |
                   ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[2 * i + 1])) << 16);
        *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(out) + e) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

__device__ __forceinline__ void unpack_bf16x2(uint32_t w, float &lo, float &hi)
{
    lo = __uint_as_float(w << 16);
    hi = __uint_as_float(w & 0xffff0000u);
}

__device__ __forceinline__ void load8any(const void *x, bool f32, int64_t e, float v[8])
{
    if (f32) {
        const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(x) + e);
        float4 a = __ldg(p), b = __ldg(p + 1);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
        uint4 u = __ldg(reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(x) + e));
        unpack_bf16x2(u.x, v[0], v[1]);
        unpack_bf16x2(u.y, v[2], v[3]);
        unpack_bf16x2(u.z, v[4], v[5]);
        unpack_bf16x2(u.w, v[6], v[7]);
    }
}

// ------------------------------------------------------------ dequantize --
// Thread = 8 consecutive elements of a row (every axis); the rotation, when
// on, runs along rows (row and 2D layouts).
__global__ void __launch_bounds__(kThreads) k_dequant_chunk(const DParams p)
{
    const int lane = threadIdx.x & 31;
    const int64_t nchunks = p.rows * p.cols / 8;
    const int64_t ntiles = (nchunks + 31) / 32;
    const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const float sT = (p.ts_mode != TS_NONE && p.tensor_scale) ? *p.tensor_scale : 1.0f;
    for (int64_t t = gw; t < ntiles; t += nw) {
        const int64_t c = t * 32 + lane;
        const bool ok = c < nchunks;
        float v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        if (ok) {
            const int64_t e0 = c * 8;
            const int64_t row = e0 / p.cols, col0 = e0 - row * p.cols;
            uint32_t lo, hi = 0;
            if (p.ed.code_bits == 4) {
                lo = reinterpret_cast<const uint32_t *>(p.codes)[c];
            } else {
                const uint2 w = reinterpret_cast<const uint2 *>(p.codes)[c];
                lo = w.x;
                hi = w.y;
            }
            uint32_t sc[8];
            uint16_t of[8];
            uint32_t mc[8];
            if (p.axis == AX_COL) {
                const int64_t b0 = (row / p.block) * p.cols + col0;
                const uint2 s2 = *reinterpret_cast<const uint2 *>(p.scales + b0);
#pragma unroll
                for (int j = 0; j < 8; ++j) sc[j] = ((j < 4 ? s2.x : s2.y) >> (8 * (j & 3))) & 0xffu;
                if (p.asym)
#pragma unroll
                    for (int j = 0; j < 8; ++j) of[j] = p.offsets[b0 + j];
                if (p.mbs) {
                    const uint2 m2 = *reinterpret_cast<const uint2 *>(p.macro + (row / 128) * p.cols + col0);
#pragma unroll
                    for (int j = 0; j < 8; ++j) mc[j] = ((j < 4 ? m2.x : m2.y) >> (8 * (j & 3))) & 0xffu;
                }
            } else {
                const int64_t b = (p.axis == AX_ROW) ? e0 / p.block
                                                     : (row / 32) * (p.cols / 32) + col0 / 32;
                uint32_t s;
                if (p.axis == AX_ROW && p.sf_gemm) {
                    const int64_t S = p.cols / p.block;
                    s = p.scales[sf_chunk_index(row, col0 / p.block, S)];
                } else {
                    s = p.scales[b];
                }
                const uint16_t o = p.asym ? p.offsets[b] : 0;
                const uint32_t m = p.mbs ? p.macro[row * (p.cols / 128) + col0 / 128] : 0u;
#pragma unroll
                for (int j = 0; j < 8; ++j) { sc[j] = s; of[j] = o; mc[j] = m; }
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t code = (p.ed.code_bits == 4) ? (lo >> (4 * j)) & 0xfu
                                    : ((j < 4 ? lo : hi) >> (8 * (j & 3))) & 0x3fu;
                const float sm = p.mbs ? e4m3_value(mc[j]) : 1.0f;
                const float o = p.asym ? __uint_as_float((uint32_t)of[j] << 16) : 0.0f;
                v[j] = deq_one(p, code, sc[j], sT, sm, o);
            }
        }
        if (p.had) hadamard8(v, p.had, lane);
        if (ok) store8(p.out, p.out_fp32, c * 8, v);
    }
}

// Column axis with the rotation along columns: thread = 4 columns x `block`
// rows, rotated back in registers.
__global__ void __launch_bounds__(kThreads) k_dequant_colhad(const DParams p)
{
    const int lane = threadIdx.x & 31;
    const int RB = p.block;
    const int64_t ncc = p.cols / 4;
    const int64_t nwg = (ncc + 31) / 32;
    const int64_t nitems = (p.rows / RB) * nwg;
    const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const float sT = (p.ts_mode != TS_NONE && p.tensor_scale) ? *p.tensor_scale : 1.0f;
    const float cn = hadamard_scale(p.had);
    for (int64_t item = gw; item < nitems; item += nw) {
        const int64_t rg = item / nwg, wg = item - rg * nwg;
        const int64_t cc = wg * 32 + lane;
        if (cc >= ncc) continue;
        const int64_t c0 = cc * 4, r0 = rg * RB;
        float f[32][4];
        uint32_t sc[4], mc[4];
        uint16_t of[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            sc[j] = p.scales[rg * p.cols + c0 + j];
            of[j] = p.asym ? p.offsets[rg * p.cols + c0 + j] : 0;
            mc[j] = p.mbs ? p.macro[(r0 / 128) * p.cols + c0 + j] : 0u;
        }
#pragma unroll
        for (int r = 0; r < 32; ++r) {
            if (r < RB) {
                const int64_t e0 = (r0 + r) * p.cols + c0;
                uint32_t w;
                if (p.ed.code_bits == 4) w = *reinterpret_cast<const uint16_t *>(static_cast<const uint8_t *>(p.codes) + e0 / 2);
                else w = *reinterpret_cast<const uint32_t *>(static_cast<const uint8_t *>(p.codes) + e0);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t code = (p.ed.code_bits == 4) ? (w >> (4 * j)) & 0xfu : (w >> (8 * j)) & 0x3fu;
                    const float sm = p.mbs ? e4m3_value(mc[j]) : 1.0f;
                    const float o = p.asym ? __uint_as_float((uint32_t)of[j] << 16) : 0.0f;
                    f[r][j] = deq_one(p, code, sc[j], sT, sm, o);
                }
            } else {
#pragma unroll
                for (int j = 0; j < 4; ++j) f[r][j] = 0.0f;
            }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
            for (int h = 1; h < 32; h <<= 1) {
                if (h >= p.had) break;
#pragma unroll
                for (int i = 0; i < 32; i += 2 * h)
#pragma unroll
                    for (int r = i; r < i + h; ++r) {
                        float a = f[r][j], b = f[r + h][j];
                        f[r][j] = __fadd_rn(a, b);
                        f[r + h][j] = __fsub_rn(a, b);
                    }
            }
        }
#pragma unroll
        for (int r = 0; r < 32; ++r) {
            if (r >= RB) continue;
            const int64_t e0 = (r0 + r) * p.cols + c0;
            float v[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) v[j] = __fmul_rn(f[r][j], cn);
            if (p.out_fp32) {
                *reinterpret_cast<float4 *>(static_cast<float *>(p.out) + e0) = make_float4(v[0], v[1], v[2], v[3]);
            } else {
                uint32_t w0 = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[0])) |
                              ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[1])) << 16);
                uint32_t w1 = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[2])) |
                              ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[3])) << 16);
                *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(p.out) + e0) = make_uint2(w0, w1);
            }
        }
    }
}

// ------------------------------------------------------------ reductions --
struct Acc {
    double x2, e2, e, ftz, nz;
};

__device__ __forceinline__ double warp_sum(double v)
{
    for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(kFull, v, o);
    return v;
}

__device__ void write_record(double *partials, const Acc &a)
{
    __shared__ double sh[32][5];
    double v[5] = {a.x2, a.e2, a.e, a.ftz, a.nz};
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int i = 0; i < 5; ++i) v[i] = warp_sum(v[i]);
    if (lane == 0)
#pragma unroll
        for (int i = 0; i < 5; ++i) sh[w][i] = v[i];
    __syncthreads();
    if (threadIdx.x == 0) {
        double s[5] = {0, 0, 0, 0, 0};
        for (int k = 0; k < (int)(blockDim.x >> 5); ++k)
            for (int i = 0; i < 5; ++i) s[i] += sh[k][i];
        double *o = partials + (int64_t)blockIdx.x * kPartialDoubles;
        for (int i = 0; i < 5; ++i) o[i] = s[i];
        o[5] = o[6] = o[7] = 0.0;
    }
}

// Streaming sums; per-block MSE of row-axis blocks (B / 8 lanes per block).
__global__ void __launch_bounds__(kThreads) k_qsnr_chunk(const SParams p)
{
    const int lane = threadIdx.x & 31;
    const int64_t nchunks = p.rows * p.cols / 8;
    const int64_t ntiles = (nchunks + 31) / 32;
    const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int G = p.block / 8;
    Acc acc = {0, 0, 0, 0, 0};
    for (int64_t t = gw; t < ntiles; t += nw) {
        const int64_t c = t * 32 + lane;
        const bool ok = c < nchunks;
        float x[8] = {0, 0, 0, 0, 0, 0, 0, 0}, xh[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        if (ok) {
            load8any(p.x, p.x_fp32, c * 8, x);
            load8any(p.xh, p.xh_fp32, c * 8, xh);
        }
        float sx = 0.f, se = 0.f, sb = 0.f;
        int f = 0, z = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float d = x[j] - xh[j];
            sx = fmaf(x[j], x[j], sx);
            se = fmaf(d, d, se);
            sb -= d;
            const int nzj = (x[j] != 0.0f);
            z += nzj;
            f += nzj & (xh[j] == 0.0f);
        }
        if (p.per_block_mse) {
            float bs = se;
            for (int o = 1; o < G; o <<= 1) bs += __shfl_xor_sync(kFull, bs, o);
            if (ok && (lane & (G - 1)) == 0) p.per_block_mse[c / G] = bs / (float)p.block;
        }
        if (ok) {
            acc.x2 += (double)sx;
            acc.e2 += (double)se;
            acc.e += (double)sb;
            acc.ftz += (double)f;
            acc.nz += (double)z;
        }
    }
    write_record(p.partials, acc);
}

// Per-block MSE of column-axis and 2D blocks: thread = 4 columns x RB rows.
__global__ void __launch_bounds__(kThreads) k_qsnr_blocks_col(const SParams p)
{
    const int lane = threadIdx.x & 31;
    const int RB = (p.axis == AX_2D) ? 32 : p.block;
    const int64_t ncc = p.cols / 4;
    const int64_t nwg = (ncc + 31) / 32;
    const int64_t nitems = (p.rows / RB) * nwg;
    const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    Acc acc = {0, 0, 0, 0, 0};
    for (int64_t item = gw; item < nitems; item += nw) {
        const int64_t rg = item / nwg, wg = item - rg * nwg;
        const int64_t cc = wg * 32 + lane;
        const bool ok = cc < ncc;
        const int64_t c0 = cc * 4, r0 = rg * RB;
        float se_col[4] = {0, 0, 0, 0};
        for (int r = 0; r < RB; ++r) {
            float x[4] = {0, 0, 0, 0}, xh[4] = {0, 0, 0, 0};
            if (ok) {
                const int64_t e0 = (r0 + r) * p.cols + c0;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    x[j] = p.x_fp32 ? static_cast<const float *>(p.x)[e0 + j]
                                    : __bfloat162float(static_cast<const __nv_bfloat16 *>(p.x)[e0 + j]);
                    xh[j] = p.xh_fp32 ? static_cast<const float *>(p.xh)[e0 + j]
                                      : __bfloat162float(static_cast<const __nv_bfloat16 *>(p.xh)[e0 + j]);
                }
            }
            float sx = 0.f, se = 0.f, sb = 0.f;
            int f = 0, z = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float d = x[j] - xh[j];
                sx = fmaf(x[j], x[j], sx);
                se_col[j] = fmaf(d, d, se_col[j]);
                se = fmaf(d, d, se);
                sb -= d;
                const int nzj = (x[j] != 0.0f);
                z += nzj;
                f += nzj & (xh[j] == 0.0f);
            }
            if (ok) {
                acc.x2 += (double)sx;
                acc.e2 += (double)se;
                acc.e += (double)sb;
                acc.ftz += (double)f;
                acc.nz += (double)z;
            }
        }
        if (p.axis == AX_COL) {
            if (ok)
#pragma unroll
                for (int j = 0; j < 4; ++j) p.per_block_mse[rg * p.cols + c0 + j] = se_col[j] / (float)RB;
        } else {
            float s = se_col[0] + se_col[1] + se_col[2] + se_col[3];
            for (int o = 1; o < 8; o <<= 1) s += __shfl_xor_sync(kFull, s, o);
            if (ok && (lane & 7) == 0) p.per_block_mse[rg * (p.cols / 32) + c0 / 32] = s / 1024.0f;
        }
    }
    write_record(p.partials, acc);
}

template <typename K>
int grid_of(K kernel, int64_t work_warps)
{
    const int occ = cached_occupancy(reinterpret_cast<const void *>(kernel), kThreads, 0);
    int64_t g = (int64_t)device_sm_count() * occ;
    const int64_t need = (work_warps + (kThreads / 32) - 1) / (kThreads / 32);
    if (need < g) g = need;
    if (g < 1) g = 1;
    if (g > kMaxPartials) g = kMaxPartials;
    return (int)g;
}
}  // namespace

int launch_dequantize(const DParams &p, cudaStream_t st)
{
    if (p.axis == AX_COL && p.had) {
        const int64_t items = (p.rows / p.block) * ((p.cols / 4 + 31) / 32);
        const int g = grid_of(k_dequant_colhad, items);
        k_dequant_colhad<<<g, kThreads, 0, st>>>(p);
    } else {
        const int64_t tiles = (p.rows * p.cols / 8 + 31) / 32;
        const int g = grid_of(k_dequant_chunk, tiles);
        k_dequant_chunk<<<g, kThreads, 0, st>>>(p);
    }
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

int launch_qsnr(const SParams &p, cudaStream_t st, int *grid_out)
{
    if (p.per_block_mse && p.axis != AX_ROW) {
        const int RB = (p.axis == AX_2D) ? 32 : p.block;
        const int64_t items = (p.rows / RB) * ((p.cols / 4 + 31) / 32);
        const int g = grid_of(k_qsnr_blocks_col, items);
        k_qsnr_blocks_col<<<g, kThreads, 0, st>>>(p);
        *grid_out = g;
    } else {
        const int64_t tiles = (p.rows * p.cols / 8 + 31) / 32;
        const int g = grid_of(k_qsnr_chunk, tiles);
        k_qsnr_chunk<<<g, kThreads, 0, st>>>(p);
        *grid_out = g;
    }
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace mxk
