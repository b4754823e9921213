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
// Thread = 32 consecutive elements of a row (every axis): one 16-byte code
// load (4-bit) or two (FP6), the block scales of those elements, and 64 / 128
// output bytes; the rotation, when on, runs along rows inside the thread
// (row and 2D layouts).
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

template <bool FAST>
__global__ void __launch_bounds__(kThreads) k_dequant_chunk(const DParams p)
{
    const int lane = threadIdx.x & 31;
    const uint32_t nch = (uint32_t)(p.rows * p.cols / 32);
    const uint32_t cpr = (uint32_t)(p.cols / 32);                 // chunks per row
    const uint32_t gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t nw = (gridDim.x * blockDim.x) >> 5;
    const float sT = (p.ts_mode != TS_NONE && p.tensor_scale) ? *p.tensor_scale : 1.0f;
    const bool nearest = p.sd.fmt != S_E8M0 && p.sd.rule == R_NEAREST;
    const int B = p.block;
    const int lb = __ffs(B) - 1;                                   // B is a power of two
    const uint32_t S = (uint32_t)(p.cols >> lb);                   // row-axis scales per row
    for (uint32_t c0 = gw * 32; c0 < nch; c0 += nw * 32) {
        const uint32_t c = c0 + lane;
        const bool ok = c < nch;
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = 0.0f;
        if (ok) {
            const uint32_t row = c / cpr;
            const uint32_t col0 = (c - row * cpr) * 32;
            uint32_t w[8];
            if (p.ed.code_bits == 4) {
                const uint4 u = reinterpret_cast<const uint4 *>(p.codes)[c];
                w[0] = u.x; w[1] = u.y; w[2] = u.z; w[3] = u.w;
            } else {
                if (p.sf_gemm) {                    // dense tensor-core operand form
                    uint4 g0, g1;
                    fp6_load_dense(static_cast<const uint8_t *>(p.codes) + 24 * (size_t)c, g0, g1);
                    fp6_group_unpack(g0, w);
                    fp6_group_unpack(g1, w + 4);
                } else {
                    const uint4 u0 = reinterpret_cast<const uint4 *>(p.codes)[2 * (size_t)c];
                    const uint4 u1 = reinterpret_cast<const uint4 *>(p.codes)[2 * (size_t)c + 1];
                    w[0] = u0.x; w[1] = u0.y; w[2] = u0.z; w[3] = u0.w;
                    w[4] = u1.x; w[5] = u1.y; w[6] = u1.z; w[7] = u1.w;
                }
            }
            if (FAST) {
                // E2M1, symmetric, power-of-two or NEAREST scales, row or 2D axis, no MBS
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const uint32_t col = col0 + 8 * g;
                    uint32_t sc;
                    if (p.axis == AX_ROW)
                        sc = p.sf_gemm ? p.scales[sf_chunk_index(row, col >> lb, S)]
                                       : p.scales[(size_t)row * S + (col >> lb)];
                    else
                        sc = p.scales[(size_t)(row >> 5) * (p.cols >> 5) + (col >> 5)];
                    const float sb = scale_value(p.sd, sc);
                    const float2 sb2 = make_float2(sb, sb), sT2 = make_float2(sT, sT);
                    float q[8];
                    e2m1x8_values(w[g], q);
#pragma unroll
                    for (int i = 0; i < 8; i += 2) {
                        // (q * s_b) [* s_T], each product one binary32 rounding per lane
                        float2 t = __fmul2_rn(make_float2(q[i], q[i + 1]), sb2);
                        if (nearest) t = __fmul2_rn(t, sT2);
                        v[8 * g + i] = t.x;
                        v[8 * g + i + 1] = t.y;
                    }
                }
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const uint32_t col = col0 + j;
                    size_t b;
                    if (p.axis == AX_ROW) b = (size_t)row * S + (col >> lb);
                    else if (p.axis == AX_COL) b = (size_t)(row >> lb) * p.cols + col;
                    else b = (size_t)(row >> 5) * (p.cols >> 5) + (col >> 5);
                    const uint32_t sc = (p.axis == AX_ROW && p.sf_gemm)
                                            ? p.scales[sf_chunk_index(row, col >> lb, S)]
                                            : p.scales[b];
                    const uint32_t code = (p.ed.code_bits == 4) ? (w[j >> 3] >> (4 * (j & 7))) & 0xfu
                                                                : (w[j >> 2] >> (8 * (j & 3))) & 0x3fu;
                    float sm = 1.0f;
                    if (p.mbs) {
                        const size_t mi = (p.axis == AX_COL) ? (size_t)(row / 128) * p.cols + col
                                                             : (size_t)row * (p.cols / 128) + col / 128;
                        sm = e4m3_value(p.macro[mi]);
                    }
                    const float o = p.asym ? __uint_as_float((uint32_t)p.offsets[b] << 16) : 0.0f;
                    v[j] = deq_one(p, code, sc, sT, sm, o);
                }
            }
        }
        if (p.had) hadamard32(v, p.had);
        if (ok) {
            const int64_t e0 = (int64_t)c * 32;
            if (p.out_fp32) {
                float4 *o = reinterpret_cast<float4 *>(static_cast<float *>(p.out) + e0);
#pragma unroll
                for (int i = 0; i < 8; ++i) o[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            } else {
                uint4 *o = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.out) + e0);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    uint32_t t[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        __nv_bfloat162 h = __floats2bfloat162_rn(v[8 * i + 2 * k], v[8 * i + 2 * k + 1]);
                        t[k] = *reinterpret_cast<uint32_t *>(&h);
                    }
                    o[i] = make_uint4(t[0], t[1], t[2], t[3]);
                }
            }
        }
    }
}

// ---------------------------------------------------- E2M1, 8 per lane --
// Exact unsigned division by a runtime divisor d >= 2 through a multiply-high
// (Granlund and Montgomery, PLDI 1994, Fig. 4.1): t = umulhi(n, m),
// q = (t + ((n - t) >> s1)) >> s2 for every 32-bit n.
struct FastDiv {
    uint32_t m;
    int s1, s2;
};

__device__ __forceinline__ uint32_t fast_div(uint32_t n, const FastDiv &f)
{
    const uint32_t t = __umulhi(n, f.m);
    return (t + ((n - t) >> f.s1)) >> f.s2;
}

// E8M0 / unsigned-minifloat block-scale value without branches on the code
__device__ __forceinline__ float scale_value_fast(const ScaleDesc &sd, uint32_t code)
{
    if (sd.fmt == S_E8M0)
        return __uint_as_float(code == 0xffu ? 0x7fc00000u : code ? code << 23 : 0x00400000u);
    return ue_value(sd, code);
}

// E2M1, symmetric, no macro scale or rotation, every axis and scale layout.
// Thread = 8 consecutive elements of a row (an octet: one 32-bit code word
// in, 16 bytes of bf16 or 32 of fp32 out), so consecutive lanes read and
// write consecutive addresses; four octets in flight per thread.
template <int AXIS, bool OUT32>
__global__ void __launch_bounds__(kThreads) k_dequant_oct(const DParams p, const FastDiv opr_div, uint32_t noct)
{
    constexpr int U = 4;
    const uint32_t T = gridDim.x * blockDim.x;
    pdl_trigger();
    pdl_wait();
    const float sT = (p.ts_mode != TS_NONE && p.tensor_scale) ? *p.tensor_scale : 1.0f;
    const bool nearest = p.sd.fmt != S_E8M0 && p.sd.rule == R_NEAREST;
    const int lb = __ffs(p.block) - 1;
    const uint32_t cols = (uint32_t)p.cols, opr = cols >> 3;
    const uint32_t S = cols >> lb;
    const uint32_t *codes = static_cast<const uint32_t *>(p.codes);
    for (uint32_t o0 = blockIdx.x * blockDim.x + threadIdx.x; o0 < noct; o0 += U * T) {
        uint32_t w[U], sc[U][AXIS == AX_COL ? 2 : 1];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const uint32_t o = o0 + u * T;
            w[u] = 0;
            sc[u][0] = 0;
            if (AXIS == AX_COL) sc[u][AXIS == AX_COL ? 1 : 0] = 0;
            if (o < noct) {
                w[u] = __ldg(codes + o);
                if (AXIS == AX_ROW && !p.sf_gemm) {
                    sc[u][0] = __ldg(p.scales + (o >> (lb - 3)));
                } else {
                    const uint32_t row = fast_div(o, opr_div), col = (o - row * opr) << 3;
                    if (AXIS == AX_ROW) {
                        sc[u][0] = __ldg(p.scales + sf_chunk_index(row, col >> lb, S));
                    } else if (AXIS == AX_2D) {
                        sc[u][0] = __ldg(p.scales + (size_t)(row >> 5) * (cols >> 5) + (col >> 5));
                    } else {
                        const uint2 b = __ldg(reinterpret_cast<const uint2 *>(p.scales + (size_t)(row >> lb) * cols + col));
                        sc[u][0] = b.x;
                        sc[u][AXIS == AX_COL ? 1 : 0] = b.y;
                    }
                }
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const uint32_t o = o0 + u * T;
            if (o >= noct) break;
            float q[8];
            e2m1x8_values(w[u], q);
            float v[8];
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
                float s0, s1;
                if (AXIS == AX_COL) {
                    const uint32_t word = sc[u][i >> 2];
                    s0 = scale_value_fast(p.sd, (word >> (8 * (i & 3))) & 0xffu);
                    s1 = scale_value_fast(p.sd, (word >> (8 * ((i + 1) & 3))) & 0xffu);
                } else {
                    s0 = s1 = scale_value_fast(p.sd, sc[u][0]);
                }
                float2 t = __fmul2_rn(make_float2(q[i], q[i + 1]), make_float2(s0, s1));
                if (nearest) t = __fmul2_rn(t, make_float2(sT, sT));
                v[i] = t.x;
                v[i + 1] = t.y;
            }
            if (OUT32) {
                float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(p.out) + (size_t)o * 8);
                dst[0] = make_float4(v[0], v[1], v[2], v[3]);
                dst[1] = make_float4(v[4], v[5], v[6], v[7]);
            } else {
                uint32_t t[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
                    t[k] = *reinterpret_cast<uint32_t *>(&h);
                }
                reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.out))[o] = make_uint4(t[0], t[1], t[2], t[3]);
            }
        }
    }
}

FastDiv make_fast_div(uint32_t d)
{
    int l = 0;
    while ((1ull << l) < d) ++l;
    FastDiv f;
    f.m = (uint32_t)((((1ull << l) - d) << 32) / d + 1);
    f.s1 = l < 1 ? l : 1;
    f.s2 = l > 1 ? l - 1 : 0;
    return f;
}

template <int AXIS>
int launch_dequant_oct(const DParams &p, cudaStream_t st)
{
    const uint64_t noct = (uint64_t)(p.rows * p.cols / 8);
    const FastDiv f = make_fast_div((uint32_t)(p.cols / 8));
    cudaError_t e;
    if (p.out_fp32) {
        const int g = grid_of(k_dequant_oct<AXIS, true>, (int64_t)(noct / 4 + 255) / 256 * 8);
        e = launch_pdl(k_dequant_oct<AXIS, true>, g, kThreads, 0, st, p, f, (uint32_t)noct);
    } else {
        const int g = grid_of(k_dequant_oct<AXIS, false>, (int64_t)(noct / 4 + 255) / 256 * 8);
        e = launch_pdl(k_dequant_oct<AXIS, false>, g, kThreads, 0, st, p, f, (uint32_t)noct);
    }
    return e == cudaSuccess ? 0 : -1;
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
    } else if (p.ed.elem == E2M1 && !p.asym && !p.mbs && !p.had && p.rows * p.cols / 8 < (INT64_C(1) << 32)) {
        if (p.axis == AX_ROW) return launch_dequant_oct<AX_ROW>(p, st);
        if (p.axis == AX_COL) return launch_dequant_oct<AX_COL>(p, st);
        return launch_dequant_oct<AX_2D>(p, st);
    } else {
        const int64_t warps = (p.rows * p.cols / 32 + 31) / 32;
        const bool fast = p.ed.elem == E2M1 && !p.asym && !p.mbs && p.axis != AX_COL;
        if (fast) {
            const int g = grid_of(k_dequant_chunk<true>, warps);
            k_dequant_chunk<true><<<g, kThreads, 0, st>>>(p);
        } else {
            const int g = grid_of(k_dequant_chunk<false>, warps);
            k_dequant_chunk<false><<<g, kThreads, 0, st>>>(p);
        }
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
