// Device helpers shared by the quantizer kernels: vector loads, lane-group
// reductions, the binary64 fidelity accumulators, the dequantization rule,
// the MBS macro-scale code and the row-direction Hadamard butterflies.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <float.h>
#include <stdint.h>

#include "mx_device.cuh"
#include "mx_internal.h"

namespace mxk {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kThreads = 256;

// maximum that propagates NaN (the non-finite block test reads it)
__device__ __forceinline__ float fmax_nan(float a, float b)
{
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

// three-operand maximum / minimum (sm_100)
__device__ __forceinline__ float fmax3_nan(float a, float b, float c)
{
    float r;
    asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
__device__ __forceinline__ float fmin3(float a, float b, float c)
{
    float r;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// number of zero-magnitude E2M1 codes among the 8 nibbles of w: a nibble's
// magnitude m (0..7) plus 7 sets bit 3 exactly when m != 0, with no carry out
__device__ __forceinline__ int e2m1_zero_codes8(uint32_t w)
{
    return 8 - __popc(((w & 0x77777777u) + 0x77777777u) & 0x88888888u);
}

// max |v| (NaN-propagating) and min |v| of L = 8, 16 or 32 values: L / 8
// independent chains of three-operand ops, then a short combine (the chains
// overlap in the pipeline instead of one dependent chain of L / 2 ops)
template <int L>
__device__ __forceinline__ float absmax_nan(const float *v)
{
    float c[L / 8];
#pragma unroll
    for (int i = 0; i < L / 8; ++i) {
        const float *w = v + 8 * i;
        float a = fmax3_nan(fabsf(w[0]), fabsf(w[1]), fabsf(w[2]));
        a = fmax3_nan(a, fabsf(w[3]), fabsf(w[4]));
        a = fmax3_nan(a, fabsf(w[5]), fabsf(w[6]));
        c[i] = fmax_nan(a, fabsf(w[7]));
    }
    if constexpr (L == 8) return c[0];
    else if constexpr (L == 16) return fmax_nan(c[0], c[L == 16 ? 1 : 0]);
    else return fmax_nan(fmax3_nan(c[0], c[L / 8 > 1 ? 1 : 0], c[L / 8 > 2 ? 2 : 0]), c[L / 8 > 3 ? 3 : 0]);
}
template <int L>
__device__ __forceinline__ float absmin(const float *v)
{
    float c[L / 8];
#pragma unroll
    for (int i = 0; i < L / 8; ++i) {
        const float *w = v + 8 * i;
        float a = fmin3(fabsf(w[0]), fabsf(w[1]), fabsf(w[2]));
        a = fmin3(a, fabsf(w[3]), fabsf(w[4]));
        a = fmin3(a, fabsf(w[5]), fabsf(w[6]));
        c[i] = fminf(a, fabsf(w[7]));
    }
    if constexpr (L == 8) return c[0];
    else if constexpr (L == 16) return fminf(c[0], c[L == 16 ? 1 : 0]);
    else return fminf(fmin3(c[0], c[L / 8 > 1 ? 1 : 0], c[L / 8 > 2 ? 2 : 0]), c[L / 8 > 3 ? 3 : 0]);
}

// ------------------------------------------------------------------ loads --
__device__ __forceinline__ void unpack_bf16x2(uint32_t w, float &lo, float &hi)
{
    lo = __uint_as_float(w << 16);
    hi = __uint_as_float(w & 0xffff0000u);
}

// 8 consecutive elements starting at element index e (e % 8 == 0)
__device__ __forceinline__ void load8(const __nv_bfloat16 *x, int64_t e, float v[8])
{
    uint4 u = __ldg(reinterpret_cast<const uint4 *>(x + e));
    unpack_bf16x2(u.x, v[0], v[1]);
    unpack_bf16x2(u.y, v[2], v[3]);
    unpack_bf16x2(u.z, v[4], v[5]);
    unpack_bf16x2(u.w, v[6], v[7]);
}
__device__ __forceinline__ void load8(const float *x, int64_t e, float v[8])
{
    float4 a = __ldg(reinterpret_cast<const float4 *>(x + e));
    float4 b = __ldg(reinterpret_cast<const float4 *>(x + e) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// CPT consecutive elements of one row (CPT * sizeof(T) in {8, 16} bytes)
template <int CPT>
__device__ __forceinline__ void load_row(const __nv_bfloat16 *x, int64_t e, float v[CPT])
{
    if constexpr (CPT == 8) {
        load8(x, e, v);
    } else {
        uint2 u = __ldg(reinterpret_cast<const uint2 *>(x + e));
        unpack_bf16x2(u.x, v[0], v[1]);
        unpack_bf16x2(u.y, v[2], v[3]);
    }
}
template <int CPT>
__device__ __forceinline__ void load_row(const float *x, int64_t e, float v[CPT])
{
    static_assert(CPT == 4, "fp32 rows are loaded 4 at a time");
    float4 a = __ldg(reinterpret_cast<const float4 *>(x + e));
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}

__device__ __forceinline__ void store8f(float *y, int64_t e, const float v[8])
{
    reinterpret_cast<float4 *>(y + e)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4 *>(y + e)[1] = make_float4(v[4], v[5], v[6], v[7]);
}

// ------------------------------------------------------ group reductions --
// Reductions over aligned groups of G lanes (G a power of two, warp-uniform).
__device__ __forceinline__ float grp_max(float v, int G)
{
    for (int o = 1; o < G; o <<= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
    return v;
}
__device__ __forceinline__ float grp_min(float v, int G)
{
    for (int o = 1; o < G; o <<= 1) v = fminf(v, __shfl_xor_sync(kFull, v, o));
    return v;
}
__device__ __forceinline__ int grp_or(int v, int G)
{
    for (int o = 1; o < G; o <<= 1) v |= __shfl_xor_sync(kFull, v, o);
    return v;
}

__device__ __forceinline__ int nonfinite(float v) { return !(fabsf(v) <= FLT_MAX); }

// ---------------------------------------------------------------- stats ----
struct Acc {
    double x2, e2, e, ftz, nz;
};

// binary32 sums over a handful of elements, folded into binary64
template <int N>
__device__ __forceinline__ void acc_add(Acc &a, const float y[N], const float xh[N])
{
    float sx = 0.f, se = 0.f, sb = 0.f;
    int f = 0, z = 0;
#pragma unroll
    for (int j = 0; j < N; ++j) {
        float d = y[j] - xh[j];
        sx = fmaf(y[j], y[j], sx);
        se = fmaf(d, d, se);
        sb -= d;
        int nzj = (y[j] != 0.0f);
        z += nzj;
        f += nzj & (xh[j] == 0.0f);
    }
    a.x2 += (double)sx;
    a.e2 += (double)se;
    a.e += (double)sb;
    a.ftz += (double)f;
    a.nz += (double)z;
}

__device__ __forceinline__ double warp_sum(double v)
{
    for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(kFull, v, o);
    return v;
}

// CTA reduction in a fixed order (lanes, then the warps' sums as one more
// warp reduction); thread 0 writes the CTA's record.
static __device__ __forceinline__ void write_partials(double *partials, const Acc &a, uint32_t rec)
{
    __shared__ double sh[5][32];
    double v[5] = {a.x2, a.e2, a.e, a.ftz, a.nz};
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int i = 0; i < 5; ++i) v[i] = warp_sum(v[i]);
    if (lane == 0)
#pragma unroll
        for (int i = 0; i < 5; ++i) sh[i][w] = v[i];
    __syncthreads();
    if (w == 0) {
        const int nw = (int)(blockDim.x >> 5);
        double *o = partials + (int64_t)rec * kPartialDoubles;
#pragma unroll
        for (int i = 0; i < 5; ++i) {
            const double t = warp_sum(lane < nw ? sh[i][lane] : 0.0);
            if (lane == 0) o[i] = t;
        }
        if (lane == 0) o[5] = o[6] = o[7] = 0.0;
    }
}

// Tensor scale of a launch: given, or s_T = amax / (max_elem * scale_max)
// from the tensor-amax word of the pre-pass (amax = 0 -> 1); CTA 0 stores it.
__device__ __forceinline__ float launch_tensor_scale(const QParams &p, bool first_cta)
{
    if (p.ts_mode == TS_NONE) return 1.0f;
    if (p.ts_mode == TS_GIVEN) return *p.tensor_scale;
    const float amax = __uint_as_float(__ldcg(p.amax_word));
    const float ts = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, __fmul_rn(p.ed.maxv, p.sd.ue_maxv));
    if (first_cta && threadIdx.x == 0) *p.tensor_scale = ts;
    return ts;
}
__device__ __forceinline__ float launch_tensor_scale(const QParams &p)
{
    return launch_tensor_scale(p, blockIdx.x == 0);
}

// The derived statistics of the summed records: MSE, R-MSE, QSNR Eq. (1),
// bias and the flush-to-zero share.
__device__ __forceinline__ void store_stats(double *stats, const double s[5], double count)
{
    const double x2 = s[0], e2 = s[1], e = s[2], ftz = s[3], nz = s[4];
    stats[0] = x2;
    stats[1] = e2;
    stats[2] = e;
    stats[3] = ftz;
    stats[4] = nz;
    const double mse = count > 0 ? e2 / count : 0.0;
    stats[5] = mse;
    stats[6] = sqrt(mse);
    stats[7] = (x2 == 0.0) ? __longlong_as_double(0x7ff8000000000000ll)
             : (e2 == 0.0) ? __longlong_as_double(0x7ff0000000000000ll)
                           : 10.0 * log10(x2 / e2);
    stats[8] = count > 0 ? e / count : 0.0;
    stats[9] = nz > 0 ? ftz / nz : 0.0;
    stats[10] = count;
    for (int k = 11; k < 16; ++k) stats[k] = 0.0;
}

// Epilogue of a quantizer launch (every thread of the CTA calls it): this
// CTA's record of the fidelity sums; then the last CTA to finish sums all
// records in a fixed order into the statistics, and clears the tensor-amax
// word and the ticket.
__device__ __forceinline__ void finish_launch(const QParams &p, const Acc &a, uint32_t cta, uint32_t ncta)
{
    if (p.partials) write_partials(p.partials, a, cta);
    if (!p.ticket) return;
    // thread 0 wrote the record; its release-acquire ticket orders the record
    // before the last CTA's reads of it (the barrier below extends that
    // order to the other threads of the last CTA)
    __shared__ unsigned s_last;
    if (threadIdx.x == 0) {
        unsigned prev;
        asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], 1;" : "=r"(prev) : "l"(p.ticket) : "memory");
        s_last = prev == ncta - 1;
    }
    __syncthreads();
    if (!s_last) return;
    if (p.partials) {
        // every thread of the last CTA takes a strided share of the records
        // (two in flight), then warps, then the warps' sums (a fixed order
        // for a given launch shape)
        __shared__ double red[5][32];
        double s[5] = {0, 0, 0, 0, 0};
        for (unsigned i0 = threadIdx.x; i0 < ncta; i0 += 2 * blockDim.x) {
            const unsigned i1 = i0 + blockDim.x;
            double r0[5], r1[5];
#pragma unroll
            for (int k = 0; k < 5; ++k) r0[k] = __ldcg(p.partials + (size_t)i0 * kPartialDoubles + k);
#pragma unroll
            for (int k = 0; k < 5; ++k)
                r1[k] = i1 < ncta ? __ldcg(p.partials + (size_t)i1 * kPartialDoubles + k) : 0.0;
#pragma unroll
            for (int k = 0; k < 5; ++k) s[k] += r0[k] + r1[k];
        }
#pragma unroll
        for (int k = 0; k < 5; ++k) s[k] = warp_sum(s[k]);
        const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
        if (lane == 0)
#pragma unroll
            for (int k = 0; k < 5; ++k) red[k][w] = s[k];
        __syncthreads();
        if (w == 0) {
            const int nw = (int)(blockDim.x >> 5);
            double t[5];
#pragma unroll
            for (int k = 0; k < 5; ++k) t[k] = warp_sum(lane < nw ? red[k][lane] : 0.0);
            if (lane == 0) store_stats(p.stats, t, p.count);
        }
    }
    if (threadIdx.x == 0) {
        if (p.ts_mode == TS_COMPUTE) *p.amax_word = 0u;
        *p.ticket = 0u;
    }
}
__device__ __forceinline__ void finish_launch(const QParams &p, const Acc &a)
{
    finish_launch(p, a, blockIdx.x, gridDim.x);
}

// x_hat of one element from its grid value q (the dequantization rule).
__device__ __forceinline__ float deq_value(const QParams &p, float q, const BlockScale &bs,
                                           float sm, float o, float sT)
{
    if (bs.nan) return __uint_as_float(0x7fc00000u);
    if (p.sd.fmt != S_E8M0 && p.sd.rule == R_NEAREST) return __fmul_rn(__fmul_rn(q, bs.deq), sT);
    float v = __fmul_rn(q, bs.deq);
    if (p.mbs) v = __fmul_rn(v, sm);
    if (p.asym) v = __fadd_rn(v, o);
    return v;
}

// A power of two P near 1 / a and 1 / P, both normal (a zero or subnormal a:
// 1, 1): y P is exact and below 2 in magnitude for |y| <= a, so the residuals
// of a flushed block (x_hat = 0) can be summed as (y P)^2 (1 / P)^2 without a
// binary32 overflow.
__device__ __forceinline__ float2 pow2_near_inv(float a)
{
    const uint32_t ef = (__float_as_uint(a) >> 23) & 0xffu;
    const uint32_t fe = ef == 0u ? 127u : (ef > 253u ? 253u : ef);
    return make_float2(__uint_as_float((254u - fe) << 23), __uint_as_float(fe << 23));
}

// Macro-block (MBS) scale code from the macro absmax and a non-finite flag:
// E4M3 nearest to m / (max_elem / 2^emax), m the mantissa of the absmax.
__device__ __forceinline__ uint32_t macro_code(const ElemDesc &ed, float amax, int bad)
{
    if (bad) return 0x7fu;
    if (amax == 0.0f) return e4m3_encode_pos(1.0f);
    int e;
    float m;
    frexp_exact(amax, e, m);
    return e4m3_encode_pos(__fdiv_rn(m, __fdiv_rn(ed.maxv, (float)(1 << ed.emax))));
}

// Same code as macro_code() without an IEEE division per call: d = max_elem /
// 2^emax (exact) and r_d = RN(1/d) are the launch's; m / d goes through
// div_by_recip (correctly rounded).  m is in [1, 2) and d in [1, 2), so the
// quotient lies in (1/2, 2), inside E4M3's normal range, where the hardware
// conversion rounds to nearest-even like e4m3_encode_pos().
__device__ __forceinline__ uint32_t macro_code_recip(float d, float r_d, float amax, int bad)
{
    if (bad) return 0x7fu;
    if (amax == 0.0f) return 0x38u;                 // E4M3 1.0
    int e;
    float m;
    frexp_exact(amax, e, m);
    const float x = div_by_recip(m, d, r_d);
    uint16_t h;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(0.0f), "f"(x));
    return h & 0xffu;
}

// ------------------------------------------------------------ rotation -----
// Butterfly stages of the Sylvester-ordered fast Walsh-Hadamard transform on
// a row chunk of 8 elements held by consecutive lanes (stride 8 and 16 are
// across lanes), then the binary32 1/sqrt(n) multiply.
__device__ __forceinline__ void hadamard_chunk8(float y[8], int n, int lane)
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


template <typename K>
static int grid_for(K kernel, int64_t work_warps, int threads = kThreads, size_t smem = 0)
{
    const int occ = cached_occupancy(reinterpret_cast<const void *>(kernel), threads, smem);
    int64_t g = (int64_t)device_sm_count() * occ;
    const int64_t need = (work_warps + (threads / 32) - 1) / (threads / 32);
    if (need < g) g = need;
    if (g < 1) g = 1;
    if (g > kMaxPartials) g = kMaxPartials;
    return (int)g;
}

}  // namespace mxk
