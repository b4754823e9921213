// sm_100a quantizer for the other element types and rounding modes of
// "Microscaling Data Formats for Deep Learning" as used in the training study
// summarised by fmread (Yang et al.: E2M1 / E3M0 / E2M3 / E3M2 / INT4 element
// types; round to nearest even, Ceil and stochastic rounding; asymmetric
// per-block offsets), row axis, blocks of 32, fed by the same TMA ring as the
// E2M1 nearest-even quantizer.
//
// The element type and the rounding mode are template parameters, so the
// grid arithmetic below folds to a few integer and binary32 operations per
// element.  The rounding of a scaled magnitude a to a minifloat grid with M
// mantissa bits and smallest normal exponent EMIN:
//   e   = max(exponent(a), EMIN)        the spacing of the grid at a is 2^(e-M)
//   as  = a * 2^(M-e)                    exact, in [0, 2^(M+1))
//   i   = floor(as), rem = as - i        both exact
//   lo  = code (e - EMIN) * 2^M + i      the grid point at or below a
// and the mode picks lo or lo + 1 (codes are monotone in the value, across
// the subnormal / normal boundary and across binades).  Integer grids are the
// same with a spacing of 1.  E2M1 / E2M3 / E3M2 nearest-even rounding uses the
// sm_100a conversion instructions instead.
#include "tma_ring.cuh"

namespace mxk {

namespace {

constexpr int kWaitFull = 31, kWaitEmpty = 32;   // status codes of the bounded waits

template <int ELEM>
struct GFmt;
template <> struct GFmt<E2M1> { static constexpr int M = 1, EMIN = 0, MAXC = 7, BITS = 4; static constexpr bool INT = false; };
template <> struct GFmt<E3M0> { static constexpr int M = 0, EMIN = -2, MAXC = 7, BITS = 4; static constexpr bool INT = false; };
template <> struct GFmt<E2M3> { static constexpr int M = 3, EMIN = 0, MAXC = 31, BITS = 6; static constexpr bool INT = false; };
template <> struct GFmt<E3M2> { static constexpr int M = 2, EMIN = -2, MAXC = 31, BITS = 6; static constexpr bool INT = false; };
template <> struct GFmt<INT4> { static constexpr int M = 0, EMIN = 0, MAXC = 7, BITS = 4; static constexpr bool INT = true; };

// largest magnitude (INT4 with an offset: unsigned 0..15)
template <int ELEM, bool ASYM>
__device__ __forceinline__ float max_value()
{
    if constexpr (ELEM == E2M1) return 6.0f;
    else if constexpr (ELEM == E3M0) return 16.0f;
    else if constexpr (ELEM == E2M3) return 7.5f;
    else if constexpr (ELEM == E3M2) return 28.0f;
    else return ASYM ? 15.0f : 7.0f;
}

// Magnitude code of a >= 0 (finite or +inf) under the rounding mode; qm gets
// the grid value.  u: the element's 32-bit random word (stochastic rounding).
template <int ELEM, int RD, bool ASYM>
__device__ __forceinline__ uint32_t round_grid(float a, uint32_t u, float &qm)
{
    using F = GFmt<ELEM>;
    // saturation without a branch: the maximum is a grid point, so a clamped
    // magnitude lands on it with a zero remainder under every mode (NaN and
    // +inf clamp to it as well)
    a = fminf(a, max_value<ELEM, ASYM>());
    float sc = 1.0f, isc = 1.0f;
    int cbase = 0;
    if constexpr (!F::INT) {
        const int e = max((int)(__float_as_uint(a) >> 23) - 127, F::EMIN);
        sc = __uint_as_float((uint32_t)(127 + F::M - e) << 23);     // 2^(M-e)
        isc = __uint_as_float((uint32_t)(127 - F::M + e) << 23);    // 2^(e-M)
        cbase = (e - F::EMIN) << F::M;
    }
    const float as = F::INT ? a : __fmul_rn(a, sc);
    const float t = __fadd_rz(as, 8388608.0f);                      // 2^23 + floor(as)
    const int i = (int)(__float_as_uint(t) - 0x4B000000u);
    const float lo = __fsub_rn(t, 8388608.0f);
    const int c0 = cbase + i;
    bool up;
    if constexpr (RD == RD_RTNE) {
        const float rem = __fsub_rn(as, lo);
        up = rem > 0.5f || (rem == 0.5f && (c0 & 1));
    } else if constexpr (RD == RD_CEIL) {
        up = as > lo;
    } else {
        // p = (a - lo) / (hi - lo), rounded as one binary32 quotient
        const float lo_u = F::INT ? lo : __fmul_rn(lo, isc);
        const float pr = F::INT ? __fsub_rn(a, lo_u) : __fmul_rn(__fsub_rn(a, lo_u), sc);
        up = __uint2float_rn(u >> 8) < __fmul_rn(pr, 16777216.0f);
    }
    const float qs = up ? __fadd_rn(lo, 1.0f) : lo;
    qm = F::INT ? qs : __fmul_rn(qs, isc);
    return (uint32_t)(c0 + (up ? 1 : 0));
}

// Element code of a scaled value v and its signed grid value.
template <int ELEM, int RD, bool ASYM>
__device__ __forceinline__ uint32_t encode_grid(float v, uint32_t u, float &q)
{
    using F = GFmt<ELEM>;
    if constexpr (F::INT && ASYM) {
        return round_grid<ELEM, RD, ASYM>(fmaxf(v, 0.0f), u, q);      // negatives (and NaN) -> 0
    } else {
        const uint32_t neg = __float_as_uint(v) >> 31;
        float m;
        const uint32_t c = round_grid<ELEM, RD, ASYM>(fabsf(v), u, m);
        q = neg ? -m : m;
        if constexpr (F::INT) return (neg ? (0u - c) : c) & 0xfu;
        else return (neg << (F::BITS - 1)) | c;
    }
}

// MSE-optimal E8M0 scale of a 32-element block (alpha > 0 finite): the
// exponent among k_floor and k_floor + 1 whose nearest-even codes leave the
// smaller squared error, 4^k sum (v - q)^2 with v = RN(y 2^-k); the two sums
// are accumulated in binary64 in element order (every term exact) and
// compared as S(k_floor) <= 4 S(k_floor + 1), ties to k_floor.
template <int ELEM>
__device__ __forceinline__ BlockScale mse_block_scale(const float y[32], float alpha, int emax)
{
    const uint32_t b = __float_as_uint(alpha);
    const int kf = (b >> 23) == 0 ? -1000 : (int)(b >> 23) - 127 - emax;
    const int k0 = min(max(kf, -127), 127), k1 = min(max(kf + 1, -127), 127);
    int k = k0;
    if (k1 != k0) {
        double sum[2];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const float inv = exp2i(-(c ? k1 : k0));
            double acc = 0.0;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float v = __fmul_rn(y[j], inv);
                float q;
                (void)encode_grid<ELEM, RD_RTNE, false>(v, 0u, q);
                const double d = (double)v - (double)q;
                acc = __dadd_rn(acc, __dmul_rn(d, d));
            }
            sum[c] = acc;
        }
        k = (sum[0] <= 4.0 * sum[1]) ? k0 : k1;
    }
    BlockScale r;
    r.code = (uint32_t)(k + 127);
    r.inv = exp2i(-k);
    r.deq = exp2i(k);
    r.zero = 0;
    r.nan = 0;
    return r;
}

// nearest-even conversion instructions: two binary32 values -> two codes
__device__ __forceinline__ uint32_t cvt_e2m3x2(float a0, float a1)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e2m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(a1), "f"(a0));
    return r;
}
__device__ __forceinline__ uint32_t cvt_e3m2x2(float a0, float a1)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e3m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(a1), "f"(a0));
    return r;
}
__device__ __forceinline__ float2 e2m3x2_values(uint32_t w16)
{
    uint32_t h;
    asm("cvt.rn.f16x2.e2m3x2 %0, %1;" : "=r"(h) : "h"((uint16_t)w16));
    return __half22float2(*reinterpret_cast<__half2 *>(&h));
}
__device__ __forceinline__ float2 e3m2x2_values(uint32_t w16)
{
    uint32_t h;
    asm("cvt.rn.f16x2.e3m2x2 %0, %1;" : "=r"(h) : "h"((uint16_t)w16));
    return __half22float2(*reinterpret_cast<__half2 *>(&h));
}
template <typename InT, int ELEM, int RD, bool ASYM>
__global__ void __launch_bounds__(kRingThreads, 2) k_quant_gen(const QParams p, const __grid_constant__ CUtensorMap tm)
{
    using F = GFmt<ELEM>;
    constexpr bool HW = RD == RD_RTNE && ELEM != E3M0 && ELEM != INT4;
    constexpr int NW = F::BITS == 4 ? 4 : 8;          // code words per 32 elements
    extern __shared__ uint8_t smem_raw[];
    const Ring<InT> ring(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t nch = (uint32_t)(p.rows * p.cols / 32);
    const uint32_t ntiles = (nch + kRingConsumers - 1) / kRingConsumers;
    pdl_trigger();
    if (threadIdx.x == 0) ring.init();
    pdl_wait();
    __syncthreads();

    Acc acc = {0, 0, 0, 0, 0};
    const bool stats = p.partials != nullptr;
    if (warp == kRingConsumers / 32) {
        if (lane == 0) ring.produce(&tm, ntiles, kWaitEmpty, blockIdx.x, gridDim.x);
    } else {
        const float sT = launch_tensor_scale(p);
        const bool nearest = p.sd.fmt != S_E8M0 && p.sd.rule == R_NEAREST;
        const int t = threadIdx.x;
        uint32_t it = 0;
        for (uint32_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
            if (!ring.acquire(it, kWaitFull)) break;
            float y[32];
            ring_read_chunk(ring.stage(it % RingCfg<InT>::kStages), t, static_cast<const InT *>(nullptr), y);
            ring.release(it);
            const uint32_t c = tile * kRingConsumers + t;
            const bool ok = c < nch;

            // block statistic (and offset)
            float a = 0.0f, mn = FLT_MAX, mx = -FLT_MAX;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                a = fmax_nan(a, fabsf(y[j]));
                if (ASYM) { mn = fminf(mn, y[j]); mx = fmaxf(mx, y[j]); }
            }
            const int bad = !(a <= FLT_MAX);
            float o = 0.0f;
            if (ASYM) {
                if (!bad) o = F::INT ? bf16_round(mn) : bf16_round(__fmul_rn(__fadd_rn(mx, mn), 0.5f));
                float ra = 0.0f;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float r = __fsub_rn(y[j], o);
                    ra = fmaxf(ra, F::INT ? r : fabsf(r));
                }
                a = ra;
            }
            const BlockScale bs = (!ASYM && p.sd.rule == R_MSE && !bad && a > 0.0f)
                                      ? mse_block_scale<ELEM>(y, a, p.ed.emax)
                                      : block_scale(p.ed, p.sd, bad ? 0.0f : a, bad, sT);
            // a flushed block (x_hat = 0, or o with an offset; not NaN): the
            // residuals are the (offset-removed) values themselves
            const bool flushed = bs.zero && !bs.nan;
            const float inv = flushed ? 1.0f : bs.inv;
            const float2 inv2 = make_float2(inv, inv);
            float deqT = bs.nan ? __uint_as_float(0x7fc00000u) : nearest ? __fmul_rn(bs.deq, sT) : bs.deq;
            if (flushed) deqT = 1.0f;

            // element codes and grid values; the statistics on the scaled
            // values: y - x_hat = deqT (v - q), exact for power-of-two scales
            // without an offset, within an ulp of y otherwise
            uint32_t words[NW];
#pragma unroll
            for (int w = 0; w < NW; ++w) words[w] = 0;
            float2 re2 = make_float2(0.f, 0.f), rb2 = re2, sx2 = re2;
            int qz = 0, xhz = 0;
            const float2 m1 = make_float2(-1.0f, -1.0f);
            // residual sums of one pair (v, q); q = 0 in a flushed block
            auto pair_stats = [&](float2 v, float q0, float q1, float x0, float x1) {
                if (bs.zero) { q0 = 0.0f; q1 = 0.0f; }
                const float2 d = __ffma2_rn(make_float2(q0, q1), m1, v);
                re2 = __ffma2_rn(d, d, re2);
                rb2 = __fadd2_rn(rb2, d);
                const float2 yv = make_float2(x0, x1);
                sx2 = __ffma2_rn(yv, yv, sx2);
                if (ASYM || nearest) {
                    // x_hat exactly as the dequantizer forms it (zero test)
                    float h0, h1;
                    if (bs.nan) { h0 = h1 = __uint_as_float(0x7fc00000u); }
                    else if (nearest) {
                        h0 = __fmul_rn(__fmul_rn(q0, bs.deq), sT);
                        h1 = __fmul_rn(__fmul_rn(q1, bs.deq), sT);
                    } else {
                        h0 = __fadd_rn(__fmul_rn(q0, bs.deq), o);
                        h1 = __fadd_rn(__fmul_rn(q1, bs.deq), o);
                    }
                    xhz += (h0 == 0.0f && x0 != 0.0f) + (h1 == 0.0f && x1 != 0.0f);
                } else {
                    qz += (q0 == 0.0f) + (q1 == 0.0f);
                }
            };
            if constexpr (HW && ELEM == E2M1) {
#pragma unroll
                for (int j = 0; j < 32; j += 8) {
                    float s8[8], q8[8];
#pragma unroll
                    for (int e = 0; e < 8; e += 2) {
                        const float2 r = ASYM ? make_float2(__fsub_rn(y[j + e], o), __fsub_rn(y[j + e + 1], o))
                                              : make_float2(y[j + e], y[j + e + 1]);
                        const float2 v = __fmul2_rn(r, inv2);
                        s8[e] = v.x;
                        s8[e + 1] = v.y;
                    }
                    words[j >> 3] = cvt_e2m1x8(s8);
                    if (stats) {
                        e2m1x8_values_alu(words[j >> 3], q8);
#pragma unroll
                        for (int e = 0; e < 8; e += 2)
                            pair_stats(make_float2(s8[e], s8[e + 1]), q8[e], q8[e + 1], y[j + e], y[j + e + 1]);
                    }
                }
            } else {
                uint4 rw = make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    const float2 r = ASYM ? make_float2(__fsub_rn(y[j], o), __fsub_rn(y[j + 1], o))
                                          : make_float2(y[j], y[j + 1]);
                    const float2 v = __fmul2_rn(r, inv2);
                    float2 qq;
                    if constexpr (HW) {
                        const uint32_t pair = ELEM == E2M3 ? cvt_e2m3x2(v.x, v.y) : cvt_e3m2x2(v.x, v.y);
                        if (stats) qq = ELEM == E2M3 ? e2m3x2_values(pair) : e3m2x2_values(pair);
                        words[j >> 2] |= pair << (8 * (j & 3));
                    } else {
                        if (RD == RD_SR && (j & 3) == 0) rw = element_words(p.seed, ((uint64_t)c * 32 + j) >> 2);
                        const uint32_t u0 = (j & 3) ? rw.z : rw.x, u1 = (j & 3) ? rw.w : rw.y;
                        const uint32_t c0 = encode_grid<ELEM, RD, ASYM>(v.x, u0, qq.x);
                        const uint32_t c1 = encode_grid<ELEM, RD, ASYM>(v.y, u1, qq.y);
                        if constexpr (F::BITS == 4) words[j >> 3] |= (c0 | (c1 << 4)) << (4 * (j & 7));
                        else words[j >> 2] |= (c0 | (c1 << 8)) << (8 * (j & 3));
                    }
                    if (stats) pair_stats(v, qq.x, qq.y, y[j], y[j + 1]);
                }
            }
            if (bs.zero) {
#pragma unroll
                for (int w = 0; w < NW; ++w) words[w] = 0;
            }

            if (ok) {
                if constexpr (F::BITS == 4) {
                    reinterpret_cast<uint4 *>(p.codes)[c] = make_uint4(words[0], words[1], words[2], words[3]);
                } else {
                    uint4 *dst = reinterpret_cast<uint4 *>(p.codes) + 2 * (size_t)c;
                    if (p.sf_gemm) {                // dense tensor-core operand form, 24 bytes
                        fp6_store_dense(static_cast<uint8_t *>(p.codes) + 24 * (size_t)c,
                                        fp6_group_pack(words[0], words[1], words[2], words[3]),
                                        fp6_group_pack(words[NW > 4 ? 4 : 0], words[NW > 4 ? 5 : 0],
                                                       words[NW > 4 ? 6 : 0], words[NW > 4 ? 7 : 0]));
                    } else {
                        dst[0] = make_uint4(words[0], words[1], words[2], words[3]);
                        dst[NW > 4 ? 1 : 0] = make_uint4(words[NW > 4 ? 4 : 0], words[NW > 4 ? 5 : 0],
                                                         words[NW > 4 ? 6 : 0], words[NW > 4 ? 7 : 0]);
                    }
                }
                if (p.sf_gemm) {
                    const uint32_t S = (uint32_t)(p.cols / 32), r = c / S;
                    p.scales[sf_chunk_index(r, c - r * S, S)] = (uint8_t)bs.code;
                } else {
                    p.scales[c] = (uint8_t)bs.code;
                }
                if (ASYM) p.offsets[c] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
            }

            if (stats && ok) {
                const double X = (double)deqT;
                acc.e2 += (double)(re2.x + re2.y) * X * X;
                acc.e -= (double)(rb2.x + rb2.y) * X;
                acc.x2 += (double)(sx2.x + sx2.y);
                // exact zeros (rare): the block's minimum magnitude is zero
                int xz = 0;
                if (absmin<32>(y) == 0.0f)
#pragma unroll
                    for (int j = 0; j < 32; ++j) xz += (y[j] == 0.0f);
                acc.nz += (double)(32 - xz);
                if (ASYM || nearest) acc.ftz += (double)xhz;
                else if (!bs.nan) acc.ftz += (double)(qz - xz);
            }
        }
    }
    finish_launch(p, acc);
}

template <typename InT, int ELEM, int RD, bool ASYM>
int launch_gen_k(const QParams &p, cudaStream_t st, int *grid_out)
{
    const uint64_t nch = (uint64_t)(p.rows * p.cols / 32);
    CUtensorMap tm;
    if (ring_map<InT>(&tm, p.x, nch) != 0) return -1;
    auto k = k_quant_gen<InT, ELEM, RD, ASYM>;
    const unsigned g = ring_grid(reinterpret_cast<const void *>(k), RingCfg<InT>::kSmem, nch);
    const cudaError_t e = launch_pdl(k, g, kRingThreads, RingCfg<InT>::kSmem, st, p, tm);
    *grid_out = (int)g;
    return e == cudaSuccess ? 0 : -1;
}

template <typename InT, int ELEM, bool ASYM>
int launch_gen_r(const QParams &p, cudaStream_t st, int *grid_out)
{
    switch (p.round_mode) {
    case RD_RTNE: return launch_gen_k<InT, ELEM, RD_RTNE, ASYM>(p, st, grid_out);
    case RD_CEIL: return launch_gen_k<InT, ELEM, RD_CEIL, ASYM>(p, st, grid_out);
    case RD_SR: return launch_gen_k<InT, ELEM, RD_SR, ASYM>(p, st, grid_out);
    default: return -1;
    }
}

template <typename InT, bool ASYM>
int launch_gen_e(const QParams &p, cudaStream_t st, int *grid_out)
{
    switch (p.ed.elem) {
    case E2M1: return launch_gen_r<InT, E2M1, ASYM>(p, st, grid_out);
    case E3M0: return launch_gen_r<InT, E3M0, ASYM>(p, st, grid_out);
    case E2M3: return launch_gen_r<InT, E2M3, ASYM>(p, st, grid_out);
    case E3M2: return launch_gen_r<InT, E3M2, ASYM>(p, st, grid_out);
    case INT4: return launch_gen_r<InT, INT4, ASYM>(p, st, grid_out);
    default: return -1;
    }
}

}  // namespace

// Row axis, blocks of 32, no rotation, macro scale or rotated output.
int launch_quantize_gen(const QParams &p, int in_fp32, cudaStream_t st, int *grid_out)
{
    if (in_fp32) return p.asym ? launch_gen_e<float, true>(p, st, grid_out) : launch_gen_e<float, false>(p, st, grid_out);
    return p.asym ? launch_gen_e<__nv_bfloat16, true>(p, st, grid_out)
                  : launch_gen_e<__nv_bfloat16, false>(p, st, grid_out);
}

int take_status_gen(cudaStream_t st, int *v) { return take_ring_status(st, v); }

}  // namespace mxk
