// Device-side number formats, scale rules, rounding and the counter-based
// generator of the sm_100a quantizer kernels.
//
// Element formats ("Unveiling the Potential of Quantization with MXFP4",
// Sec.2/Sec.3; fmread summary of Yang et al., design-choice study):
//   E2M1 {0,.5,1,1.5,2,3,4,6}, E3M0 {0, 2^-2..2^4}, E2M3 / E3M2 (OCP FP6),
//   INT4 (-7..7 two's complement, or 0..15 with a block offset).
// Scale formats: E8M0 (power of two), UE4M3 (min 2^-9, max 448), UE5M3
//   (min 2^-17, max 1.75*2^16) ("Is Finer Better?", theoretical framework and
//   core contributions).
//
// All decisions that yield an integer code are single IEEE binary32
// operations with explicit round-to-nearest intrinsics (no contraction).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mxk {

enum { E2M1 = 0, E3M0 = 1, E2M3 = 2, E3M2 = 3, INT4 = 4 };
enum { S_E8M0 = 0, S_UE4M3 = 1, S_UE5M3 = 2 };
enum { R_FLOOR = 0, R_CEIL = 1, R_OAS = 2, R_NEAREST = 3, R_MSE = 4 };
enum { RD_RTNE = 0, RD_CEIL = 1, RD_SR = 2 };
enum { AX_ROW = 0, AX_COL = 1, AX_2D = 2 };
enum { TS_NONE = 0, TS_COMPUTE = 1, TS_GIVEN = 2 };

// Element grid, as a minifloat (mbits mantissa bits, exponent bias) or an
// integer grid; filled on the host per launch.
struct ElemDesc {
    int elem;
    int asym;
    int is_int;
    int mbits;       // FP only
    int bias;        // FP only
    int code_bits;   // 4 or 6
    int max_code;    // largest magnitude code
    int emax;        // exponent of the largest power of two <= maxv
    float maxv;      // largest magnitude
    float sub_lim;   // FP: 2^(1-bias), start of the normal range
    float sub_inv_q; // FP: 1 / subnormal spacing = 2^(bias+mbits-1)
};

// Scale rule of a launch.
struct ScaleDesc {
    int fmt;        // S_*
    int rule;       // R_*
    float tau;      // OAS threshold
    int kmin, kmax; // clamp of power-of-two exponents
    // unsigned minifloat (UE4M3 / UE5M3) parameters
    int ue_bias, ue_max_code, ue_nan_code;
    float ue_maxv;
};

__device__ __forceinline__ float bits2f(uint32_t b) { return __uint_as_float(b); }

// 2^k for k in [-149, 127]
__device__ __forceinline__ float exp2i(int k)
{
    return k >= -126 ? bits2f((uint32_t)(k + 127) << 23) : bits2f(1u << (k + 149));
}

// alpha = m 2^e, m in [1,2), alpha > 0 finite
__device__ __forceinline__ void frexp_exact(float alpha, int &e, float &m)
{
    uint32_t b = __float_as_uint(alpha);
    uint32_t ef = (b >> 23) & 0xffu;
    uint32_t frac = b & 0x7fffffu;
    if (ef != 0) {
        e = (int)ef - 127;
        m = bits2f(0x3f800000u | frac);
    } else {
        int p = 31 - __clz(frac);            // position of the leading one
        e = p - 149;                          // alpha = frac * 2^-149
        m = bits2f(0x3f800000u | ((frac << (23 - p)) & 0x7fffffu));
    }
}

// ---------------------------------------------------------------- elements --
// Value of a magnitude code.
__device__ __forceinline__ float mag_value(const ElemDesc &d, int c)
{
    if (d.is_int) return (float)c;
    int e = c >> d.mbits;
    int m = c & ((1 << d.mbits) - 1);
    if (e == 0) return __fdiv_rn((float)m, d.sub_inv_q);   // m * 2^(1-bias-mbits), exact
    return bits2f(((uint32_t)(e - d.bias + 127) << 23) | ((uint32_t)m << (23 - d.mbits)));
}

// Largest code whose value is <= a, for a finite, 0 <= a < maxv.
__device__ __forceinline__ int floor_code(const ElemDesc &d, float a)
{
    if (d.is_int) return (int)a;                               // truncation
    if (a < d.sub_lim) return (int)__fmul_rn(a, d.sub_inv_q);  // exact scaling
    return (int)(__float_as_uint(a) >> (23 - d.mbits)) - ((127 - d.bias) << d.mbits);
}

// Magnitude code of a >= 0 under the rounding mode; `u` is the element's
// 32-bit random word (stochastic rounding only).
__device__ __forceinline__ int round_mag(const ElemDesc &d, int mode, float a, uint32_t u)
{
    if (!(a < d.maxv)) return d.max_code;
    int i = floor_code(d, a);
    float lo = mag_value(d, i);
    if (a == lo) return i;
    float hi = mag_value(d, i + 1);
    if (mode == RD_RTNE) {
        float mid = __fmul_rn(__fadd_rn(lo, hi), 0.5f);
        if (a < mid) return i;
        if (a > mid) return i + 1;
        return (i & 1) ? i + 1 : i;
    }
    if (mode == RD_CEIL) return i + 1;
    float p = __fdiv_rn(__fsub_rn(a, lo), __fsub_rn(hi, lo));
    float thr = __fmul_rn(p, 16777216.0f);
    return (__uint2float_rn(u >> 8) < thr) ? i + 1 : i;
}

// Code of a scaled value v, and (through qv) its grid value with sign.
__device__ __forceinline__ uint32_t encode_elem(const ElemDesc &d, int mode, float v, uint32_t u,
                                                float &qv)
{
    if (d.is_int && d.asym) {
        if (!(v > 0.0f)) { qv = 0.0f; return 0u; }
        int m = round_mag(d, mode, v, u);
        qv = (float)m;
        return (uint32_t)m;
    }
    uint32_t neg = __float_as_uint(v) >> 31;
    int m = round_mag(d, mode, fabsf(v), u);
    if (d.is_int) {
        int q = neg ? -m : m;
        qv = (float)q;
        return (uint32_t)q & 0xfu;
    }
    float mv = mag_value(d, m);
    qv = neg ? -mv : mv;
    return (neg << (d.code_bits - 1)) | (uint32_t)m;
}

// Grid value of a code with sign.
__device__ __forceinline__ float decode_elem(const ElemDesc &d, uint32_t code)
{
    if (d.is_int) {
        if (d.asym) return (float)(code & 0xfu);
        int q = (int)(code & 0xfu);
        return (float)(q >= 8 ? q - 16 : q);
    }
    uint32_t sbit = 1u << (d.code_bits - 1);
    float mv = mag_value(d, (int)(code & (sbit - 1)));
    return (code & sbit) ? -mv : mv;
}

// FP6 codes of 32 elements, one per byte (4 per word, code j in byte j % 4
// of word j / 4), <-> the dense tensor-core operand form: each 16 codes
// packed into 12 bytes (code i at bits [6i, 6i + 6) of the little-endian
// 96-bit group; the fourth word of the uint4 is unused), a 32-code chunk in
// 24 consecutive bytes.  The GEMM's TMA expands every 12-byte group to the
// 16-byte shared-memory form of kind::mxf8f6f4 (4 zero bytes added).
__device__ __forceinline__ uint4 fp6_group_pack(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3)
{
    uint32_t c[16];
    const uint32_t w[4] = {w0, w1, w2, w3};
#pragma unroll
    for (int i = 0; i < 16; ++i) c[i] = (w[i >> 2] >> (8 * (i & 3))) & 0x3fu;
    uint4 r;
    r.x = c[0] | (c[1] << 6) | (c[2] << 12) | (c[3] << 18) | (c[4] << 24) | (c[5] << 30);
    r.y = (c[5] >> 2) | (c[6] << 4) | (c[7] << 10) | (c[8] << 16) | (c[9] << 22) | (c[10] << 28);
    r.z = (c[10] >> 4) | (c[11] << 2) | (c[12] << 8) | (c[13] << 14) | (c[14] << 20) | (c[15] << 26);
    r.w = 0u;
    return r;
}
// 24 bytes of a chunk's two groups at dst (8-byte aligned), and back
__device__ __forceinline__ void fp6_store_dense(uint8_t *dst, uint4 g0, uint4 g1)
{
    uint2 *d = reinterpret_cast<uint2 *>(dst);
    d[0] = make_uint2(g0.x, g0.y);
    d[1] = make_uint2(g0.z, g1.x);
    d[2] = make_uint2(g1.y, g1.z);
}
__device__ __forceinline__ void fp6_load_dense(const uint8_t *src, uint4 &g0, uint4 &g1)
{
    const uint2 *s = reinterpret_cast<const uint2 *>(src);
    const uint2 a = s[0], b = s[1], c = s[2];
    g0 = make_uint4(a.x, a.y, b.x, 0u);
    g1 = make_uint4(b.y, c.x, c.y, 0u);
}
__device__ __forceinline__ void fp6_group_unpack(uint4 g, uint32_t w[4])
{
    const uint64_t lo = (uint64_t)g.x | ((uint64_t)g.y << 32);
    const uint64_t hi = (uint64_t)g.y | ((uint64_t)g.z << 32);
#pragma unroll
    for (int k = 0; k < 4; ++k) w[k] = 0u;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int bit = 6 * i;
        const uint32_t c = bit < 32 + 26 ? (uint32_t)(lo >> bit) & 0x3fu : (uint32_t)(hi >> (bit - 32)) & 0x3fu;
        w[i >> 2] |= c << (8 * (i & 3));
    }
}

// E2M1 fast path: eight binary32 values -> eight nibbles, element j in bits
// [4j, 4j+4); round to nearest even with saturation at +-6 (sm_100a cvt).
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float v[8])
{
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return r;
}

// Eight E2M1 nibbles -> their grid values (exact through f16).
__device__ __forceinline__ void e2m1x8_values(uint32_t packed, float out[8])
{
    uint32_t h0, h1, h2, h3;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h0), "=r"(h1), "=r"(h2), "=r"(h3) : "r"(packed));
    uint32_t h[4] = {h0, h1, h2, h3};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __half2 t = *reinterpret_cast<__half2 *>(&h[i]);
        float2 f = __half22float2(t);
        out[2 * i] = f.x;
        out[2 * i + 1] = f.y;
    }
}

// Eight E2M1 nibbles -> their grid values without the conversion
// instruction: the magnitude bits moved to bits 22..24 form the binary32
// denormal m * 2^-127, so one exact multiply by 2^126 gives the grid value
// (0, 0.5, 1, 1.5, 2, 3, 4, 6); the nibble's sign bit becomes bit 31.
__device__ __forceinline__ void e2m1x8_values_alu(uint32_t packed, float out[8])
{
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
        const uint32_t t0 = packed >> (4 * j), t1 = packed >> (4 * j + 4);
        const float2 d = make_float2(bits2f(((t0 & 7u) << 22) | ((t0 & 8u) << 28)),
                                     bits2f(((t1 & 7u) << 22) | ((t1 & 8u) << 28)));
        const float2 v = __fmul2_rn(d, make_float2(0x1p126f, 0x1p126f));
        out[j] = v.x;
        out[j + 1] = v.y;
    }
}

// Eight E2M1 nibbles -> four f16x2 words of their grid values (exact).
__device__ __forceinline__ void e2m1x8_halves(uint32_t packed, uint32_t h[4])
{
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3]) : "r"(packed));
}

// (s0 - q0, s1 - q1) in binary32, q the two halves of an f16x2 word: one
// mixed-precision multiply-add per lane (q * -1 + s, a single rounding).
__device__ __forceinline__ float2 sub_f16x2_from(float s0, float s1, uint32_t qh)
{
    float d0, d1;
    asm("{\n\t.reg .f16 q0, q1, m1;\n\t"
        "mov.b32 {q0, q1}, %2;\n\t"
        "mov.b16 m1, 0xBC00;\n\t"
        "fma.rn.f32.f16 %0, q0, m1, %3;\n\t"
        "fma.rn.f32.f16 %1, q1, m1, %4;\n\t}"
        : "=f"(d0), "=f"(d1) : "r"(qh), "f"(s0), "f"(s1));
    return make_float2(d0, d1);
}

// E2M1 code -> value (sign-magnitude nibble)
__device__ __forceinline__ float e2m1_value(uint32_t code)
{
    uint32_t mag = code & 7u;
    uint32_t b = mag >= 2u ? ((((mag >> 1) + 126u) << 23) | ((mag & 1u) << 22))
                           : (mag ? 0x3f000000u : 0u);
    return bits2f(b | ((code & 8u) << 28));
}

// ------------------------------------------------------------------ scales --
// Unsigned minifloat with 3 mantissa bits: value of a code.
__device__ __forceinline__ float ue_value(const ScaleDesc &s, uint32_t c)
{
    if ((int)c >= s.ue_nan_code) return __uint_as_float(0x7fc00000u);
    uint32_t e = c >> 3, m = c & 7u;
    if (e == 0) return __fmul_rn((float)m, exp2i(1 - s.ue_bias - 3));
    return bits2f(((e - (uint32_t)s.ue_bias + 127u) << 23) | (m << 20));
}

// Round x to the unsigned minifloat: nearest, ties to even, saturating at the
// largest finite code; x <= 0 -> 0, NaN -> NaN code.
__device__ __forceinline__ uint32_t ue_encode_rtne(const ScaleDesc &s, float x)
{
    if (x != x) return (uint32_t)s.ue_nan_code;
    if (!(x > 0.0f)) return 0u;
    if (x >= s.ue_maxv) return (uint32_t)s.ue_max_code;
    int emin = 1 - s.ue_bias;                  // exponent of the first normal binade
    int e; float m;
    frexp_exact(x, e, m);
    int code;
    if (e < emin) {
        // subnormal range: multiples of 2^(emin-3)
        if (e < emin - 3 - 2) return 0u;       // below a quarter step: rounds to zero
        float t = __fmul_rn(x, exp2i(3 - emin));   // exact unless far below range
        code = __float2int_rn(t);                  // 0..8 (8 = first normal)
    } else {
        float t = __fmul_rn(m, 8.0f);              // 8..16, exact
        int n = __float2int_rn(t);                 // ties to even
        code = ((e - emin + 1) << 3) + (n - 8);
    }
    if (code > s.ue_max_code) code = s.ue_max_code;
    return (uint32_t)code;
}

// UE4M3 nearest-even code of x through the sm_100a E4M3 conversion (round to
// nearest even, saturating at 448); x <= 0 -> 0, NaN -> 0x7F.
__device__ __forceinline__ uint32_t ue4m3_encode_hw(float x)
{
    if (x != x) return 0x7fu;
    if (!(x > 0.0f)) return 0u;
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
    return (uint32_t)(r & 0xffu);
}

// Code of 2^k in the unsigned minifloat (k within [kmin, kmax]).
__device__ __forceinline__ uint32_t ue_encode_pow2(const ScaleDesc &s, int k)
{
    int emin = 1 - s.ue_bias;
    if (k >= emin) return (uint32_t)((k - emin + 1) << 3);
    return 1u << (k - (emin - 3));
}

// Power-of-two block exponent for amax alpha > 0 (finite) under the rule.
__device__ __forceinline__ int pow2_exponent(const ElemDesc &d, const ScaleDesc &s, float alpha)
{
    int e; float m;
    frexp_exact(alpha, e, m);
    int k = e - d.emax;
    float ratio = __fmul_rn(m, (float)(1 << d.emax));
    if (s.rule == R_CEIL) k += (ratio > d.maxv) ? 1 : 0;
    else if (s.rule == R_OAS) k += (ratio > s.tau) ? 1 : 0;
    return k;
}

struct BlockScale {
    uint32_t code;  // stored byte
    float inv;      // multiplier applied to the elements
    float deq;      // dequantization factor: 2^k, or s_b (times s_T applied separately)
    int zero;       // all element codes are zero
    int nan;        // NaN scale
};

// Shared scale of a block from its statistic alpha (>= 0) and whether it
// holds a non-finite value.  sT: per-tensor scale (1 without).
__device__ __forceinline__ BlockScale block_scale(const ElemDesc &d, const ScaleDesc &s,
                                                  float alpha, int nonfinite, float sT)
{
    BlockScale r;
    r.zero = 0; r.nan = 0; r.inv = 0.0f; r.deq = 0.0f;
    if (s.fmt == S_E8M0) {
        if (nonfinite) { r.code = 0xffu; r.zero = 1; r.nan = 1; return r; }
        if (alpha == 0.0f) { r.code = 0u; r.zero = 1; r.deq = exp2i(-127); return r; }
        int k = pow2_exponent(d, s, alpha);
        k = max(-127, min(127, k));
        r.code = (uint32_t)(k + 127);
        r.inv = exp2i(-k);
        r.deq = exp2i(k);
        return r;
    }
    if (nonfinite) { r.code = (uint32_t)s.ue_nan_code; r.zero = 1; r.nan = 1; return r; }
    if (s.rule == R_NEAREST) {
        float sb_real = __fdiv_rn(__fdiv_rn(alpha, d.maxv), sT);
        r.code = (s.fmt == S_UE4M3) ? ue4m3_encode_hw(sb_real) : ue_encode_rtne(s, sb_real);
        float sb = ue_value(s, r.code);
        r.deq = sb;
        if (sb != sb) { r.zero = 1; r.nan = 1; return r; }
        float dd = __fmul_rn(sb, sT);
        r.inv = __fdiv_rn(1.0f, dd);
        if (sb == 0.0f || !(r.inv < __uint_as_float(0x7f800000u))) r.zero = 1;
        return r;
    }
    int k;
    if (alpha == 0.0f) { k = s.kmin; r.zero = 1; }
    else k = pow2_exponent(d, s, alpha);
    k = max(s.kmin, min(s.kmax, k));
    r.code = ue_encode_pow2(s, k);
    r.inv = exp2i(-k);
    r.deq = exp2i(k);
    return r;
}

// Correctly rounded a / b from y = RN(1/b) (b and y normal): q0 = RN(a y)
// is within 2 ulp of a/b; one residual correction, r = a - b q evaluated by
// the fused multiply-add, brings it within 1 ulp, and a second one is
// Markstein's theorem (Markstein, IBM J. Res. Develop. 34(1), 1990): with y
// within half an ulp of 1/b and q within one ulp of a/b, RN(q + (a - b q) y)
// is RN(a/b).  Quotients outside the normal range take the IEEE division.
__device__ __forceinline__ float div_by_recip(float a, float b, float y)
{
    const float q0 = __fmul_rn(a, y);
    if (!(q0 >= 0x1p-124f && q0 <= 0x1p124f)) return __fdiv_rn(a, b);
    const float q1 = __fmaf_rn(__fmaf_rn(-q0, b, a), y, q0);
    return __fmaf_rn(__fmaf_rn(-q1, b, a), y, q1);
}

// Per-launch constants of the nearest (UE4M3 / UE5M3) block scale.
struct NearScale {
    float maxv, r_max;      // largest element magnitude and RN(1 / maxv)
    float sT, r_T;          // tensor scale and RN(1 / sT); r_T = 0: IEEE division
    float c;                // UE4M3 shortcut: RN(1 / RN(maxv sT)), or 0 (no shortcut)
    const float2 *tab;      // per scale code: {RN(s_b sT), RN(1 / RN(s_b sT))}; NaN code: {NaN, 0}
};

// Same codes as block_scale() with a nearest rule: the two quotients of
// s_b = RTNE((alpha / max) / s_T) through div_by_recip; the dequantization
// factor s_b s_T (in deq) and the element multiplier from the launch's table.
// A zero block: s_b = 0 (1/0 = +inf).
//
// UE4M3 shortcut: v = RN(alpha c) with c = RN(1 / RN(maxv sT)) is within
// 5 ulp of the two-quotient value w (each of the three roundings in v and the
// two in w is at most half an ulp, relative 2^-24, and the ulp of a binade
// is at least 2^-24 of its values), so when v lies in E4M3's normal range and
// more than 6 ulp from a rounding midpoint of E4M3 (mantissa bits below the
// top 3 equal to 1000...0, i.e. low 20 bits 0x80000), v and w round to the
// same code; every other block takes the two quotients.
__device__ __forceinline__ BlockScale near_block_scale(const ScaleDesc &s, const NearScale &ns, float alpha,
                                                       int nonfinite)
{
    BlockScale r;
    uint32_t code;
    const float v = __fmul_rn(alpha, ns.c);
    const uint32_t mid = (__float_as_uint(v) & 0xfffffu) - 0x80000u + 6u;
    if (s.fmt == S_UE4M3 && v >= 0x1p-6f && v <= 0x1p100f && mid > 12u) {
        uint16_t h;
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(0.0f), "f"(v));
        code = h & 0xffu;
    } else {
        const float q1 = div_by_recip(alpha, ns.maxv, ns.r_max);
        const float sb_real = ns.sT == 1.0f ? q1
                            : ns.r_T != 0.0f ? div_by_recip(q1, ns.sT, ns.r_T) : __fdiv_rn(q1, ns.sT);
        code = (s.fmt == S_UE4M3) ? ue4m3_encode_hw(sb_real) : ue_encode_rtne(s, sb_real);
    }
    r.code = nonfinite ? (uint32_t)s.ue_nan_code : code;
    const float2 t = ns.tab[r.code];
    r.deq = t.x;
    r.inv = t.y;
    r.nan = r.code >= (uint32_t)s.ue_nan_code;
    r.zero = r.nan || !(t.y < __uint_as_float(0x7f800000u));
    return r;
}

// E8M0 scale of a block without branches: k = e - emax (+1 when the
// significand times 2^emax exceeds thr: the ceil rule with thr = max element,
// OAS with thr = tau, floor with thr = +inf), clamped to [-127, 127]; a zero
// or subnormal alpha lands on k = -127, the code of the zero block.
// thr_m = thr / 2^emax.
__device__ __forceinline__ BlockScale e8m0_block_scale(float alpha, int nonfinite, int emax, float thr_m)
{
    const uint32_t b = __float_as_uint(alpha);
    const int ef = (int)(b >> 23);
    const float m = __uint_as_float((b & 0x7fffffu) | 0x3f800000u);
    int k = ef - 127 - emax + (m > thr_m ? 1 : 0);
    k = ef == 0 ? -127 : min(max(k, -127), 127);
    BlockScale r;
    r.code = nonfinite ? 0xffu : (uint32_t)(k + 127);
    r.zero = nonfinite || alpha == 0.0f;
    r.nan = nonfinite;
    r.inv = __uint_as_float(k <= 126 ? (uint32_t)(127 - k) << 23 : 0x00400000u);
    r.deq = __uint_as_float(k >= -126 ? (uint32_t)(k + 127) << 23 : 0x00400000u);
    return r;
}

// thr_m of e8m0_block_scale for a launch
__device__ __forceinline__ float e8m0_threshold(const ElemDesc &d, const ScaleDesc &s)
{
    const float thr = s.rule == R_CEIL ? d.maxv : s.rule == R_OAS ? s.tau : __uint_as_float(0x7f800000u);
    return __fmul_rn(thr, __uint_as_float((uint32_t)(127 - d.emax) << 23));
}

// E4M3 (positive) for the MBS macro scale: nearest-even code of x in
// [2^-6, 448), and the value of a code.
__device__ __forceinline__ uint32_t e4m3_encode_pos(float x)
{
    ScaleDesc s;
    s.ue_bias = 7; s.ue_max_code = 0x7e; s.ue_nan_code = 0x7f; s.ue_maxv = 448.0f;
    return ue_encode_rtne(s, x);
}
__device__ __forceinline__ float e4m3_value(uint32_t c)
{
    ScaleDesc s;
    s.ue_bias = 7; s.ue_max_code = 0x7e; s.ue_nan_code = 0x7f; s.ue_maxv = 448.0f;
    return ue_value(s, c & 0x7fu);
}

// ----------------------------------------------------- Philox4x32-10 --------
// Salmon et al., SC'11: ten rounds of two 32x32 -> 64-bit products, key bumped
// by the Weyl constants between rounds.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint2 k)
{
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        if (r) { k.x += 0x9E3779B9u; k.y += 0xBB67AE85u; }
        uint32_t lo0 = 0xD2511F53u * c.x, hi0 = __umulhi(0xD2511F53u, c.x);
        uint32_t lo1 = 0xCD9E8D57u * c.z, hi1 = __umulhi(0xCD9E8D57u, c.z);
        c = make_uint4(hi1 ^ c.y ^ k.x, lo1, hi0 ^ c.w ^ k.y, lo0);
    }
    return c;
}

// Four random words for the elements 4q .. 4q+3 (row-major logical index).
__device__ __forceinline__ uint4 element_words(uint64_t seed, uint64_t q)
{
    return philox4x32_10(make_uint4((uint32_t)q, (uint32_t)(q >> 32), 0u, 0u),
                         make_uint2((uint32_t)seed, (uint32_t)(seed >> 32)));
}

__device__ __forceinline__ uint32_t word_of(const uint4 &w, int j)
{
    return j == 0 ? w.x : j == 1 ? w.y : j == 2 ? w.z : w.w;
}

// binary32 -> bf16 -> binary32 (round to nearest even), zero made +0
__device__ __forceinline__ float bf16_round(float v)
{
    return __fadd_rn(__bfloat162float(__float2bfloat16_rn(v)), 0.0f);
}

// Byte of scale j of row r in the tcgen05 chunk layout: 512-byte chunks of
// 128 rows x 4 scales, row r at (r % 32) * 16 + ((r / 32) % 4) * 4 (S scales
// per row, S % 4 == 0).
__device__ __forceinline__ int64_t sf_chunk_index(int64_t r, int64_t j, int64_t S)
{
    return (((r >> 7) * (S >> 2) + (j >> 2)) << 9) + ((r & 31) << 4) + (((r >> 5) & 3) << 2) + (j & 3);
}

// binary32 1/sqrt(n) of the normalised rotation
__device__ __forceinline__ float hadamard_scale(int n)
{
    return n == 16 ? 0.25f : 0.17677669227123260498046875f;
}

}  // namespace mxk
