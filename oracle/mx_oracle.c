/*
 * mx_oracle.c -- plain, slow, scalar CPU oracle for microscaling (MX) block
 * quantization.  TEST INFRASTRUCTURE ONLY: it exists so that the tests, the
 * smoke check and the CPU-baseline leg of the benchmark can check the CUDA
 * path against an independent implementation.  Nothing in the product path
 * may call it.
 *
 * It shares no code, header, table or constant with the CUDA library.  It is
 * written straight from the definitions on the source pages:
 *
 *   [MXFP4-OAS]  "Unveiling the Potential of Quantization with MXFP4:
 *                 Strategies for Quantization Error Reduction" (Qiita
 *                 explainer and nubint review): Sec.2 FP4 formats (MXFP4 =
 *                 E2M1 + E8M0 per 32, NVFP4 = E2M1 + E4M3 per 16 + FP32
 *                 per-tensor scale), Sec.3 QSNR Eq. (1) and Eq. (2), the
 *                 12x E2M1 range and the ~20% error in (4,6), Sec.4 block
 *                 granularity (E4M3 used as power-of-two scales), OAS and
 *                 MBS (1x128 macro blocks).
 *   [FINER]      "Is Finer Better? The Limits of Microscaling Formats in
 *                 Large Language Models": UE4M3 minimum 2^-9, UE5M3
 *                 minimum 2^-17, per-tensor FP32 scale (UE4M3-S).
 *   [BRIDGING]   "Bridging the Gap Between Promise and Performance for
 *                 Microscaling FP4 Quantization": sec. 2.1/2.2 block-wise
 *                 Hadamard rotation before quantization, MSE-optimised
 *                 grids (alternating global / group scales).
 *   [MX-TRAIN]   fmread summary of Yang et al., "MX quantization for LLM
 *                 training" (ARITH 2025): element types E2M1/E3M0/INT4,
 *                 RTNE / Ceil / stochastic rounding, asymmetric scaling,
 *                 row-wise / column-wise / 2D blocks, R-MSE.
 *
 * Where the pages leave a step open the reading taken is marked (READING)
 * and is listed in the design notes of the repository.
 *
 * Precision: every decision that produces an integer code (scale exponent,
 * element code) is taken with single IEEE binary32 operations in the order
 * written here (compile with -ffp-contract=off, no fast-math), except the
 * MSE rules, which compare block squared errors summed in binary64 in
 * element order; the fidelity reductions are accumulated in binary64.
 *
 * Parity status of each function is stated beside it: "pinned" functions are
 * checked by the CPU tests against values fixed by the pages or by
 * mathematics; "parity unpinned" marks the parts only checked against
 * invariants.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* enumerations (numbering is the interface convention of the library)      */
/* ------------------------------------------------------------------------ */
enum { E_E2M1 = 0, E_E3M0 = 1, E_E2M3 = 2, E_E3M2 = 3, E_INT4 = 4 };
enum { S_E8M0 = 0, S_UE4M3 = 1, S_UE5M3 = 2 };
enum { R_FLOOR = 0, R_CEIL = 1, R_OAS = 2, R_NEAREST = 3, R_MSE = 4 };
enum { RD_RTNE = 0, RD_CEIL = 1, RD_SR = 2 };
enum { AX_ROW = 0, AX_COL = 1, AX_2D = 2 };
enum { DT_BF16 = 0, DT_FP32 = 1 };
enum { TS_NONE = 0, TS_COMPUTE = 1, TS_GIVEN = 2 };

typedef struct {
    int32_t elem, scale_fmt, rule;
    float oas_tau;
    int32_t block, axis, round_mode, asymmetric;
    int32_t tensor_scale, macro_block, hadamard, reserved;
    uint64_t seed;
} orc_cfg;

/* ------------------------------------------------------------------------ */
/* bit helpers                                                              */
/* ------------------------------------------------------------------------ */
static float f_from_bits(uint32_t b) { float f; memcpy(&f, &b, 4); return f; }
static uint32_t bits_of_f(float f) { uint32_t b; memcpy(&b, &f, 4); return b; }

float orc_bf16_to_f32(uint16_t h) { return f_from_bits(((uint32_t)h) << 16); }

/* fp32 -> bf16, round to nearest even (finite inputs). */
uint16_t orc_f32_to_bf16(float f)
{
    uint32_t b = bits_of_f(f);
    if ((b & 0x7f800000u) == 0x7f800000u) return (uint16_t)((b >> 16) | ((b & 0xffff) ? 0x40 : 0));
    uint32_t lsb = (b >> 16) & 1u;
    b += 0x7fffu + lsb;
    return (uint16_t)(b >> 16);
}

/* 2^k as a binary32 value for k in [-149, 127] (subnormal below -126). */
static float pow2f(int k)
{
    if (k >= -126) return f_from_bits((uint32_t)(k + 127) << 23);
    return f_from_bits(1u << (k + 149));
}

/* alpha = m * 2^e with m in [1,2), read off the bits (alpha > 0, finite). */
static void split_pow2(float alpha, int *e, float *m)
{
    uint32_t b = bits_of_f(alpha);
    int ef = (int)((b >> 23) & 0xff);
    uint32_t frac = b & 0x7fffffu;
    if (ef == 0) {                       /* subnormal: normalise the fraction */
        int msb = 31;
        while (!((frac >> msb) & 1u)) msb--;
        *e = msb - 149;
        uint32_t f2 = (frac << (23 - msb)) & 0x7fffffu;
        *m = f_from_bits((127u << 23) | f2);
    } else {
        *e = ef - 127;
        *m = f_from_bits((127u << 23) | frac);
    }
}

/* ------------------------------------------------------------------------ */
/* element grids                                                            */
/* [MXFP4-OAS] Sec.2 / Sec.3: E2M1 magnitudes {0,0.5,1,1.5,2,3,4,6}.         */
/* [MX-TRAIN]: E3M0 and INT4 element types; MXFP6 (E2M3/E3M2) configs.      */
/* (READING) E3M0 = exponent field f in 0..7, f=0 -> 0, else 2^(f-3).       */
/* (READING) E2M3 / E3M2 grids follow the OCP MX FP6 element definitions.   */
/* (READING) INT4 symmetric = integers -7..7 in a two's-complement nibble;  */
/*           INT4 asymmetric = unsigned 0..15 plus a per-block offset.      */
/* ------------------------------------------------------------------------ */
static const float E2M1_MAG[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

typedef struct {
    int nmag;          /* number of magnitude codes */
    int bits;          /* code width in bits (4 or 6) */
    int emax;          /* exponent of the largest power of two <= max */
    float mag[32];     /* non-negative grid, ascending */
    int is_int;        /* INT4 */
} grid_t;

static void make_grid(int elem, int asym, grid_t *g)
{
    memset(g, 0, sizeof(*g));
    switch (elem) {
    case E_E2M1:
        g->nmag = 8; g->bits = 4; g->emax = 2;
        for (int i = 0; i < 8; i++) g->mag[i] = E2M1_MAG[i];
        break;
    case E_E3M0:
        g->nmag = 8; g->bits = 4; g->emax = 4;
        g->mag[0] = 0.0f;
        for (int f = 1; f < 8; f++) g->mag[f] = pow2f(f - 3);
        break;
    case E_E2M3:   /* 2 exponent bits (bias 1), 3 mantissa bits */
        g->nmag = 32; g->bits = 6; g->emax = 2;
        for (int c = 0; c < 32; c++) {
            int e = c >> 3, m = c & 7;
            g->mag[c] = (e == 0) ? (float)m / 8.0f : (1.0f + (float)m / 8.0f) * pow2f(e - 1);
        }
        break;
    case E_E3M2:   /* 3 exponent bits (bias 3), 2 mantissa bits */
        g->nmag = 32; g->bits = 6; g->emax = 4;
        for (int c = 0; c < 32; c++) {
            int e = c >> 2, m = c & 3;
            g->mag[c] = (e == 0) ? (float)m / 16.0f : (1.0f + (float)m / 4.0f) * pow2f(e - 3);
        }
        break;
    case E_INT4:
        g->is_int = 1; g->bits = 4;
        if (asym) { g->nmag = 16; g->emax = 3; }
        else      { g->nmag = 8;  g->emax = 2; }
        for (int i = 0; i < g->nmag; i++) g->mag[i] = (float)i;
        break;
    }
}

static float grid_max(const grid_t *g) { return g->mag[g->nmag - 1]; }

/* Round a magnitude a >= 0 (may be +inf) to a magnitude code.
 * RTNE: nearest grid point, ties to the even code; saturate at the maximum.
 * CEIL: (READING) next grid point up in magnitude, saturating.
 * SR:   round up with probability (a-lo)/(hi-lo): up iff float(u>>8) <
 *       p * 2^24, u the element's 32-bit Philox word.
 * Pinned: tie list and brute force against the printed E2M1 grid. */
static int round_mag(const grid_t *g, int mode, float a, uint32_t u)
{
    int top = g->nmag - 1;
    if (!(a < g->mag[top])) return top;          /* saturate (also +inf) */
    int i = 0;
    while (i + 1 <= top && g->mag[i + 1] <= a) i++;   /* mag[i] <= a < mag[i+1] */
    float lo = g->mag[i], hi = g->mag[i + 1];
    if (a == lo) return i;
    if (mode == RD_RTNE) {
        float mid = (lo + hi) * 0.5f;            /* exact: small dyadic values */
        if (a < mid) return i;
        if (a > mid) return i + 1;
        return (i % 2 == 0) ? i : i + 1;
    } else if (mode == RD_CEIL) {
        return i + 1;
    } else {
        float p = (a - lo) / (hi - lo);          /* exact (Sterbenz, /2^j) */
        float thr = p * 16777216.0f;
        float r = (float)(u >> 8);
        return (r < thr) ? i + 1 : i;
    }
}

/* Element code from a scaled value v.  FP formats: sign-magnitude with the
 * sign bit kept for a zero magnitude (READING).  INT4 symmetric: two's
 * complement nibble.  INT4 asymmetric: unsigned, negatives clamp to 0. */
static uint8_t encode_elem(const grid_t *g, int asym, int mode, float v, uint32_t u)
{
    if (g->is_int && asym) {
        if (!(v > 0.0f)) return 0;
        return (uint8_t)round_mag(g, mode, v, u);
    }
    int neg = signbit(v) ? 1 : 0;
    float a = fabsf(v);
    int m = round_mag(g, mode, a, u);
    if (g->is_int) {
        int q = neg ? -m : m;
        return (uint8_t)(q & 0xf);
    }
    return (uint8_t)((neg << (g->bits - 1)) | m);
}

/* Grid value of an element code. */
static float decode_elem(const grid_t *g, int asym, uint8_t code)
{
    if (g->is_int) {
        if (asym) return (float)(code & 0xf);
        int q = (int)(code & 0xf);
        if (q >= 8) q -= 16;
        return (float)q;
    }
    int sbit = 1 << (g->bits - 1);
    float mag = g->mag[code & (sbit - 1)];
    return (code & sbit) ? -mag : mag;
}

/* Exposed for the exhaustive tests. */
uint8_t orc_encode_elem(int elem, int asym, int mode, float v, uint32_t u)
{
    grid_t g; make_grid(elem, asym, &g);
    return encode_elem(&g, asym, mode, v, u);
}

float orc_decode_elem(int elem, int asym, uint8_t code)
{
    grid_t g; make_grid(elem, asym, &g);
    return decode_elem(&g, asym, code);
}

/* ------------------------------------------------------------------------ */
/* scale formats                                                            */
/* E8M0: 2^(code-127), 0xFF = NaN  ([MXFP4-OAS] Sec.2: exponent-only scale). */
/* UE4M3: 4 exponent bits (bias 7), 3 mantissa bits, min 2^-9, max 448,     */
/*        0x7F = NaN ([FINER]).                                             */
/* UE5M3: 5 exponent bits (bias 15), 3 mantissa bits, min 2^-17 ([FINER]);  */
/*        (READING) all-ones 0xFF = NaN, so max = 1.75 * 2^16.              */
/* ------------------------------------------------------------------------ */
typedef struct { int ebits, mbits, bias, nan_code, max_code; } ufmt_t;

static ufmt_t ufmt(int fmt)
{
    ufmt_t u;
    if (fmt == S_UE4M3) { u.ebits = 4; u.mbits = 3; u.bias = 7;  u.nan_code = 0x7f; u.max_code = 0x7e; }
    else                { u.ebits = 5; u.mbits = 3; u.bias = 15; u.nan_code = 0xff; u.max_code = 0xfe; }
    return u;
}

float orc_scale_decode(int fmt, uint8_t code)
{
    if (fmt == S_E8M0) {
        if (code == 0xff) return NAN;
        return pow2f((int)code - 127);
    }
    ufmt_t u = ufmt(fmt);
    if (code == u.nan_code) return NAN;
    if (code > u.nan_code) return NAN;    /* UE4M3 uses 7 bits */
    int e = code >> u.mbits, m = code & ((1 << u.mbits) - 1);
    float frac = (float)m / (float)(1 << u.mbits);
    if (e == 0) return frac * pow2f(1 - u.bias);
    return (1.0f + frac) * pow2f(e - u.bias);
}

/* Round a positive binary32 value to the nearest unsigned-minifloat code,
 * ties to the even code, saturating at the largest finite code; values <= 0
 * map to code 0, NaN to the NaN code.  Plain search over every finite code:
 * the distances |x - value(code)| are exact in binary64. */
uint8_t orc_scale_encode_nearest(int fmt, float x)
{
    ufmt_t u = ufmt(fmt);
    if (isnan(x)) return (uint8_t)u.nan_code;
    if (!(x > 0.0f)) return 0;
    double xd = (double)x;
    double vmax = (double)orc_scale_decode(fmt, (uint8_t)u.max_code);
    if (xd >= vmax) return (uint8_t)u.max_code;
    int best = 0;
    double bestd = fabs(xd - 0.0);
    for (int c = 1; c <= u.max_code; c++) {
        double d = fabs(xd - (double)orc_scale_decode(fmt, (uint8_t)c));
        if (d < bestd || (d == bestd && (c % 2 == 0))) { best = c; bestd = d; }
    }
    return (uint8_t)best;
}

/* E4M3 (the macro-block scale of MBS), positive values only: same encoding
 * as UE4M3 for a cleared sign bit. */
static uint8_t e4m3_encode_pos(float x) { return orc_scale_encode_nearest(S_UE4M3, x); }
static float e4m3_decode(uint8_t c) { return orc_scale_decode(S_UE4M3, (uint8_t)(c & 0x7f)); }

/* ------------------------------------------------------------------------ */
/* Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as  */
/* easy as 1, 2, 3", SC'11): round = two 32x32->64 multiplies, key bumped   */
/* by the Weyl constants between rounds.  Pinned: known-answer vectors.     */
/* ------------------------------------------------------------------------ */
void orc_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4])
{
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int r = 0; r < 10; r++) {
        if (r > 0) { k0 += 0x9E3779B9u; k1 += 0xBB67AE85u; }
        uint64_t p0 = (uint64_t)0xD2511F53u * (uint64_t)c0;
        uint64_t p1 = (uint64_t)0xCD9E8D57u * (uint64_t)c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0, n1 = lo1, n2 = hi0 ^ c3 ^ k1, n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* Random word of logical element i (row-major index r*cols+c): counter =
 * (lo32(i/4), hi32(i/4), 0, 0), key = (lo32(seed), hi32(seed)), word i%4. */
static uint32_t elem_random(uint64_t seed, uint64_t i)
{
    uint64_t q = i >> 2;
    uint32_t ctr[4] = {(uint32_t)q, (uint32_t)(q >> 32), 0u, 0u};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t out[4];
    orc_philox4x32_10(ctr, key, out);
    return out[i & 3];
}

/* ------------------------------------------------------------------------ */
/* Block Hadamard rotation ([BRIDGING] 2.1-2.2).  (READING) Sylvester       */
/* ordering; in-place fast Walsh-Hadamard stages h = 1, 2, 4, ..., each a   */
/* butterfly (a, b) -> (a + b, a - b) in binary32, then every output is     */
/* multiplied by binary32(1/sqrt(n)).  Pinned: H H^T = n I on unit vectors, */
/* and against an explicit matrix-vector product.                          */
/* ------------------------------------------------------------------------ */
static float hadamard_norm(int n)
{
    if (n == 16) return 0.25f;
    if (n == 32) return 0.176776692271232604980f;   /* binary32 nearest to 1/sqrt(32) */
    return (float)(1.0 / sqrt((double)n));
}

void orc_fwht(int n, float *v, int normalise)
{
    for (int h = 1; h < n; h <<= 1) {
        for (int i = 0; i < n; i += 2 * h) {
            for (int j = i; j < i + h; j++) {
                float a = v[j], b = v[j + h];
                v[j] = a + b;
                v[j + h] = a - b;
            }
        }
    }
    if (normalise) {
        float c = hadamard_norm(n);
        for (int j = 0; j < n; j++) v[j] = v[j] * c;
    }
}

/* ------------------------------------------------------------------------ */
/* Block geometry                                                           */
/* ------------------------------------------------------------------------ */
/* number of blocks and the element (r, c) of position t in block b */
static int64_t n_blocks(int axis, int B, int64_t rows, int64_t cols)
{
    if (axis == AX_ROW) return rows * (cols / B);
    if (axis == AX_COL) return (rows / B) * cols;
    return (rows / B) * (cols / B);
}

static int block_len(int axis, int B) { return axis == AX_2D ? B * B : B; }

static void block_elem(int axis, int B, int64_t rows, int64_t cols, int64_t b, int t,
                       int64_t *r, int64_t *c)
{
    (void)rows;
    if (axis == AX_ROW) {
        int64_t nb = cols / B;
        *r = b / nb; *c = (b % nb) * B + t;
    } else if (axis == AX_COL) {
        *r = (b / cols) * B + t; *c = b % cols;
    } else {
        int64_t nb = cols / B;
        *r = (b / nb) * B + t / B; *c = (b % nb) * B + t % B;
    }
}

/* Macro-block (MBS) index of element (r, c): 1 x 128 along the block axis;
 * the 2D layout takes the row direction (READING). */
static int64_t macro_index(int axis, int64_t rows, int64_t cols, int64_t r, int64_t c)
{
    (void)rows;
    if (axis == AX_COL) return (r / 128) * cols + c;
    return r * (cols / 128) + c / 128;
}

static int64_t n_macro(int axis, int64_t rows, int64_t cols)
{
    if (axis == AX_COL) return (rows / 128) * cols;
    return rows * (cols / 128);
}

/* ------------------------------------------------------------------------ */
/* Load input, apply the optional rotation -> reference tensor y (binary32) */
/* ------------------------------------------------------------------------ */
static void load_input(const void *x, int dtype, int64_t n, float *out)
{
    if (dtype == DT_BF16) {
        const uint16_t *h = (const uint16_t *)x;
        for (int64_t i = 0; i < n; i++) out[i] = orc_bf16_to_f32(h[i]);
    } else {
        memcpy(out, x, (size_t)n * sizeof(float));
    }
}

/* rotate groups of n along the block axis (row direction for 2D) */
static void rotate(int axis, int n, int64_t rows, int64_t cols, float *y)
{
    float buf[32];
    if (axis == AX_COL) {
        for (int64_t c = 0; c < cols; c++)
            for (int64_t g = 0; g < rows / n; g++) {
                for (int t = 0; t < n; t++) buf[t] = y[(g * n + t) * cols + c];
                orc_fwht(n, buf, 1);
                for (int t = 0; t < n; t++) y[(g * n + t) * cols + c] = buf[t];
            }
    } else {
        for (int64_t r = 0; r < rows; r++)
            for (int64_t g = 0; g < cols / n; g++) {
                float *p = y + r * cols + g * n;
                for (int t = 0; t < n; t++) buf[t] = p[t];
                orc_fwht(n, buf, 1);
                for (int t = 0; t < n; t++) p[t] = buf[t];
            }
    }
}

/* ------------------------------------------------------------------------ */
/* Shared-scale rules for power-of-two scales                               */
/* [MXFP4-OAS] Sec.4 OAS; (READING) floor = OCP rule 2^(floor(log2 a)-emax);*/
/* ceil = smallest k with a <= max * 2^k (the "no overflow" rule);          */
/* OAS(tau) = floor exponent, plus one when a / 2^k_floor > tau.            */
/* Pinned: exhaustive single-value blocks for floor; ceil never saturates;  */
/* OAS(6) == ceil and OAS(8) == floor for E2M1.                             */
/* ------------------------------------------------------------------------ */
static int pow2_exponent(const grid_t *g, int rule, float tau, float alpha)
{
    int e; float m;
    split_pow2(alpha, &e, &m);
    int k = e - g->emax;
    float ratio = m * pow2f(g->emax);     /* alpha / 2^k_floor, exact */
    if (rule == R_CEIL) { if (ratio > grid_max(g)) k += 1; }
    else if (rule == R_OAS) { if (ratio > tau) k += 1; }
    return k;
}

/* (READING) MSE-optimal power-of-two scale (a per-block MSE-min scale     */
/* search, the third follow-up after the core path): among the E8M0         */
/* exponents k_floor and k_floor + 1 (clamped), the one whose block of     */
/* nearest-even element codes has the smaller squared error; ties keep     */
/* k_floor.  The error of exponent k is 4^k sum (v_t - q_t)^2 with          */
/* v_t = binary32(r_t 2^-k) and q_t its grid value, so the two sums are    */
/* compared as S(k_floor) against 4 S(k_floor + 1), each accumulated in    */
/* binary64 in element order (every term is exact there).                  */
/* Pinned: brute force against an independent grid rounding (tests), and  */
/* the closed forms of constant blocks.                                    */
static int mse_exponent(const grid_t *g, int asym, const float *res, int L, float alpha)
{
    int kf = pow2_exponent(g, R_FLOOR, 0.0f, alpha);
    int k0 = kf < -127 ? -127 : kf > 127 ? 127 : kf;
    int k1 = kf + 1 < -127 ? -127 : kf + 1 > 127 ? 127 : kf + 1;
    if (k0 == k1) return k0;
    double sum[2];
    for (int c = 0; c < 2; c++) {
        float inv = pow2f(-(c ? k1 : k0));
        double acc = 0.0;
        for (int t = 0; t < L; t++) {
            float v = res[t] * inv;
            float q = decode_elem(g, asym, encode_elem(g, asym, RD_RTNE, v, 0u));
            double d = (double)v - (double)q;
            acc += d * d;
        }
        sum[c] = acc;
    }
    return (sum[0] <= 4.0 * sum[1]) ? k0 : k1;
}

/* (READING) MSE-optimal UE4M3 / UE5M3 block scale for a given tensor scale */
/* s_T ([BRIDGING] sec. 2.2: MSE-optimised grids, the group-scale half of   */
/* the alternating optimisation): the pages name the objective, not the     */
/* search, so the plainest reading is the exact argmin over every finite    */
/* scale code c of the block's squared error                                */
/*   SSE(c) = sum_t (x_t - x_hat_t)^2,  x_hat_t = (q_t s_c) s_T,             */
/* q_t the nearest-even grid value of x_t * RN(1 / RN(s_c s_T)) (the        */
/* element rule of the nearest-scale formats), a block of zeros when        */
/* s_c = 0 or the reciprocal overflows.  Each SSE is accumulated in binary64 */
/* in element order (x_t - x_hat_t rounded once to binary64, squared, added) */
/* and ties keep the lower code.  Pinned: never above the nearest rule's    */
/* block error; single values q s reproduced exactly (tests).               */
static uint8_t mse_ue_code(const grid_t *g, int fmt, const float *res, int L, float sT, double *sse_out)
{
    ufmt_t u = ufmt(fmt);
    int best = 0;
    double best_sse = INFINITY;
    for (int c = 0; c < u.nan_code; c++) {
        float sb = orc_scale_decode(fmt, (uint8_t)c);
        float d = sb * sT;
        float inv = 1.0f / d;
        int zero = (sb == 0.0f) || !(inv < INFINITY);
        double acc = 0.0;
        for (int t = 0; t < L; t++) {
            float xh = 0.0f;
            if (!zero) {
                float v = res[t] * inv;
                float q = decode_elem(g, 0, encode_elem(g, 0, RD_RTNE, v, 0u));
                xh = (q * sb) * sT;
            }
            double e = (double)res[t] - (double)xh;
            acc += e * e;
        }
        if (acc < best_sse) { best_sse = acc; best = c; }
    }
    if (sse_out) *sse_out = best_sse;
    return (uint8_t)best;
}

/* (READING) the global-scale half ([BRIDGING] sec. 2.2: alternating        */
/* optimisation of the global and the group scales).  Starting from the     */
/* amax rule's s_T, each round takes the group step above for every block,  */
/* then, with the codes and element values u_t = q_t s_c held fixed, the    */
/* s_T minimising sum (x_t - u_t s_T)^2: the least-squares factor           */
/* s_T = sum x_t u_t / sum u_t^2 (binary64 sums in block and element order,  */
/* every product exact there; rounded once to binary32; kept when it is not */
/* a positive finite number).  The pages give no round count: MSE_ROUNDS.   */
/* Blocks with a non-finite value take no part.  The squared error after    */
/* each group step cannot rise from one round to the next (up to binary32   */
/* rounding of x_hat and s_T): the pin of the tests.                         */
#define MSE_ROUNDS 4

static float mse_grid_alternate(const grid_t *g, int fmt, int axis, int B, const float *y, int64_t rows,
                                int64_t cols, float sT, int rounds, float *sT_trace, double *sse_trace)
{
    const int64_t nb = n_blocks(axis, B, rows, cols);
    const int L = block_len(axis, B);
    float *res = (float *)malloc((size_t)L * sizeof(float));
    if (!res) return NAN;
    for (int it = 0; ; it++) {
        double num = 0.0, den = 0.0, sse = 0.0;
        for (int64_t b = 0; b < nb; b++) {
            int nonfinite = 0;
            for (int t = 0; t < L; t++) {
                int64_t r, c;
                block_elem(axis, B, rows, cols, b, t, &r, &c);
                res[t] = y[r * cols + c];
                if (!isfinite(res[t])) nonfinite = 1;
            }
            if (nonfinite) continue;
            double bsse;
            uint8_t code = mse_ue_code(g, fmt, res, L, sT, &bsse);
            sse += bsse;
            float sb = orc_scale_decode(fmt, code);
            float inv = 1.0f / (sb * sT);
            if (sb == 0.0f || !(inv < INFINITY)) continue;
            for (int t = 0; t < L; t++) {
                float q = decode_elem(g, 0, encode_elem(g, 0, RD_RTNE, res[t] * inv, 0u));
                float u = q * sb;
                num += (double)res[t] * (double)u;
                den += (double)u * (double)u;
            }
        }
        if (sT_trace) sT_trace[it] = sT;
        if (sse_trace) sse_trace[it] = sse;
        if (it == rounds) break;
        if (den > 0.0) {
            float s = (float)(num / den);
            if (s > 0.0f && isfinite(s)) sT = s;
        }
    }
    free(res);
    return sT;
}

/* ------------------------------------------------------------------------ */
/* Quantize                                                                 */
/* ------------------------------------------------------------------------ */
/* Tensor scale ([MXFP4-OAS] Sec.2 NVFP4's FP32 per-tensor scale; [FINER]):  */
/* (READING) s_T = amax_T / (max_elem * max_scale), amax_T over |y| with    */
/* NaN skipped; amax_T = 0 gives s_T = 1.                                   */
float orc_tensor_scale(int elem, int scale_fmt, const float *y, int64_t n)
{
    grid_t g; make_grid(elem, 0, &g);
    float amax = 0.0f;
    for (int64_t i = 0; i < n; i++) {
        float a = fabsf(y[i]);
        if (a > amax) amax = a;
    }
    if (amax == 0.0f) return 1.0f;
    float smax = orc_scale_decode(scale_fmt, (uint8_t)ufmt(scale_fmt).max_code);
    float denom = grid_max(&g) * smax;
    return amax / denom;
}

/*
 * orc_quantize: reference tensor y (input, rotated if cfg->hadamard), one
 * element code per element (unpacked), one scale code per block, optional
 * macro scale codes and bf16 offsets.  x_hat comes from orc_dequantize.
 * Returns 0, or -1 on an unsupported configuration.
 */
int orc_quantize(const orc_cfg *cfg, const void *x, int dtype, int64_t rows, int64_t cols,
                 uint8_t *codes, uint8_t *scales, float *tensor_scale,
                 uint8_t *macro, uint16_t *offsets, float *y_out)
{
    const int B = cfg->block;
    const int64_t n = rows * cols;
    const int asym = cfg->asymmetric;
    grid_t g; make_grid(cfg->elem, asym, &g);

    float *y = (float *)malloc((size_t)n * sizeof(float));
    float *yq = (float *)malloc((size_t)n * sizeof(float));   /* input of the block rule */
    if (!y || !yq) { free(y); free(yq); return -1; }
    load_input(x, dtype, n, y);
    if (cfg->hadamard) rotate(cfg->axis, cfg->hadamard, rows, cols, y);
    if (y_out) memcpy(y_out, y, (size_t)n * sizeof(float));
    memcpy(yq, y, (size_t)n * sizeof(float));

    /* per-tensor scale */
    float sT = 1.0f;
    if (cfg->tensor_scale == TS_COMPUTE) {
        sT = orc_tensor_scale(cfg->elem, cfg->scale_fmt, y, n);
        /* MSE rule with a nearest-scale format: the alternating optimisation */
        if (cfg->rule == R_MSE && cfg->scale_fmt != S_E8M0)
            sT = mse_grid_alternate(&g, cfg->scale_fmt, cfg->axis, B, y, rows, cols, sT, MSE_ROUNDS, NULL, NULL);
        if (tensor_scale) *tensor_scale = sT;
    } else if (cfg->tensor_scale == TS_GIVEN) {
        sT = *tensor_scale;
    }

    /* Macro Block Scaling ([MXFP4-OAS] Sec.4 MBS, Fig. 5).  (READING) per
     * 1x128 macro block S_M = E4M3_rtne(m_M / c) with m_M the mantissa of the
     * macro-block absmax in [1,2) and c = max_elem / 2^emax (1.5 for E2M1),
     * so the macro maximum lands on the top grid point; S_M = 1 for an
     * all-zero macro block; y' = y * (1 / S_M).  Parity unpinned beyond the
     * invariants in the tests (no formula on the pages). */
    float *sm_val = NULL;
    if (cfg->macro_block) {
        int64_t nm = n_macro(cfg->axis, rows, cols);
        float *amaxm = (float *)calloc((size_t)nm, sizeof(float));
        uint8_t *nanm = (uint8_t *)calloc((size_t)nm, 1);
        sm_val = (float *)malloc((size_t)nm * sizeof(float));
        for (int64_t r = 0; r < rows; r++)
            for (int64_t c = 0; c < cols; c++) {
                int64_t mi = macro_index(cfg->axis, rows, cols, r, c);
                float v = y[r * cols + c];
                if (!isfinite(v)) nanm[mi] = 1;
                else if (fabsf(v) > amaxm[mi]) amaxm[mi] = fabsf(v);
            }
        float cdiv = grid_max(&g) / pow2f(g.emax);
        for (int64_t mi = 0; mi < nm; mi++) {
            uint8_t code;
            if (nanm[mi]) code = 0x7f;
            else if (amaxm[mi] == 0.0f) code = e4m3_encode_pos(1.0f);
            else {
                int e; float m;
                split_pow2(amaxm[mi], &e, &m);
                code = e4m3_encode_pos(m / cdiv);
            }
            macro[mi] = code;
            sm_val[mi] = e4m3_decode(code);
        }
        for (int64_t r = 0; r < rows; r++)
            for (int64_t c = 0; c < cols; c++) {
                float s = sm_val[macro_index(cfg->axis, rows, cols, r, c)];
                float inv = 1.0f / s;
                yq[r * cols + c] = y[r * cols + c] * inv;
            }
        free(amaxm); free(nanm);
    }

    const int64_t nb = n_blocks(cfg->axis, B, rows, cols);
    const int L = block_len(cfg->axis, B);
    int64_t *ri = (int64_t *)malloc((size_t)L * sizeof(int64_t));
    int64_t *ci = (int64_t *)malloc((size_t)L * sizeof(int64_t));
    float *res = (float *)malloc((size_t)L * sizeof(float));

    for (int64_t b = 0; b < nb; b++) {
        int nonfinite = 0;
        for (int t = 0; t < L; t++) {
            block_elem(cfg->axis, B, rows, cols, b, t, &ri[t], &ci[t]);
            if (!isfinite(yq[ri[t] * cols + ci[t]])) nonfinite = 1;
        }
        /* offset (asymmetric scaling, [MX-TRAIN]); (READING) INT4: o =
         * bf16(min); FP elements: o = bf16((max + min) / 2); a zero offset is
         * +0. */
        float o = 0.0f;
        if (asym && !nonfinite) {
            float mn = yq[ri[0] * cols + ci[0]], mx = mn;
            for (int t = 1; t < L; t++) {
                float v = yq[ri[t] * cols + ci[t]];
                if (v < mn) mn = v;
                if (v > mx) mx = v;
            }
            if (g.is_int) o = orc_bf16_to_f32(orc_f32_to_bf16(mn));
            else          o = orc_bf16_to_f32(orc_f32_to_bf16((mx + mn) * 0.5f));
            o = o + 0.0f;
            for (int t = 0; t < L; t++) res[t] = yq[ri[t] * cols + ci[t]] - o;
        } else {
            for (int t = 0; t < L; t++) res[t] = yq[ri[t] * cols + ci[t]];
        }
        if (offsets) offsets[b] = asym ? orc_f32_to_bf16(o) : 0;

        /* block statistic alpha: absmax of the residuals; for INT4 with an
         * offset the range max(r) (READING: smallest k with max - o <= 15 2^k
         * under the ceil rule) */
        float alpha = 0.0f;
        if (!nonfinite) {
            for (int t = 0; t < L; t++) {
                float a = (g.is_int && asym) ? res[t] : fabsf(res[t]);
                if (a > alpha) alpha = a;
            }
        }

        /* shared scale */
        uint8_t scode;
        float inv = 0.0f;          /* multiplier applied to the residuals */
        int zero_block = 0;
        if (cfg->scale_fmt == S_E8M0) {
            if (nonfinite) { scode = 0xff; zero_block = 1; }
            else if (alpha == 0.0f) { scode = 0; zero_block = 1; }
            else {
                int k = (cfg->rule == R_MSE) ? mse_exponent(&g, asym, res, L, alpha)
                                             : pow2_exponent(&g, cfg->rule, cfg->oas_tau, alpha);
                if (k < -127) k = -127;
                if (k > 127) k = 127;
                scode = (uint8_t)(k + 127);
                inv = pow2f(-k);
            }
        } else if (cfg->rule == R_NEAREST || cfg->rule == R_MSE) {
            ufmt_t u = ufmt(cfg->scale_fmt);
            if (nonfinite) { scode = (uint8_t)u.nan_code; zero_block = 1; }
            else {
                float sb_real = (alpha / grid_max(&g)) / sT;
                scode = cfg->rule == R_MSE ? mse_ue_code(&g, cfg->scale_fmt, res, L, sT, NULL)
                                           : orc_scale_encode_nearest(cfg->scale_fmt, sb_real);
                float sb = orc_scale_decode(cfg->scale_fmt, scode);
                if (isnan(sb)) zero_block = 1;
                else {
                    float d = sb * sT;
                    inv = 1.0f / d;
                    if (sb == 0.0f || !(inv < INFINITY)) zero_block = 1;
                }
            }
        } else {
            /* power-of-two scales stored in UE4M3 / UE5M3 ([MXFP4-OAS] Sec.4,
             * E4M3 used as power-of-two "E4M0" scales); exponent clamped to the
             * format's powers of two */
            ufmt_t u = ufmt(cfg->scale_fmt);
            int kmin = 1 - u.bias - u.mbits;                 /* smallest subnormal */
            int kmax = ((u.max_code >> u.mbits)) - u.bias;   /* largest binade */
            if (nonfinite) { scode = (uint8_t)u.nan_code; zero_block = 1; }
            else {
                int k;
                if (alpha == 0.0f) { k = kmin; zero_block = 1; }
                else k = pow2_exponent(&g, cfg->rule, cfg->oas_tau, alpha);
                if (k < kmin) k = kmin;
                if (k > kmax) k = kmax;
                scode = orc_scale_encode_nearest(cfg->scale_fmt, pow2f(k));
                inv = pow2f(-k);
            }
        }
        scales[b] = scode;

        for (int t = 0; t < L; t++) {
            int64_t idx = ri[t] * cols + ci[t];
            uint8_t q = 0;
            if (!zero_block) {
                float v = res[t] * inv;
                uint32_t u = (cfg->round_mode == RD_SR) ? elem_random(cfg->seed, (uint64_t)idx) : 0u;
                q = encode_elem(&g, asym, cfg->round_mode, v, u);
            }
            codes[idx] = q;
        }
    }
    free(ri); free(ci); free(res);
    free(y); free(yq); free(sm_val);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Packing (READING): 4-bit codes two per byte along a row, the lower        */
/* column in the low nibble; 6-bit codes one per byte (low 6 bits).          */
/* Pinned: 4.25 / 4.5 bits per element for MXFP4 / NVFP4 storage.            */
/* ------------------------------------------------------------------------ */
/* The alternating optimisation's s_T and squared error after each group
 * step (rounds + 1 entries each), for the tests: row-axis E2M1 blocks, a
 * nearest scale format, bf16 or fp32 input.  Returns the final s_T. */
float orc_mse_grid_trace(int scale_fmt, int block, const void *x, int dtype, int64_t rows, int64_t cols,
                         int rounds, float *sT_trace, double *sse_trace)
{
    grid_t g; make_grid(0, 0, &g);
    const int64_t n = rows * cols;
    float *y = (float *)malloc((size_t)n * sizeof(float));
    if (!y) return NAN;
    load_input(x, dtype, n, y);
    float sT = orc_tensor_scale(0, scale_fmt, y, n);
    sT = mse_grid_alternate(&g, scale_fmt, AX_ROW, block, y, rows, cols, sT, rounds, sT_trace, sse_trace);
    free(y);
    return sT;
}

int64_t orc_packed_bytes(int elem, int64_t rows, int64_t cols)
{
    grid_t g; make_grid(elem, 0, &g);
    return g.bits == 4 ? rows * (cols / 2) : rows * cols;
}

void orc_pack(int elem, const uint8_t *codes, int64_t rows, int64_t cols, uint8_t *packed)
{
    grid_t g; make_grid(elem, 0, &g);
    if (g.bits == 6) {
        for (int64_t i = 0; i < rows * cols; i++) packed[i] = codes[i] & 0x3f;
        return;
    }
    for (int64_t r = 0; r < rows; r++)
        for (int64_t j = 0; j < cols / 2; j++) {
            uint8_t lo = codes[r * cols + 2 * j] & 0xf, hi = codes[r * cols + 2 * j + 1] & 0xf;
            packed[r * (cols / 2) + j] = (uint8_t)(lo | (hi << 4));
        }
}

void orc_unpack(int elem, const uint8_t *packed, int64_t rows, int64_t cols, uint8_t *codes);

/* (READING) Tensor-core operand form of FP6 codes (the library's
 * sf_layout = 1): every 16 consecutive codes of a row are packed into 12
 * bytes, code i at bits [6i, 6i + 6) of the little-endian 96-bit value, the
 * groups back to back: 6 bits per element, 12 bytes per 16.  That is the
 * packed global form of CUDA's 16 x U6 tensor-map type, which the copy into
 * shared memory widens to 16 bytes per group.  FP4 codes keep their packing
 * (two per byte). */
int64_t orc_packed_tc_bytes(int elem, int64_t rows, int64_t cols)
{
    grid_t g; make_grid(elem, 0, &g);
    return g.bits == 6 ? rows * cols / 16 * 12 : rows * (cols / 2);
}

void orc_pack_tc(int elem, const uint8_t *codes, int64_t rows, int64_t cols, uint8_t *packed)
{
    grid_t g; make_grid(elem, 0, &g);
    if (g.bits != 6) { orc_pack(elem, codes, rows, cols, packed); return; }
    for (int64_t i0 = 0; i0 < rows * cols; i0 += 16) {
        uint8_t *dst = packed + i0 / 16 * 12;
        memset(dst, 0, 12);
        for (int i = 0; i < 16; i++) {
            unsigned v = codes[i0 + i] & 0x3fu;
            for (int b = 0; b < 6; b++)
                if (v & (1u << b)) dst[(6 * i + b) / 8] |= (uint8_t)(1u << ((6 * i + b) % 8));
        }
    }
}

void orc_unpack_tc(int elem, const uint8_t *packed, int64_t rows, int64_t cols, uint8_t *codes)
{
    grid_t g; make_grid(elem, 0, &g);
    if (g.bits != 6) { orc_unpack(elem, packed, rows, cols, codes); return; }
    for (int64_t i0 = 0; i0 < rows * cols; i0 += 16) {
        const uint8_t *src = packed + i0 / 16 * 12;
        for (int i = 0; i < 16; i++) {
            unsigned v = 0;
            for (int b = 0; b < 6; b++)
                if (src[(6 * i + b) / 8] & (1u << ((6 * i + b) % 8))) v |= 1u << b;
            codes[i0 + i] = (uint8_t)v;
        }
    }
}

void orc_unpack(int elem, const uint8_t *packed, int64_t rows, int64_t cols, uint8_t *codes)
{
    grid_t g; make_grid(elem, 0, &g);
    if (g.bits == 6) {
        for (int64_t i = 0; i < rows * cols; i++) codes[i] = packed[i] & 0x3f;
        return;
    }
    for (int64_t r = 0; r < rows; r++)
        for (int64_t j = 0; j < cols / 2; j++) {
            uint8_t p = packed[r * (cols / 2) + j];
            codes[r * cols + 2 * j] = p & 0xf;
            codes[r * cols + 2 * j + 1] = p >> 4;
        }
}

/* ------------------------------------------------------------------------ */
/* Dequantize ([MX-TRAIN] fake quantization: quantize then return to high   */
/* precision).  (READING) x_hat = (q * s_b) * s_T, times S_M for MBS, plus   */
/* the offset for asymmetric blocks, each product / sum one binary32 op.     */
/* A NaN scale gives NaN.  With a rotation, the normalised Hadamard (its own */
/* inverse) is applied afterwards to return to the input space when          */
/* `unrotate` is set.                                                        */
/* ------------------------------------------------------------------------ */
int orc_dequantize(const orc_cfg *cfg, const uint8_t *packed, const uint8_t *scales,
                   const float *tensor_scale, const uint8_t *macro, const uint16_t *offsets,
                   int64_t rows, int64_t cols, int unrotate, float *out)
{
    const int B = cfg->block;
    const int asym = cfg->asymmetric;
    grid_t g; make_grid(cfg->elem, asym, &g);
    uint8_t *codes = (uint8_t *)malloc((size_t)(rows * cols));
    if (!codes) return -1;
    orc_unpack(cfg->elem, packed, rows, cols, codes);
    float sT = (cfg->tensor_scale != TS_NONE && tensor_scale) ? *tensor_scale : 1.0f;
    const int64_t nb = n_blocks(cfg->axis, B, rows, cols);
    const int L = block_len(cfg->axis, B);
    for (int64_t b = 0; b < nb; b++) {
        uint8_t sc = scales[b];
        float s = orc_scale_decode(cfg->scale_fmt, sc);
        float o = asym ? orc_bf16_to_f32(offsets[b]) : 0.0f;
        for (int t = 0; t < L; t++) {
            int64_t r, c;
            block_elem(cfg->axis, B, rows, cols, b, t, &r, &c);
            int64_t idx = r * cols + c;
            float q = decode_elem(&g, asym, codes[idx]);
            float v;
            if (isnan(s)) v = NAN;
            else if (cfg->scale_fmt != S_E8M0 && (cfg->rule == R_NEAREST || cfg->rule == R_MSE)) v = (q * s) * sT;
            else {
                v = q * s;
                if (cfg->macro_block) v = v * e4m3_decode(macro[macro_index(cfg->axis, rows, cols, r, c)]);
                if (asym) v = v + o;
            }
            out[idx] = v;
        }
    }
    free(codes);
    if (unrotate && cfg->hadamard) rotate(cfg->axis, cfg->hadamard, rows, cols, out);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Fidelity reductions in binary64.                                          */
/* [MXFP4-OAS] Sec.3 Eq. (1): QSNR = 10 log10(||A||_F^2 / ||A - A^Q||_F^2).  */
/* [MX-TRAIN]: R-MSE = sqrt(MSE).  [MXFP4-OAS] Sec.3: flush-to-zero share.    */
/* stats: [0] sum x^2  [1] sum (x - xh)^2  [2] sum (xh - x)  [3] #ftz         */
/*        [4] #nonzero [5] mse [6] rmse [7] qsnr_db [8] bias [9] ftz frac     */
/*        [10] element count                                                  */
/* (READING) sum x^2 = 0 -> QSNR NaN; zero error -> +inf.                     */
/* Pinned: closed form x_hat = (1 - eps) x  =>  QSNR = -20 log10(eps).        */
/* ------------------------------------------------------------------------ */
void orc_finalize_stats(double *st)
{
    double n = st[10];
    st[5] = n > 0 ? st[1] / n : 0.0;
    st[6] = sqrt(st[5]);
    if (st[0] == 0.0) st[7] = NAN;
    else if (st[1] == 0.0) st[7] = INFINITY;
    else st[7] = 10.0 * log10(st[0] / st[1]);
    st[8] = n > 0 ? st[2] / n : 0.0;
    st[9] = st[4] > 0 ? st[3] / st[4] : 0.0;
}

void orc_stats(const float *ref, const float *xhat, int64_t rows, int64_t cols, int block,
               int axis, double *stats, float *per_block_mse)
{
    for (int i = 0; i < 16; i++) stats[i] = 0.0;
    for (int64_t i = 0; i < rows * cols; i++) {
        double x = (double)ref[i], xh = (double)xhat[i];
        double d = x - xh;
        stats[0] += x * x;
        stats[1] += d * d;
        stats[2] += xh - x;
        if (ref[i] != 0.0f) {
            stats[4] += 1.0;
            if (xhat[i] == 0.0f) stats[3] += 1.0;
        }
    }
    stats[10] = (double)(rows * cols);
    orc_finalize_stats(stats);
    if (per_block_mse && block > 0) {
        const int64_t nb = n_blocks(axis, block, rows, cols);
        const int L = block_len(axis, block);
        for (int64_t b = 0; b < nb; b++) {
            double s = 0.0;
            for (int t = 0; t < L; t++) {
                int64_t r, c;
                block_elem(axis, block, rows, cols, b, t, &r, &c);
                double d = (double)ref[r * cols + c] - (double)xhat[r * cols + c];
                s += d * d;
            }
            per_block_mse[b] = (float)(s / (double)L);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* GEMM QSNR ([MXFP4-OAS] Sec.3 Eq. (2)), C = A B^T with A [M x K] and B     */
/* [N x K]: triple loop in binary64 for small shapes; the reference product  */
/* uses the unquantized operands, the quantized one the dequantized values.  */
/* out: [0] sum C_ref^2  [1] sum (C_ref - C_q)^2  [2] QSNR(AB) dB             */
/* ------------------------------------------------------------------------ */
void orc_gemm(const float *A, const float *B, int64_t M, int64_t N, int64_t K, double *C)
{
    for (int64_t m = 0; m < M; m++)
        for (int64_t n = 0; n < N; n++) {
            double s = 0.0;
            for (int64_t k = 0; k < K; k++) s += (double)A[m * K + k] * (double)B[n * K + k];
            C[m * N + n] = s;
        }
}

void orc_gemm_qsnr(const float *A, const float *B, const float *Ah, const float *Bh,
                   int64_t M, int64_t N, int64_t K, double *out)
{
    double sr = 0.0, se = 0.0;
    for (int64_t m = 0; m < M; m++)
        for (int64_t n = 0; n < N; n++) {
            double cr = 0.0, cq = 0.0;
            for (int64_t k = 0; k < K; k++) {
                cr += (double)A[m * K + k] * (double)B[n * K + k];
                cq += (double)Ah[m * K + k] * (double)Bh[n * K + k];
            }
            sr += cr * cr;
            se += (cr - cq) * (cr - cq);
        }
    out[0] = sr;
    out[1] = se;
    out[2] = (sr == 0.0) ? NAN : (se == 0.0 ? INFINITY : 10.0 * log10(sr / se));
}
