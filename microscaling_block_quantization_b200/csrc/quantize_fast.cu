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
// One launch may cover several tensors of one configuration (a group): the
// CTAs are split among them, and each tensor keeps its own tensor scale,
// statistics records and ticket.
#include <string.h>

#include "tma_ring.cuh"

namespace mxk {

namespace {

constexpr int kConsumers = kRingConsumers;
constexpr int kFastThreads = kRingThreads;
constexpr int kWaitFull = 21, kWaitEmpty = 22;    // status codes of the bounded waits

// number of zero-magnitude E2M1 codes among the 8 nibbles of w: a nibble's
// magnitude m (0..7) plus 7 sets bit 3 exactly when m != 0, with no carry out
__device__ __forceinline__ int zero_codes8(uint32_t w)
{
    return 8 - __popc(((w & 0x77777777u) + 0x77777777u) & 0x88888888u);
}

// in-lane block Hadamard on the 32-element chunk: groups of n (16 or 32).
// Stage 1 pairs neighbours; the later stages pair (j, j+1) with (j+h, j+h+1)
// and run as two-lane binary32 operations (a - b as fma(b, -1, a): one
// rounding, the same value as the subtraction).
template <int H>
__device__ __forceinline__ void butterfly_stage2(float y[32])
{
    const float2 m1 = make_float2(-1.0f, -1.0f);
#pragma unroll
    for (int i = 0; i < 32; i += 2 * H)
#pragma unroll
        for (int j = i; j < i + H; j += 2) {
            const float2 a = make_float2(y[j], y[j + 1]), b = make_float2(y[j + H], y[j + H + 1]);
            const float2 sum = __fadd2_rn(a, b), dif = __ffma2_rn(b, m1, a);
            y[j] = sum.x; y[j + 1] = sum.y;
            y[j + H] = dif.x; y[j + H + 1] = dif.y;
        }
}

template <int N, bool SCALE = true, bool STAGE1 = true>
__device__ __forceinline__ void hadamard_groups(float y[32])
{
    if constexpr (STAGE1) {
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
            const float a = y[j], b = y[j + 1];
            y[j] = __fadd_rn(a, b);
            y[j + 1] = __fsub_rn(a, b);
        }
    }
    butterfly_stage2<2>(y);
    butterfly_stage2<4>(y);
    butterfly_stage2<8>(y);
    if constexpr (N == 32) butterfly_stage2<16>(y);
    if constexpr (!SCALE) return;
    const float c = hadamard_scale(N);
    const float2 c2 = make_float2(c, c);
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
        const float2 v = __fmul2_rn(make_float2(y[j], y[j + 1]), c2);
        y[j] = v.x; y[j + 1] = v.y;
    }
}

// ---- bf16 inputs kept packed (two elements a 32-bit word) ------------------
// The block statistic is taken on the packed words (halfwise maximum of
// magnitudes, NaN-propagating), and each element is widened and scaled in one
// mixed-precision multiply-add, y * c + (-0) with y and c bf16 and the result
// rounded once to binary32 (exact for a power-of-two c; c = 1 widens; the
// -0 addend keeps the sign of a zero product): no separate unpacking.

// halfwise max(|a|, |b|), NaN-propagating (the result's sign bits are unused)
__device__ __forceinline__ uint32_t bf2_absmax(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
// halfwise min(|a|, |b|)
__device__ __forceinline__ uint32_t bf2_absmin(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("min.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// max |y| (NaN-propagating) of the 2N values in N words, as binary32 (a tree)
template <int N>
__device__ __forceinline__ float bf_absmax(const uint32_t *w)
{
    uint32_t m[N];
#pragma unroll
    for (int i = 0; i < N; ++i) m[i] = w[i];
#pragma unroll
    for (int st = 1; st < N; st *= 2)
#pragma unroll
        for (int i = 0; i + st < N; i += 2 * st) m[i] = bf2_absmax(m[i], m[i + st]);
    return fmax_nan(fabsf(__uint_as_float(m[0] << 16)), fabsf(__uint_as_float(m[0] & 0xffff0000u)));
}
// min |y| of the 2N values in N words, as binary32
template <int N>
__device__ __forceinline__ float bf_absmin(const uint32_t *w)
{
    uint32_t m[N];
#pragma unroll
    for (int i = 0; i < N; ++i) m[i] = w[i];
#pragma unroll
    for (int st = 1; st < N; st *= 2)
#pragma unroll
        for (int i = 0; i + st < N; i += 2 * st) m[i] = bf2_absmin(m[i], m[i + st]);
    return fminf(fabsf(__uint_as_float(m[0] << 16)), fabsf(__uint_as_float(m[0] & 0xffff0000u)));
}

// the eight bf16 values of four words times the bf16 value c (low 16 bits),
// each product rounded once to binary32
__device__ __forceinline__ void bf16x8_scale(const uint32_t *w, uint32_t c, float s[8])
{
    asm("{\n\t.reg .b16 a0, a1, a2, a3, a4, a5, a6, a7, k, kx;\n\t.reg .f32 z;\n\t"
        "mov.b32 {a0, a1}, %8;\n\t"
        "mov.b32 {a2, a3}, %9;\n\t"
        "mov.b32 {a4, a5}, %10;\n\t"
        "mov.b32 {a6, a7}, %11;\n\t"
        "mov.b32 {k, kx}, %12;\n\t"
        "mov.f32 z, 0f80000000;\n\t"
        "fma.rn.f32.bf16 %0, a0, k, z;\n\t"
        "fma.rn.f32.bf16 %1, a1, k, z;\n\t"
        "fma.rn.f32.bf16 %2, a2, k, z;\n\t"
        "fma.rn.f32.bf16 %3, a3, k, z;\n\t"
        "fma.rn.f32.bf16 %4, a4, k, z;\n\t"
        "fma.rn.f32.bf16 %5, a5, k, z;\n\t"
        "fma.rn.f32.bf16 %6, a6, k, z;\n\t"
        "fma.rn.f32.bf16 %7, a7, k, z;\n\t}"
        : "=f"(s[0]), "=f"(s[1]), "=f"(s[2]), "=f"(s[3]), "=f"(s[4]), "=f"(s[5]), "=f"(s[6]), "=f"(s[7])
        : "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(c));
}

// First butterfly stage of the rotation straight from four bf16 words: for
// the pair (a, b) of each word, b + a and a - b rounded once to binary32
// (a widened exactly, then b * (+1 / -1) + a in one mixed-precision
// multiply-add each) -- the values of the binary32 additions on the widened
// pair.
__device__ __forceinline__ void bf16x8_stage1(const uint32_t *w, float y[8])
{
    asm("{\n\t.reg .b16 a0, b0, a1, b1, a2, b2, a3, b3, p1, m1;\n\t"
        ".reg .f32 z, t0, t1, t2, t3;\n\t"
        "mov.b32 {a0, b0}, %8;\n\t"
        "mov.b32 {a1, b1}, %9;\n\t"
        "mov.b32 {a2, b2}, %10;\n\t"
        "mov.b32 {a3, b3}, %11;\n\t"
        "mov.b16 p1, 0x3F80;\n\t"
        "mov.b16 m1, 0xBF80;\n\t"
        "mov.f32 z, 0f80000000;\n\t"
        "fma.rn.f32.bf16 t0, a0, p1, z;\n\t"
        "fma.rn.f32.bf16 t1, a1, p1, z;\n\t"
        "fma.rn.f32.bf16 t2, a2, p1, z;\n\t"
        "fma.rn.f32.bf16 t3, a3, p1, z;\n\t"
        "fma.rn.f32.bf16 %0, b0, p1, t0;\n\t"
        "fma.rn.f32.bf16 %1, b0, m1, t0;\n\t"
        "fma.rn.f32.bf16 %2, b1, p1, t1;\n\t"
        "fma.rn.f32.bf16 %3, b1, m1, t1;\n\t"
        "fma.rn.f32.bf16 %4, b2, p1, t2;\n\t"
        "fma.rn.f32.bf16 %5, b2, m1, t2;\n\t"
        "fma.rn.f32.bf16 %6, b3, p1, t3;\n\t"
        "fma.rn.f32.bf16 %7, b3, m1, t3;\n\t}"
        : "=f"(y[0]), "=f"(y[1]), "=f"(y[2]), "=f"(y[3]), "=f"(y[4]), "=f"(y[5]), "=f"(y[6]), "=f"(y[7])
        : "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]));
}

// Lane t's chunk of 32 bf16 values as 16 words, out of the swizzled tile.
__device__ __forceinline__ void ring_read_words(const uint8_t *stage, int t, uint32_t w[16])
{
    const uint8_t *row = stage + 64 * t;
    const int sw = (t >> 1) & 3;                       // 64-byte swizzle
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint4 u = *reinterpret_cast<const uint4 *>(row + 16 * (k ^ sw));
        w[4 * k] = u.x; w[4 * k + 1] = u.y; w[4 * k + 2] = u.z; w[4 * k + 3] = u.w;
    }
}

// A launch over up to kFastGroupMax tensors of one configuration: the CTAs
// are split among the tensors (cta0 prefix), every CTA works on one tensor
// with that tensor's tensor map and outputs; p[0] also carries the shared
// configuration.
struct FastGroup {
    CUtensorMap tm[kFastGroupMax];
    QParams p[kFastGroupMax];
    uint32_t cta0[kFastGroupMax + 1];
    int n;
};

// HADN: block rotation over groups of HADN (0: none, 16, 32) before
// quantization; MBS: 1 x 128 macro scale over the
// 4 lanes of a macro block (consecutive chunks of a tile are consecutive lanes).
template <typename InT, int B, bool STATS, int HADN, bool MBS, bool NEAR>
__global__ void __launch_bounds__(kFastThreads, (HADN || ((MBS || STATS) && sizeof(InT) != 2)) ? 2 : 3) k_quant_fast(const __grid_constant__ FastGroup g)
{
    constexpr int NB = B <= 32 ? 32 / B : 1;
    constexpr int G = B <= 32 ? 1 : B / 32;
    constexpr int L = B <= 32 ? B : 32;
    extern __shared__ uint8_t smem_raw[];
    const Ring<InT> ring(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // this CTA's tensor, and its place among the tensor's CTAs
    int item = 0;
    while (item + 1 < g.n && blockIdx.x >= g.cta0[item + 1]) ++item;
    const QParams &pc = g.p[0];
    const QParams &p = g.p[item];
    const uint32_t cta = blockIdx.x - g.cta0[item], ncta = g.cta0[item + 1] - g.cta0[item];
    const uint32_t nch = (uint32_t)(p.rows * p.cols / 32);
    // the tensor's outputs, read once from the launch parameters
    uint4 *const codes0 = static_cast<uint4 *>(p.codes);
    uint8_t *const scales0 = p.scales;
    uint8_t *const macro0 = p.macro;
    const int64_t cols = p.cols;
    const uint32_t ntiles = (nch + kConsumers - 1) / kConsumers;
    pdl_trigger();
    if (threadIdx.x == 0) ring.init();
    pdl_wait();
    const float sT = launch_tensor_scale(p, cta == 0);
    // nearest scales: s_b s_T and its reciprocal for every scale code, once per CTA
    __shared__ float2 near_tab[NEAR ? 256 : 1];
    if constexpr (NEAR)
        for (int c = threadIdx.x; c < 256; c += blockDim.x) {
            const float d = __fmul_rn(ue_value(pc.sd, (uint32_t)c), sT);
            near_tab[c] = c < pc.sd.ue_nan_code ? make_float2(d, __fdiv_rn(1.0f, d))
                                               : make_float2(__uint_as_float(0x7fc00000u), 0.0f);
        }
    // macro scales: {S_M, RN(1 / S_M)} for every E4M3 code, once per CTA
    __shared__ float2 macro_tab[MBS ? 128 : 1];
    if constexpr (MBS)
        for (int c = threadIdx.x; c < 128; c += blockDim.x) {
            const float v = e4m3_value((uint32_t)c);
            macro_tab[c] = make_float2(v, __fdiv_rn(1.0f, v));
        }
    const float md = MBS ? __fmul_rn(pc.ed.maxv, exp2i(-pc.ed.emax)) : 1.0f;   // max_elem / 2^emax, exact
    const float r_md = MBS ? __fdiv_rn(1.0f, md) : 1.0f;
    __syncthreads();
    NearScale ns;
    ns.maxv = pc.ed.maxv;
    ns.r_max = __fdiv_rn(1.0f, pc.ed.maxv);
    ns.sT = sT;
    ns.r_T = (sT >= 0x1p-125f && sT <= 0x1p125f) ? __fdiv_rn(1.0f, sT) : 0.0f;
    {
        // the UE4M3 shortcut's constant, when max_elem s_T and its reciprocal are normal
        const float ms = __fmul_rn(pc.ed.maxv, sT);
        ns.c = (ms >= 0x1p-125f && ms <= 0x1p125f) ? __fdiv_rn(1.0f, ms) : 0.0f;
    }
    ns.tab = near_tab;

    Acc acc = {0, 0, 0, 0, 0};
    if (warp == kConsumers / 32) {
        // producer: one lane streams the CTA's tiles through the ring
        if (lane == 0) ring.produce(&g.tm[item], ntiles, kWaitEmpty, cta, ncta);
        __syncwarp();
    } else {
        // rotation with power-of-two scales: the normaliser c = 1/sqrt(n) moves
        // into the scale, s = y_H * (c * 2^-k) = (y_H * c) * 2^-k exactly
        constexpr bool FOLD = HADN != 0 && !MBS && !NEAR;
        // bf16 input without rotation: kept packed
        constexpr bool PACKED = sizeof(InT) == 2 && HADN == 0;
        constexpr bool ROT16 = sizeof(InT) == 2 && HADN != 0;
        const float hc = HADN ? hadamard_scale(HADN) : 1.0f;
        const bool e8m0 = !NEAR && pc.sd.fmt == S_E8M0;
        const float thr_m = e8m0_threshold(pc.ed, pc.sd);
        const uint32_t S = (uint32_t)(cols / B);
        const int t = threadIdx.x;
        uint32_t i = 0;
        for (uint32_t tile = cta; tile < ntiles; tile += ncta, ++i) {
            if (!ring.acquire(i, kWaitFull)) break;
            float y[PACKED ? 1 : 32];
            uint32_t w[PACKED || ROT16 ? 16 : 1];
            if constexpr (PACKED || ROT16) ring_read_words(ring.stage(i % RingCfg<InT>::kStages), t, w);
            else ring_read_chunk(ring.stage(i % RingCfg<InT>::kStages), t, static_cast<const InT *>(nullptr), y);
            ring.release(i);                  // the chunk is in registers: hand the slot back
            if constexpr (ROT16) {
                // bf16 rotation: the first butterfly stage widens the pairs
#pragma unroll
                for (int g = 0; g < 4; ++g) bf16x8_stage1(w + 4 * g, y + 8 * g);
                hadamard_groups<HADN, !FOLD, false>(y);
            } else if constexpr (HADN != 0) {
                hadamard_groups<HADN, !FOLD>(y);
            }
            // macro-block scale: y' = y * (1 / S_M), x_hat = (q X) S_M
            float sm = 1.0f;
            if constexpr (MBS && !PACKED) {
                const float m = absmax_nan<32>(y);
                int mbad = !(m <= FLT_MAX);
                float mm = grp_max(mbad ? 0.0f : m, 4);
                mbad = grp_or(mbad, 4);
                const uint32_t mcode = macro_code_recip(md, r_md, mm, mbad);
                const float2 mt = macro_tab[mcode];
                sm = mt.x;
                const float invm = mt.y;
                if ((t & 3) == 0 && tile * kConsumers + t < nch) macro0[(tile * kConsumers + t) >> 2] = (uint8_t)mcode;
                const float2 invm2 = make_float2(invm, invm);
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    const float2 v = __fmul2_rn(make_float2(y[j], y[j + 1]), invm2);
                    y[j] = v.x; y[j + 1] = v.y;
                }
            }

            const uint32_t c = tile * kConsumers + t;
            const bool ok = c < nch;
            uint32_t words[4];
            uint32_t scode[NB];
            // packed two-lane binary32 arithmetic (each lane rounded as a scalar op)
            int nzc = 0, ftzc = 0;
            if constexpr (PACKED) {
                // block statistics of the packed words
                float a[NB], mn[NB];
                int bad[NB];
#pragma unroll
                for (int k = 0; k < NB; ++k) {
                    a[k] = bf_absmax<L / 2>(w + k * (L / 2));
                    mn[k] = STATS ? bf_absmin<L / 2>(w + k * (L / 2)) : 1.0f;
                    bad[k] = !(a[k] <= FLT_MAX);
                    if (G > 1) {
                        a[k] = grp_max(bad[k] ? 0.0f : a[k], G);
                        bad[k] = grp_or(bad[k], G);
                    }
                }
                // macro-block scale over the 4 lanes of a 1 x 128 block; the
                // block rule then sees y' = RN(y / S_M), whose block max and
                // min are RN(max |y| / S_M) and RN(min |y| / S_M) (rounding is
                // monotone)
                float sm = 1.0f, invm = 1.0f;
                if constexpr (MBS) {
                    float m = a[0];
                    int mbad = bad[0];
#pragma unroll
                    for (int k = 1; k < NB; ++k) {
                        m = fmax_nan(m, a[k]);
                        mbad |= bad[k];
                    }
                    const float mm = grp_max(mbad ? 0.0f : m, 4);
                    mbad = grp_or(mbad, 4);
                    const uint32_t mcode = macro_code_recip(md, r_md, mm, mbad);
                    const float2 mt = macro_tab[mcode];
                    sm = mt.x;
                    invm = mt.y;
                    if ((t & 3) == 0 && ok) macro0[c >> 2] = (uint8_t)mcode;
                    // a block is non-finite when any of its y' is: a NaN
                    // macro scale (a non-finite value in the macro block)
                    // makes every block of it NaN, and y * (1 / S_M) may
                    // overflow for the largest bf16 values
#pragma unroll
                    for (int k = 0; k < NB; ++k) {
                        a[k] = __fmul_rn(a[k], invm);
                        mn[k] = __fmul_rn(mn[k], invm);
                        bad[k] = !(a[k] <= FLT_MAX);
                    }
                }
#pragma unroll
                for (int k = 0; k < NB; ++k) {
                    const uint32_t *wb = w + k * (L / 2);
                    const BlockScale bs = NEAR ? near_block_scale(pc.sd, ns, bad[k] ? 0.0f : a[k], bad[k])
                                        : e8m0 ? e8m0_block_scale(bad[k] ? 0.0f : a[k], bad[k], pc.ed.emax, thr_m)
                                               : block_scale(pc.ed, pc.sd, bad[k] ? 0.0f : a[k], bad[k], sT);
                    scode[k] = bs.code;
                    float deqT = bs.nan ? __uint_as_float(0x7fc00000u) : bs.deq;
                    if (MBS) deqT = __fmul_rn(deqT, sm);       // X S_M, exact (E4M3 times a power of two)
                    float inv = bs.inv, im = invm;
                    // a flushed block: residuals are the inputs themselves
                    // (scaled by a power of two from the block maximum, so that
                    // their squares stay within binary32)
                    const bool flush = bs.zero && !bs.nan;
                    if (flush) {
                        const float2 pp = pow2_near_inv(a[k]);
                        inv = pp.x;
                        im = 1.0f;
                        deqT = pp.y;
                    }
                    // power-of-two rules: s = y 2^-k straight from the packed
                    // words (exact); nearest scales and MBS: widen, then
                    // multiply (MBS: by 1 / S_M, then by 2^-k, as the rule is
                    // defined on y')
                    constexpr bool WIDEN = NEAR || MBS;
                    const uint32_t kb = WIDEN ? 0x3f80u : (__float_as_uint(inv) >> 16);
                    const float2 inv2 = make_float2(inv, inv), im2 = make_float2(im, im);
                    float2 sx2 = make_float2(0.f, 0.f), re2[2] = {sx2, sx2}, rb2[2] = {sx2, sx2};
                    int qz = 0;
#pragma unroll
                    for (int g = 0; g < L / 8; ++g) {
                        float s8[8];
                        bf16x8_scale(wb + 4 * g, kb, s8);
                        if (WIDEN) {
#pragma unroll
                            for (int e = 0; e < 8; e += 2) {
                                float2 v = make_float2(s8[e], s8[e + 1]);
                                if (MBS) v = __fmul2_rn(v, im2);
                                v = __fmul2_rn(v, inv2);
                                s8[e] = v.x;
                                s8[e + 1] = v.y;
                            }
                        }
                        const uint32_t word = bs.zero ? 0u : cvt_e2m1x8(s8);
                        words[(k * L) / 8 + g] = word;
                        if (STATS) {
                            uint32_t h[4];
                            e2m1x8_halves(word, h);
#pragma unroll
                            for (int e = 0; e < 8; e += 2) {
                                const float2 d = sub_f16x2_from(s8[e], s8[e + 1], h[e >> 1]);   // s - q
                                const int u = (e >> 1) & 1;
                                re2[u] = __ffma2_rn(d, d, re2[u]);
                                rb2[u] = __fadd2_rn(rb2[u], d);
                                // reference sum on the scaled values (y = X s,
                                // exactly for power-of-two scales): sum s^2,
                                // times X^2 below in binary64
                                const float2 sv = make_float2(s8[e], s8[e + 1]);
                                sx2 = __ffma2_rn(sv, sv, sx2);
                            }
                            qz += zero_codes8(word);
                        }
                    }
                    if (STATS) {
                        if (ok) {
                            // y - x_hat = deqT (s - q); reference sum sum s^2 X^2
                            // (a flushed block: s = y, X = 1)
                            const double X = (double)deqT;
                            acc.e2 += (double)((re2[0].x + re2[1].x) + (re2[0].y + re2[1].y)) * X * X;
                            acc.e -= (double)((rb2[0].x + rb2[1].x) + (rb2[0].y + rb2[1].y)) * X;
                            if (!bs.nan) {
                                acc.x2 += (double)(sx2.x + sx2.y) * X * X;
                            } else {
                                // a non-finite block (rare): sum y^2 of its inputs in binary64
                                double t2 = 0.0;
                                for (int j = 0; j < L / 2; ++j) {
                                    const double y0 = (double)__uint_as_float(wb[j] << 16);
                                    const double y1 = (double)__uint_as_float(wb[j] & 0xffff0000u);
                                    t2 += y0 * y0 + y1 * y1;
                                }
                                acc.x2 += t2;
                            }
                        }
                        int xz = 0;
                        if (mn[k] == 0.0f)                 // rare: count exact zeros
#pragma unroll
                            for (int j = 0; j < L / 2; ++j)
                                xz += ((wb[j] & 0x7fffu) == 0u) + ((wb[j] & 0x7fff0000u) == 0u);
                        nzc += L - xz;
                        if (!bs.nan) ftzc += qz - xz;
                    }
                }
            } else {
#pragma unroll
            for (int k = 0; k < NB; ++k) {
                const int j0 = k * L;
                float a = absmax_nan<L>(y + j0), mabs = 1.0f;
                if (STATS) mabs = absmin<L>(y + j0);
                int bad = !(a <= FLT_MAX);
                if (G > 1) {
                    a = grp_max(bad ? 0.0f : a, G);
                    bad = grp_or(bad, G);
                }
                if (FOLD) a = __fmul_rn(a, hc);            // max |y_H c| = RN(max |y_H| c)
                const BlockScale bs = NEAR ? near_block_scale(pc.sd, ns, bad ? 0.0f : a, bad)
                                    : e8m0 ? e8m0_block_scale(bad ? 0.0f : a, bad, pc.ed.emax, thr_m)
                                           : block_scale(pc.ed, pc.sd, bad ? 0.0f : a, bad, sT);
                scode[k] = bs.code;
                float deqT = bs.nan ? __uint_as_float(0x7fc00000u) : bs.deq;     // nearest: s_b s_T
                if (MBS) deqT = __fmul_rn(deqT, sm);       // X * S_M is exact (power of two times E4M3)
                float inv = bs.inv;
                // folded rotation: inv = c 2^-k, exact unless subnormal; then
                // (rare) normalise the block's values first
                float sxm = MBS ? sm : FOLD ? hc : 1.0f;  // reference values = sxm * y
                if (FOLD) {
                    if (inv >= 0x1p-123f || bs.zero) {
                        inv = __fmul_rn(inv, hc);
                    } else {
#pragma unroll
                        for (int j = j0; j < j0 + L; ++j) y[j] = __fmul_rn(y[j], hc);
                        sxm = 1.0f;
                    }
                }
                // a flushed block (x_hat = 0, not NaN): residuals are the
                // reference values themselves, s = sxm y P with factor 1 / P
                // (P a power of two from the block maximum: no binary32
                // overflow of the squares)
                if (bs.zero && !bs.nan) {
                    const float2 pp = pow2_near_inv(__fmul_rn(a, MBS ? sm : 1.0f));
                    inv = __fmul_rn(sxm, pp.x);
                    deqT = pp.y;
                }
                const float2 inv2 = make_float2(inv, inv);
                float2 sx2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                // residuals on the scaled values: y - x_hat = deqT (s - q), exact
                // for power-of-two scales, within an ulp of y otherwise
                float2 re2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)}, rb2[2] = {re2[0], re2[0]};
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
                        uint32_t h[4];
                        e2m1x8_halves(word, h);
#pragma unroll
                        for (int e = 0; e < 8; e += 2) {
                            const float2 d = sub_f16x2_from(s8[e], s8[e + 1], h[e >> 1]);   // s - q
                            const int u = (e >> 1) & 1;          // two accumulator chains
                            re2[u] = __ffma2_rn(d, d, re2[u]);
                            rb2[u] = __fadd2_rn(rb2[u], d);
                            const float2 sv = make_float2(s8[e], s8[e + 1]);
                            sx2[u] = __ffma2_rn(sv, sv, sx2[u]);     // reference values X s
                        }
                        qz += zero_codes8(word);
                    }
                }
                if (STATS) {
                    if (ok) {
                        // y - x_hat = deqT (s - q); a NaN block makes the sums NaN;
                        // reference sum sum s^2 X^2 (a flushed block: s = sxm y, X = 1)
                        const double X = (double)deqT;
                        acc.e2 += (double)((re2[0].x + re2[1].x) + (re2[0].y + re2[1].y)) * X * X;
                        acc.e -= (double)((rb2[0].x + rb2[1].x) + (rb2[0].y + rb2[1].y)) * X;
                        if (!bs.nan) {
                            acc.x2 += (double)((sx2[0].x + sx2[1].x) + (sx2[0].y + sx2[1].y)) * X * X;
                        } else {
                            // a non-finite block (rare): the reference values sxm y in binary64
                            double t2 = 0.0;
                            for (int j = j0; j < j0 + L; ++j) {
                                const double v = (double)y[j] * (double)sxm;
                                t2 += v * v;
                            }
                            acc.x2 += t2;
                        }
                    }
                    int xz = 0;
                    if (mabs == 0.0f)                      // rare: count exact zeros
#pragma unroll
                        for (int j = j0; j < j0 + L; ++j) xz += (y[j] == 0.0f);
                    nzc += L - xz;
                    if (!bs.nan) ftzc += qz - xz;
                }
            }
            }
            if (ok) {
                codes0[c] = make_uint4(words[0], words[1], words[2], words[3]);
                if (G == 1 || (lane & (G - 1)) == 0) {
                    const uint32_t b0 = (G == 1) ? c * NB : c / G;
                    if (pc.sf_gemm) {
                        const uint32_t r = b0 / S, j = b0 - r * S;
#pragma unroll
                        for (int k = 0; k < NB; ++k) scales0[sf_chunk_index(r, j + k, S)] = (uint8_t)scode[k];
                    } else if (NB == 4) {
                        *reinterpret_cast<uint32_t *>(scales0 + b0) =
                            scode[0] | (scode[NB > 1 ? 1 : 0] << 8) | (scode[NB > 2 ? 2 : 0] << 16) |
                            (scode[NB > 3 ? 3 : 0] << 24);
                    } else if (NB == 2) {
                        *reinterpret_cast<uint16_t *>(scales0 + b0) = (uint16_t)(scode[0] | (scode[NB > 1 ? 1 : 0] << 8));
                    } else {
                        scales0[b0] = (uint8_t)scode[0];
                    }
                }
                if (STATS) {
                    acc.nz += (double)nzc;
                    acc.ftz += (double)ftzc;
                }
            }
        }
    }
    finish_launch(p, acc, cta, ncta);
}

template <typename InT, int B, bool STATS, int HADN, bool MBS, bool NEAR>
int launch_fast_b(const QParams *ps, int n, cudaStream_t st)
{
    FastGroup g;
    memset(&g, 0, sizeof(g));
    uint64_t tiles[kFastGroupMax];
    for (int i = 0; i < n; ++i) {
        const uint64_t nch = (uint64_t)(ps[i].rows * ps[i].cols / 32);
        if (ring_map<InT>(&g.tm[i], ps[i].x, nch) != 0) return -1;
        g.p[i] = ps[i];
        tiles[i] = (nch + kConsumers - 1) / kConsumers;
    }
    g.n = n;
    auto k = k_quant_fast<InT, B, STATS, HADN, MBS, NEAR>;
    const int occ = cached_occupancy(reinterpret_cast<const void *>(k), kFastThreads, RingCfg<InT>::kSmem);
    uint64_t total = (uint64_t)device_sm_count() * occ;
    if (total > (uint64_t)kMaxPartials) total = kMaxPartials;
    if (total < (uint64_t)n) total = n;
    split_ctas(tiles, n, total, g.cta0);
    const cudaError_t e = launch_pdl(k, g.cta0[n], kFastThreads, RingCfg<InT>::kSmem, st, g);
    return e == cudaSuccess ? 0 : -1;
}

// statistics on / off; nearest (UE4M3 / UE5M3) or power-of-two scales (the
// macro scale comes only with E8M0)
template <typename InT, int B, int HADN, bool MBS>
int launch_fast_s(const QParams *ps, int n, cudaStream_t st)
{
    const QParams &p = ps[0];
    const bool near = p.sd.fmt != S_E8M0 && p.sd.rule == R_NEAREST;
    bool stats = false;
    for (int i = 0; i < n; ++i) stats = stats || ps[i].partials != nullptr;
    if (MBS || !near)
        return stats ? launch_fast_b<InT, B, true, HADN, MBS, false>(ps, n, st)
                     : launch_fast_b<InT, B, false, HADN, MBS, false>(ps, n, st);
    return stats ? launch_fast_b<InT, B, true, HADN, false, true>(ps, n, st)
                 : launch_fast_b<InT, B, false, HADN, false, true>(ps, n, st);
}

template <typename InT, int B>
int launch_fast_rot(const QParams *ps, int n, cudaStream_t st)
{
    const bool m = ps[0].mbs != 0;
    switch (ps[0].had) {
    case 0: return launch_fast_s<InT, B, 0, true>(ps, n, st);
    case 16: return m ? launch_fast_s<InT, B, 16, true>(ps, n, st) : launch_fast_s<InT, B, 16, false>(ps, n, st);
    case 32: return m ? launch_fast_s<InT, B, 32, true>(ps, n, st) : launch_fast_s<InT, B, 32, false>(ps, n, st);
    default: return -1;
    }
}

template <typename InT>
int launch_fast_t(const QParams *ps, int n, cudaStream_t st)
{
    const QParams &p = ps[0];
    if (p.had || p.mbs) {
        // rotation and / or macro scale: blocks of 16 and 32
        if (p.block == 32) return launch_fast_rot<InT, 32>(ps, n, st);
        return launch_fast_rot<InT, 16>(ps, n, st);
    }
    switch (p.block) {
    case 8: return launch_fast_s<InT, 8, 0, false>(ps, n, st);
    case 16: return launch_fast_s<InT, 16, 0, false>(ps, n, st);
    case 32: return launch_fast_s<InT, 32, 0, false>(ps, n, st);
    case 64: return launch_fast_s<InT, 64, 0, false>(ps, n, st);
    case 128: return launch_fast_s<InT, 128, 0, false>(ps, n, st);
    case 256: return launch_fast_s<InT, 256, 0, false>(ps, n, st);
    default: return -1;
    }
}

}  // namespace

// E2M1 / RTNE / symmetric, row axis, no rotated output; rotation and macro
// scale only with blocks of 16 or 32.  ps[0..n) share the configuration
// (n <= kFastGroupMax, every tensor non-empty).
int launch_quantize_fast_group(const QParams *ps, int n, int in_fp32, cudaStream_t st)
{
    if (n < 1 || n > kFastGroupMax) return -1;
    return in_fp32 ? launch_fast_t<float>(ps, n, st) : launch_fast_t<__nv_bfloat16>(ps, n, st);
}

int launch_quantize_fast(const QParams &p, int in_fp32, cudaStream_t st, int *grid_out)
{
    if (grid_out) *grid_out = 0;
    return launch_quantize_fast_group(&p, 1, in_fp32, st);
}

int take_status_fast(cudaStream_t st, int *v) { return take_ring_status(st, v); }

}  // namespace mxk
