// sm_100a block quantizer kernels for column-wise (B x 1) and 2D (32 x 32)
// blocks (fmread summary of Yang et al.: column-wise blocks help activations,
// 2D blocks balance accuracy and efficiency).
//
// Each warp stages a tile of RB rows x (32 lanes x CPT columns) in shared
// memory with asynchronous 16-byte copies (all rows in flight at once), then
// every lane works down its own CPT columns: column axis -> CPT blocks per
// lane; 2D -> one 32 x 32 block per 32 / CPT lanes.  Loads and stores stay
// coalesced along rows; the reduction runs along columns out of shared memory.
#include <string.h>

#include "quant_common.cuh"

namespace mxk {

namespace {

constexpr int kColWarps = 4;

constexpr int kColThreads = kColWarps * 32;

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src, bool ok)
{
    // src-size 0 fills the 16 bytes with zeros (lanes past the last column)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_addr(dst)), "l"(src),
                 "r"(ok ? 16 : 0));
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::); }

// Per-lane view of the warp tile: slot(r) is the lane's 16 bytes of row r.
// CPT == 8: eight raw bf16; CPT == 4: four binary32 values.
template <int CPT>
struct LaneTile {
    uint4 *base;   // row 0 of this lane; rows are 32 slots apart
    __device__ __forceinline__ void get(int r, float v[CPT]) const
    {
        const uint4 u = base[r * 32];
        if constexpr (CPT == 8) {
            unpack_bf16x2(u.x, v[0], v[1]);
            unpack_bf16x2(u.y, v[2], v[3]);
            unpack_bf16x2(u.z, v[4], v[5]);
            unpack_bf16x2(u.w, v[6], v[7]);
        } else {
            v[0] = __uint_as_float(u.x); v[1] = __uint_as_float(u.y);
            v[2] = __uint_as_float(u.z); v[3] = __uint_as_float(u.w);
        }
    }
    __device__ __forceinline__ void set(int r, const float v[CPT]) const
    {
        static_assert(CPT == 4, "binary32 tiles only");
        base[r * 32] = make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]),
                                  __float_as_uint(v[2]), __float_as_uint(v[3]));
    }
};

// Load RB rows of the lane's CPT columns into its tile slots.
template <typename InT, int CPT>
__device__ __forceinline__ void load_tile(const QParams &p, const LaneTile<CPT> &t, int64_t r0,
                                          int64_t c0, int RB, bool ok)
{
    const InT *x = static_cast<const InT *>(p.x);
    if constexpr (CPT * sizeof(InT) == 16) {
        for (int r = 0; r < RB; ++r) {
            const InT *src = ok ? x + (r0 + r) * p.cols + c0 : x;
            cp_async16(t.base + r * 32, src, ok);
        }
        cp_async_wait_all();
    } else {
        // bf16 with 4 columns per lane: 8-byte loads, widened to binary32
        for (int rb = 0; rb < RB; rb += 8) {
            uint2 u[8];
#pragma unroll
            for (int k = 0; k < 8; ++k)
                u[k] = ok ? __ldg(reinterpret_cast<const uint2 *>(x + (r0 + rb + k) * p.cols + c0))
                          : make_uint2(0, 0);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                float v[4];
                unpack_bf16x2(u[k].x, v[0], v[1]);
                unpack_bf16x2(u[k].y, v[2], v[3]);
                t.base[(rb + k) * 32] = make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]),
                                                   __float_as_uint(v[2]), __float_as_uint(v[3]));
            }
        }
    }
}

// Block Hadamard rotation of the staged tile (binary32 tiles, CPT == 4):
// column axis along rows (in-lane), 2D along the row direction (32/CPT lanes).
template <int AXIS>
__device__ __forceinline__ void rotate_tile(const LaneTile<4> &t, int n, int RB, int lane)
{
    const float cn = hadamard_scale(n);
    if constexpr (AXIS == AX_COL) {
        for (int h = 1; h < n; h <<= 1)
            for (int i = 0; i < RB; i += 2 * h)
                for (int r = i; r < i + h; ++r) {
                    float a[4], b[4], s[4], d[4];
                    t.get(r, a);
                    t.get(r + h, b);
#pragma unroll
                    for (int j = 0; j < 4; ++j) { s[j] = __fadd_rn(a[j], b[j]); d[j] = __fsub_rn(a[j], b[j]); }
                    t.set(r, s);
                    t.set(r + h, d);
                }
        for (int r = 0; r < RB; ++r) {
            float a[4];
            t.get(r, a);
#pragma unroll
            for (int j = 0; j < 4; ++j) a[j] = __fmul_rn(a[j], cn);
            t.set(r, a);
        }
    } else {
        for (int r = 0; r < RB; ++r) {
            float v[4];
            t.get(r, v);
#pragma unroll
            for (int h = 1; h < 4; h <<= 1)
#pragma unroll
                for (int i = 0; i < 4; i += 2 * h)
#pragma unroll
                    for (int j = i; j < i + h; ++j) {
                        float a = v[j], b = v[j + h];
                        v[j] = __fadd_rn(a, b);
                        v[j + h] = __fsub_rn(a, b);
                    }
            for (int m = 1; m < n / 4; m <<= 1) {
                const bool upper = (lane & m) != 0;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float w = __shfl_xor_sync(kFull, v[j], m);
                    v[j] = upper ? __fsub_rn(w, v[j]) : __fadd_rn(v[j], w);
                }
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) v[j] = __fmul_rn(v[j], cn);
            t.set(r, v);
        }
    }
}

template <typename InT, int CPT, int AXIS, bool HAD>
__device__ __forceinline__ void stage_block(const QParams &p, const LaneTile<CPT> &t, int64_t r0,
                                            int64_t c0, int RB, bool ok, int lane)
{
    load_tile<InT, CPT>(p, t, r0, c0, RB, ok);
    if constexpr (HAD) rotate_tile<AXIS>(t, p.had, RB, lane);
}

// E2M1 round-to-nearest-even, no macro scale or offset, on one staged RB-row
// tile (lane's CPT columns at t): one statistic pass (NaN-propagating abs
// max) and one encode pass with packed binary32 pairs; codes, scales and
// the fidelity sums.
template <int CPT, int AXIS>
__device__ __forceinline__ void col_fast_tile(const QParams &p, const LaneTile<CPT> &t, int64_t r0, int64_t c0,
                                              int RB, bool ok, int lane, float sT, bool stats, Acc &acc)
{
    constexpr int G2 = 32 / CPT;            // lanes of a 2D tile row
        constexpr int NSF = (AXIS == AX_COL) ? CPT : 1;
        float a[NSF], mabs[NSF];
#pragma unroll
        for (int s2 = 0; s2 < NSF; ++s2) { a[s2] = 0.0f; mabs[s2] = FLT_MAX; }
        if constexpr (CPT == 8) {
            // bf16 pairs straight from the tile: |x| by masking the
            // sign bits, NaN-propagating max and min per column pair
            __nv_bfloat162 am[4], mn[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                am[i] = __float2bfloat162_rn(0.0f);
                mn[i] = __float2bfloat162_rn(__uint_as_float(0x7f800000u));
            }
            for (int r = 0; r < RB; ++r) {
                const uint4 u = t.base[r * 32];
                const uint32_t wv[4] = {u.x & 0x7fff7fffu, u.y & 0x7fff7fffu, u.z & 0x7fff7fffu,
                                        u.w & 0x7fff7fffu};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&wv[i]);
                    am[i] = __hmax2_nan(am[i], b);
                    mn[i] = __hmin2(mn[i], b);
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 fa = __bfloat1622float2(am[i]), fm = __bfloat1622float2(mn[i]);
                const int s0 = (AXIS == AX_COL) ? 2 * i : 0, s1 = (AXIS == AX_COL) ? 2 * i + 1 : 0;
                a[s0] = fmax_nan(a[s0], fa.x);
                a[s1] = fmax_nan(a[s1], fa.y);
                mabs[s0] = fminf(mabs[s0], fm.x);
                mabs[s1] = fminf(mabs[s1], fm.y);
            }
        } else {
            for (int r = 0; r < RB; ++r) {
                float v[CPT];
                t.get(r, v);
#pragma unroll
                for (int j = 0; j < CPT; ++j) {
                    const int s2 = (AXIS == AX_COL) ? j : 0;
                    a[s2] = fmax_nan(a[s2], fabsf(v[j]));
                    mabs[s2] = fminf(mabs[s2], fabsf(v[j]));
                }
            }
        }
        BlockScale bsf[NSF];
#pragma unroll
        for (int s2 = 0; s2 < NSF; ++s2) {
            int bad = !(a[s2] <= FLT_MAX);
            float aa = bad ? 0.0f : a[s2];
            if (AXIS == AX_2D) {
                aa = grp_max(aa, G2);
                bad = grp_or(bad, G2);
                mabs[s2] = grp_min(mabs[s2], G2);
            }
            bsf[s2] = block_scale(p.ed, p.sd, aa, bad, sT);
        }
        if (ok) {
            if (AXIS == AX_COL) {
                uint8_t *dst = p.scales + (r0 / RB) * p.cols + c0;
                uint32_t w0 = 0, w1 = 0;
#pragma unroll
                for (int j = 0; j < CPT; ++j) {
                    if (j < 4) w0 |= bsf[(AXIS == AX_COL) ? j : 0].code << (8 * j);
                    else w1 |= bsf[(AXIS == AX_COL) ? j : 0].code << (8 * (j - 4));
                }
                if constexpr (CPT == 8) *reinterpret_cast<uint2 *>(dst) = make_uint2(w0, w1);
                else *reinterpret_cast<uint32_t *>(dst) = w0;
            } else if ((lane & (G2 - 1)) == 0) {
                p.scales[(r0 / 32) * (p.cols / 32) + c0 / 32] = (uint8_t)bsf[0].code;
            }
        }
        const bool nearest = p.sd.fmt != S_E8M0 && p.sd.rule == R_NEAREST;
        float deqT[NSF];
#pragma unroll
        for (int s2 = 0; s2 < NSF; ++s2)
            deqT[s2] = bsf[s2].nan ? __uint_as_float(0x7fc00000u)
                     : nearest ? __fmul_rn(bsf[s2].deq, sT) : bsf[s2].deq;
        float2 sx2 = make_float2(0.f, 0.f), se2 = sx2, sb2 = sx2;
        int qz = 0;                      // zero-magnitude codes of the lane
        for (int r = 0; r < RB; ++r) {
            const int64_t e0 = (r0 + r) * p.cols + c0;
            float v[CPT];
            t.get(r, v);
            float s8[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
            for (int j = 0; j < CPT; j += 2) {
                const int sa = (AXIS == AX_COL) ? j : 0, sb_ = (AXIS == AX_COL) ? j + 1 : 0;
                const float2 pr = __fmul2_rn(make_float2(v[j], v[j + 1]),
                                             make_float2(bsf[sa].inv, bsf[sb_].inv));
                s8[j] = bsf[sa].zero ? 0.0f : pr.x;
                s8[j + 1] = bsf[sb_].zero ? 0.0f : pr.y;
            }
            uint32_t lo = cvt_e2m1x8(s8);
            if (CPT == 4) lo &= 0xffffu;
            if (ok) {
                uint8_t *dst = static_cast<uint8_t *>(p.codes) + e0 / 2;
                if constexpr (CPT == 8) *reinterpret_cast<uint32_t *>(dst) = lo;
                else *reinterpret_cast<uint16_t *>(dst) = (uint16_t)lo;
            }
            if (stats && ok) {
                float q[8];
                e2m1x8_values_alu(lo, q);
#pragma unroll
                for (int j = 0; j < CPT; j += 2) {
                    const int sa = (AXIS == AX_COL) ? j : 0, sb_ = (AXIS == AX_COL) ? j + 1 : 0;
                    const float2 yv = make_float2(v[j], v[j + 1]);
                    const float2 d = __ffma2_rn(make_float2(q[j], q[j + 1]),
                                                make_float2(-deqT[sa], -deqT[sb_]), yv);
                    se2 = __ffma2_rn(d, d, se2);
                    sx2 = __ffma2_rn(yv, yv, sx2);
                    sb2 = __fadd2_rn(sb2, d);
                }
                qz += e2m1_zero_codes8(lo) - (8 - CPT);
            }
        }
        if (stats && ok) {
            acc.x2 += (double)(sx2.x + sx2.y);
            acc.e2 += (double)(se2.x + se2.y);
            acc.e += -(double)(sb2.x + sb2.y);
            // flushed = zero codes - exact zeros, NaN blocks (all codes
            // zero) left out
            int ftz = qz;
#pragma unroll
            for (int s2 = 0; s2 < NSF; ++s2) {
                int xz = 0;
                if (mabs[s2] == 0.0f)
                    for (int r = 0; r < RB; ++r) {
                        float v[CPT];
                        t.get(r, v);
#pragma unroll
                        for (int j = 0; j < CPT; ++j)
                            if ((AXIS == AX_COL) ? j == s2 : true) xz += (v[j] == 0.0f);
                    }
                const int n_lane = (AXIS == AX_COL) ? RB : RB * CPT;
                acc.nz += (double)(n_lane - xz);
                ftz -= bsf[s2].nan ? n_lane : xz;
            }
            acc.ftz += (double)ftz;
        }
}

template <typename InT, int CPT, int AXIS, bool FAST, bool HAD>
__global__ void __launch_bounds__(kColThreads) k_quant_col(const QParams p)
{
    extern __shared__ uint4 smem[];
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const LaneTile<CPT> t{smem + w * 32 * 32 + lane};
    // 2D MBS: per-row macro scale and its reciprocal, per lane
    float2 *rowsm = reinterpret_cast<float2 *>(smem + kColWarps * 32 * 32) + w * 32 * 32 + lane;

    const int RB = (AXIS == AX_2D) ? 32 : p.block;
    const int64_t ncc = p.cols / CPT;
    const int64_t nwg = (ncc + 31) / 32;
    const int NB = (AXIS == AX_COL && p.mbs) ? 128 / RB : 1;
    const int64_t nitems = (p.rows / ((int64_t)RB * NB)) * nwg;
    const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const bool stats = p.partials != nullptr;
    const float sT = launch_tensor_scale(p);
    constexpr int G2 = 32 / CPT;            // lanes of a 2D tile row
    constexpr int MG = 128 / CPT;           // lanes of a 1 x 128 macro block (2D)
    constexpr int NS = (AXIS == AX_COL) ? CPT : 1;   // blocks held by a lane
    const bool raw_max = !FAST && p.ed.is_int && p.asym;
    Acc acc = {0, 0, 0, 0, 0};

    for (int64_t item = gw; item < nitems; item += nw) {
        const int64_t rg = item / nwg, wg = item - rg * nwg;
        const int64_t cc = wg * 32 + lane;
        const bool ok = cc < ncc;
        const int64_t c0 = cc * CPT;
        const int64_t r0g = rg * (int64_t)RB * NB;

        // column-axis MBS: macro scale per column over the 128 rows (first pass)
        float smc[CPT], invmc[CPT];
#pragma unroll
        for (int j = 0; j < CPT; ++j) { smc[j] = 1.0f; invmc[j] = 1.0f; }
        if (AXIS == AX_COL && p.mbs) {
            float m[CPT];
            int badc[CPT];
#pragma unroll
            for (int j = 0; j < CPT; ++j) { m[j] = 0.0f; badc[j] = 0; }
            for (int b = 0; b < NB; ++b) {
                stage_block<InT, CPT, AXIS, HAD>(p, t, r0g + (int64_t)b * RB, c0, RB, ok, lane);
                for (int r = 0; r < RB; ++r) {
                    float v[CPT];
                    t.get(r, v);
#pragma unroll
                    for (int j = 0; j < CPT; ++j) {
                        badc[j] |= nonfinite(v[j]);
                        m[j] = fmaxf(m[j], fabsf(v[j]));
                    }
                }
            }
            uint32_t w0 = 0, w1 = 0;
#pragma unroll
            for (int j = 0; j < CPT; ++j) {
                const uint32_t code = macro_code(p.ed, m[j], badc[j]);
                smc[j] = e4m3_value(code);
                invmc[j] = __fdiv_rn(1.0f, smc[j]);
                if (j < 4) w0 |= code << (8 * j);
                else w1 |= code << (8 * (j - 4));
            }
            if (ok) {
                uint8_t *dst = p.macro + rg * p.cols + c0;
                if constexpr (CPT == 8) *reinterpret_cast<uint2 *>(dst) = make_uint2(w0, w1);
                else *reinterpret_cast<uint32_t *>(dst) = w0;
            }
        }

        for (int b = 0; b < NB; ++b) {
            const int64_t r0 = r0g + (int64_t)b * RB;
            stage_block<InT, CPT, AXIS, HAD>(p, t, r0, c0, RB, ok, lane);
            if (p.rotated && ok) {
                for (int r = 0; r < RB; ++r) {
                    float v[CPT];
                    t.get(r, v);
                    float *dst = p.rotated + (r0 + r) * p.cols + c0;
#pragma unroll
                    for (int j = 0; j < CPT; j += 4)
                        *reinterpret_cast<float4 *>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
                }
            }

            // E2M1 round-to-nearest-even without macro scale or offset: one
            // statistic pass (NaN-propagating abs max) and one encode pass with
            // packed binary32 pairs
            if constexpr (FAST) {
                if (!p.mbs) {
                    col_fast_tile<CPT, AXIS>(p, t, r0, c0, RB, ok, lane, sT, stats, acc);
                    continue;
                }
            }

            // 2D MBS: one macro scale per row and 128-column group
            if (AXIS == AX_2D && p.mbs) {
                for (int r = 0; r < 32; ++r) {
                    float v[CPT];
                    t.get(r, v);
                    float m = 0.0f;
                    int bad = 0;
#pragma unroll
                    for (int j = 0; j < CPT; ++j) {
                        bad |= nonfinite(v[j]);
                        m = fmaxf(m, fabsf(v[j]));
                    }
                    m = grp_max(m, MG);
                    bad = grp_or(bad, MG);
                    const uint32_t code = macro_code(p.ed, m, bad);
                    const float sm = e4m3_value(code);
                    rowsm[r * 32] = make_float2(sm, __fdiv_rn(1.0f, sm));
                    if (ok && (lane & (MG - 1)) == 0)
                        p.macro[(r0 + r) * (p.cols / 128) + c0 / 128] = (uint8_t)code;
                }
            }

            // values entering the block rule (after the macro scale)
            auto xq_row = [&](int r, float v[CPT]) {
                t.get(r, v);
                if (p.mbs) {
                    if (AXIS == AX_COL) {
#pragma unroll
                        for (int j = 0; j < CPT; ++j) v[j] = __fmul_rn(v[j], invmc[j]);
                    } else {
                        const float inv = rowsm[r * 32].y;
#pragma unroll
                        for (int j = 0; j < CPT; ++j) v[j] = __fmul_rn(v[j], inv);
                    }
                }
            };

            int bad[NS];
            float mn[NS], mx[NS], o[NS], alpha[NS];
#pragma unroll
            for (int s = 0; s < NS; ++s) {
                bad[s] = 0; mn[s] = FLT_MAX; mx[s] = -FLT_MAX; o[s] = 0.0f; alpha[s] = 0.0f;
            }
            for (int r = 0; r < RB; ++r) {
                float v[CPT];
                xq_row(r, v);
#pragma unroll
                for (int j = 0; j < CPT; ++j) {
                    const int s = (AXIS == AX_COL) ? j : 0;
                    bad[s] |= nonfinite(v[j]);
                    mn[s] = fminf(mn[s], v[j]);
                    mx[s] = fmaxf(mx[s], v[j]);
                    alpha[s] = fmaxf(alpha[s], fabsf(v[j]));
                }
            }
            if (AXIS == AX_2D) {
                bad[0] = grp_or(bad[0], G2);
                mn[0] = grp_min(mn[0], G2);
                mx[0] = grp_max(mx[0], G2);
            }
            if (!FAST && p.asym) {
#pragma unroll
                for (int s = 0; s < NS; ++s) {
                    if (!bad[s])
                        o[s] = p.ed.is_int ? bf16_round(mn[s])
                                           : bf16_round(__fmul_rn(__fadd_rn(mx[s], mn[s]), 0.5f));
                    alpha[s] = 0.0f;
                }
                for (int r = 0; r < RB; ++r) {
                    float v[CPT];
                    xq_row(r, v);
#pragma unroll
                    for (int j = 0; j < CPT; ++j) {
                        const int s = (AXIS == AX_COL) ? j : 0;
                        const float d = __fsub_rn(v[j], o[s]);
                        alpha[s] = fmaxf(alpha[s], raw_max ? d : fabsf(d));
                    }
                }
            }
            if (AXIS == AX_2D) alpha[0] = grp_max(alpha[0], G2);

            BlockScale bs[NS];
#pragma unroll
            for (int s = 0; s < NS; ++s) bs[s] = block_scale(p.ed, p.sd, alpha[s], bad[s], sT);

            if (ok) {
                if (AXIS == AX_COL) {
                    uint8_t *dst = p.scales + (r0 / RB) * p.cols + c0;
                    uint32_t w0 = 0, w1 = 0;
#pragma unroll
                    for (int j = 0; j < CPT; ++j) {
                        if (j < 4) w0 |= bs[j].code << (8 * j);
                        else w1 |= bs[j].code << (8 * (j - 4));
                    }
                    if constexpr (CPT == 8) *reinterpret_cast<uint2 *>(dst) = make_uint2(w0, w1);
                    else *reinterpret_cast<uint32_t *>(dst) = w0;
                    if (!FAST && p.asym) {
                        uint16_t *od = p.offsets + (r0 / RB) * p.cols + c0;
#pragma unroll
                        for (int j = 0; j < CPT; ++j) od[j] = __bfloat16_as_ushort(__float2bfloat16_rn(o[j]));
                    }
                } else if ((lane & (G2 - 1)) == 0) {
                    const int64_t bi = (r0 / 32) * (p.cols / 32) + c0 / 32;
                    p.scales[bi] = (uint8_t)bs[0].code;
                    if (!FAST && p.asym) p.offsets[bi] = __bfloat16_as_ushort(__float2bfloat16_rn(o[0]));
                }
            }

            // elements, row by row
            for (int r = 0; r < RB; ++r) {
                const int64_t e0 = (r0 + r) * p.cols + c0;
                float v[CPT], q[CPT];
                xq_row(r, v);
                uint32_t lo = 0;
                if constexpr (FAST) {
                    float s8[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
                    for (int j = 0; j < CPT; ++j) {
                        const int s = (AXIS == AX_COL) ? j : 0;
                        s8[j] = bs[s].zero ? 0.0f : __fmul_rn(v[j], bs[s].inv);
                    }
                    lo = cvt_e2m1x8(s8);
                    if (CPT == 4) lo &= 0xffffu;
                    if (stats)
#pragma unroll
                        for (int j = 0; j < CPT; ++j) q[j] = e2m1_value((lo >> (4 * j)) & 0xfu);
                } else {
                    uint4 wa = make_uint4(0, 0, 0, 0), wb = wa;
                    if (p.round_mode == RD_SR) {
                        wa = element_words(p.seed, (uint64_t)e0 >> 2);
                        if (CPT == 8) wb = element_words(p.seed, ((uint64_t)e0 >> 2) + 1);
                    }
#pragma unroll
                    for (int j = 0; j < CPT; ++j) {
                        const int s = (AXIS == AX_COL) ? j : 0;
                        const uint32_t u = word_of(j < 4 ? wa : wb, j & 3);
                        uint32_t code = 0;
                        q[j] = 0.0f;
                        if (!bs[s].zero) {
                            float vv = v[j];
                            if (p.asym) vv = __fsub_rn(vv, o[s]);
                            code = encode_elem(p.ed, p.round_mode, __fmul_rn(vv, bs[s].inv), u, q[j]);
                        }
                        lo |= code << ((p.ed.code_bits == 4 ? 4 : 8) * j);
                    }
                }
                if (ok) {
                    if (p.ed.code_bits == 4) {
                        uint8_t *dst = static_cast<uint8_t *>(p.codes) + e0 / 2;
                        if constexpr (CPT == 8) *reinterpret_cast<uint32_t *>(dst) = lo;
                        else *reinterpret_cast<uint16_t *>(dst) = (uint16_t)lo;
                    } else {
                        *reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(p.codes) + e0) = lo;
                    }
                }
                if (stats && ok) {
                    float y[CPT], xh[CPT];
                    t.get(r, y);
                    const float sm_r = (AXIS == AX_2D && p.mbs) ? rowsm[r * 32].x : 1.0f;
#pragma unroll
                    for (int j = 0; j < CPT; ++j) {
                        const int s = (AXIS == AX_COL) ? j : 0;
                        const float sm = (AXIS == AX_COL) ? smc[j] : sm_r;
                        xh[j] = deq_value(p, q[j], bs[s], sm, o[s], sT);
                    }
                    acc_add<CPT>(acc, y, xh);
                }
            }
        }
    }
    finish_launch(p, acc);
}

// Tensor absmax with the rotation along columns (column axis with rotation)
template <typename InT>
__global__ void __launch_bounds__(kColThreads) k_amax_col(const QParams p)
{
    extern __shared__ uint4 smem[];
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const LaneTile<4> t{smem + w * 32 * 32 + lane};
    const int RB = p.block;
    const int64_t ncc = p.cols / 4;
    const int64_t nwg = (ncc + 31) / 32;
    const int64_t nitems = (p.rows / RB) * nwg;
    const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    float m = 0.0f;
    for (int64_t item = gw; item < nitems; item += nw) {
        const int64_t rg = item / nwg, wg = item - rg * nwg;
        const int64_t cc = wg * 32 + lane;
        const bool ok = cc < ncc;
        stage_block<InT, 4, AX_COL, true>(p, t, rg * RB, cc * 4, RB, ok, lane);
        for (int r = 0; r < RB; ++r) {
            float v[4];
            t.get(r, v);
#pragma unroll
            for (int j = 0; j < 4; ++j) m = fmaxf(m, fabsf(v[j]));
        }
    }
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
    if (lane == 0 && m > 0.0f) atomicMax(p.amax_word, __float_as_uint(m));
}

// ---------------------------------------------------------------------------
// bf16 input, E2M1 round-to-nearest-even, symmetric, no macro scale or
// rotation: column-wise B x 1 blocks and 2D 32 x 32 tiles.  Every warp owns
// two tile buffers of RB rows x 128 columns (RB = B, or 32 for 2D; 256 bytes a
// row) and keeps the next tile's 16-byte cp.async copies in flight while it
// works the current one; lane l works columns 4l .. 4l + 3 of the tile (an
// 8-byte slot of every row).  The column statistics are taken on the packed
// bf16x2 words (halfwise maximum and minimum of magnitudes), each element is
// scaled in one mixed-precision multiply-add (y * 2^-k exactly; nearest
// scales: widened, then multiplied), and the fidelity sums are formed on the
// scaled values, s - q with q decoded by the conversion instruction, times
// the block's scale once per block.  One launch may cover several tensors
// (a group), the CTAs split among them.
constexpr int kColxWarps = 12;
constexpr int kColxThreads = kColxWarps * 32;
constexpr int kColxTileRows = 32;
constexpr int kColxCols = 128;                              // columns of a tile
constexpr int kColxBufBytes = kColxTileRows * kColxCols * 2;    // 8 KB

__device__ __forceinline__ uint32_t bfx_absmax(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
__device__ __forceinline__ uint32_t bfx_absmin(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("min.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
// |half h| of a bf16x2 word as binary32
__device__ __forceinline__ float bfx_half_abs(uint32_t w, int h)
{
    return fabsf(__uint_as_float(h ? (w & 0xffff0000u) : (w << 16)));
}
// the two bf16 values of a word times the bf16 values k0 / k1 (low 16 bits),
// each product rounded once to binary32
__device__ __forceinline__ float2 bfx_scale2(uint32_t w, uint32_t k0, uint32_t k1)
{
    float a, b;
    asm("{\n\t.reg .b16 y0, y1, c0, c1, cx;\n\t.reg .f32 z;\n\t"
        "mov.b32 {y0, y1}, %2;\n\t"
        "mov.b32 {c0, cx}, %3;\n\t"
        "mov.b32 {c1, cx}, %4;\n\t"
        "mov.f32 z, 0f80000000;\n\t"
        "fma.rn.f32.bf16 %0, y0, c0, z;\n\t"
        "fma.rn.f32.bf16 %1, y1, c1, z;\n\t}"
        : "=f"(a), "=f"(b) : "r"(w), "r"(k0), "r"(k1));
    return make_float2(a, b);
}
// two rows of four binary32 values -> eight E2M1 nibbles: the first row in
// bits 0..15 (its first value in bits 0..3), the second in bits 16..31
__device__ __forceinline__ uint32_t cvt_e2m1x4x2(const float v[8])
{
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r) : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return r;
}
// A launch over up to kFastGroupMax tensors of one configuration: the CTAs
// are split among the tensors (cta0 prefix), every CTA works on one tensor;
// p[0] also carries the shared configuration.
struct ColxGroup {
    QParams p[kFastGroupMax];
    uint32_t cta0[kFastGroupMax + 1];
    int n;
};

template <int AXIS, bool STATS, bool NEAR, int RB>
__global__ void __launch_bounds__(kColxThreads) k_quant_colx(const __grid_constant__ ColxGroup g)
{
    // RB: rows of a block (the column block size, or 32 for 2D tiles)
    constexpr int NS = (AXIS == AX_COL) ? 4 : 1;          // blocks a lane holds per tile
    extern __shared__ uint4 smem[];
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // this CTA's tensor, and its place among the tensor's CTAs
    int item = 0;
    while (item + 1 < g.n && blockIdx.x >= g.cta0[item + 1]) ++item;
    const QParams &pc = g.p[0];
    const QParams &p = g.p[item];
    const uint32_t cta = blockIdx.x - g.cta0[item], ncta = g.cta0[item + 1] - g.cta0[item];
    uint8_t *const bufs = reinterpret_cast<uint8_t *>(smem) + (size_t)w * 2 * kColxBufBytes;
    // the tensor's shape and outputs, read once from the launch parameters
    const int64_t cols = p.cols, rows = p.rows;
    uint8_t *const codes0 = static_cast<uint8_t *>(p.codes);
    uint8_t *const scales0 = p.scales;
    const int64_t ngc = (cols + kColxCols - 1) / kColxCols;
    const int64_t nitems = (rows / RB) * ngc;
    const int64_t gw = (int64_t)cta * kColxWarps + w, nw = (int64_t)ncta * kColxWarps;
    const float sT = launch_tensor_scale(p, cta == 0);
    // nearest scales: s_b s_T and its reciprocal for every scale code, once per CTA
    __shared__ float2 near_tab[NEAR ? 256 : 1];
    if constexpr (NEAR)
        for (int c = threadIdx.x; c < 256; c += blockDim.x) {
            const float d = __fmul_rn(ue_value(pc.sd, (uint32_t)c), sT);
            near_tab[c] = c < pc.sd.ue_nan_code ? make_float2(d, __fdiv_rn(1.0f, d))
                                               : make_float2(__uint_as_float(0x7fc00000u), 0.0f);
        }
    __syncthreads();
    NearScale ns;
    ns.maxv = pc.ed.maxv;
    ns.r_max = __fdiv_rn(1.0f, pc.ed.maxv);
    ns.sT = sT;
    ns.r_T = (sT >= 0x1p-125f && sT <= 0x1p125f) ? __fdiv_rn(1.0f, sT) : 0.0f;
    {
        const float ms = __fmul_rn(pc.ed.maxv, sT);
        ns.c = (ms >= 0x1p-125f && ms <= 0x1p125f) ? __fdiv_rn(1.0f, ms) : 0.0f;
    }
    ns.tab = near_tab;
    const bool e8m0 = !NEAR && pc.sd.fmt == S_E8M0;
    const float thr_m = e8m0_threshold(pc.ed, pc.sd);
    const uint8_t *const xb = static_cast<const uint8_t *>(p.x);
    const int64_t pitch = cols * 2;                          // bytes per row
    Acc acc = {0, 0, 0, 0, 0};

    // the tile's RB rows x 256 bytes as 16-byte copies, RB / 2 per lane
    auto issue = [&](int64_t item, uint8_t *buf) {
        const int64_t rg = item / ngc, cg = item - rg * ngc;
#pragma unroll
        for (int k = 0; k < RB / 2; ++k) {
            const int f = k * 32 + lane, r = f >> 4, ch = f & 15;
            const int64_t cb = cg * (kColxCols * 2) + ch * 16;
            const bool in = cb < pitch;
            const uint8_t *src = in ? xb + (rg * RB + r) * pitch + cb : xb;
            cp_async16(buf + r * 256 + ch * 16, src, in);
        }
        asm volatile("cp.async.commit_group;\n" ::: "memory");
    };

    int cur = 0;
    if (gw < nitems) issue(gw, bufs);
    for (int64_t item = gw; item < nitems; item += nw, cur ^= 1) {
        const uint2 *b = reinterpret_cast<const uint2 *>(bufs + cur * kColxBufBytes) + lane;
        if (item + nw < nitems) {
            // the other buffer was read in the previous iteration by every lane
            __syncwarp();
            issue(item + nw, bufs + (cur ^ 1) * kColxBufBytes);
            asm volatile("cp.async.wait_group 1;\n" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;\n" ::: "memory");
        }
        __syncwarp();                    // every lane's copies of this tile have landed
        const int64_t rg = item / ngc, cg = item - rg * ngc;
        const int64_t c0 = cg * kColxCols + lane * 4;
        const bool ok = c0 < cols;
        const int64_t r0 = rg * RB;

        // column statistics on the packed words (two chains per word)
        uint32_t am[4] = {0u, 0u, 0u, 0u}, mn[4] = {0x7f807f80u, 0x7f807f80u, 0x7f807f80u, 0x7f807f80u};
#pragma unroll
        for (int r = 0; r < RB; r += 2) {
            const uint2 u0 = b[r * 32], u1 = b[(r + 1) * 32];
            am[0] = bfx_absmax(am[0], u0.x);
            am[1] = bfx_absmax(am[1], u0.y);
            am[2] = bfx_absmax(am[2], u1.x);
            am[3] = bfx_absmax(am[3], u1.y);
            if (STATS) {
                mn[0] = bfx_absmin(mn[0], u0.x);
                mn[1] = bfx_absmin(mn[1], u0.y);
                mn[2] = bfx_absmin(mn[2], u1.x);
                mn[3] = bfx_absmin(mn[3], u1.y);
            }
        }
        float a[4], mabs[4];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const uint32_t m = bfx_absmax(am[i], am[2 + i]);
            a[2 * i] = bfx_half_abs(m, 0);
            a[2 * i + 1] = bfx_half_abs(m, 1);
            const uint32_t n = bfx_absmin(mn[i], mn[2 + i]);
            mabs[2 * i] = bfx_half_abs(n, 0);
            mabs[2 * i + 1] = bfx_half_abs(n, 1);
        }

        // shared scales: one per column (column axis) or per 32 x 32 tile (8 lanes)
        BlockScale bs[NS];
        if constexpr (AXIS == AX_COL) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int bad = !(a[j] <= FLT_MAX);
                bs[j] = NEAR ? near_block_scale(pc.sd, ns, bad ? 0.0f : a[j], bad)
                      : e8m0 ? e8m0_block_scale(bad ? 0.0f : a[j], bad, pc.ed.emax, thr_m)
                             : block_scale(pc.ed, pc.sd, bad ? 0.0f : a[j], bad, sT);
            }
        } else {
            float m = fmax_nan(fmax_nan(a[0], a[1]), fmax_nan(a[2], a[3]));
            int bad = !(m <= FLT_MAX);
            m = grp_max(bad ? 0.0f : m, 8);
            bad = grp_or(bad, 8);
            bs[0] = NEAR ? near_block_scale(pc.sd, ns, m, bad)
                  : e8m0 ? e8m0_block_scale(m, bad, pc.ed.emax, thr_m)
                         : block_scale(pc.ed, pc.sd, m, bad, sT);
        }
        if (ok) {
            if constexpr (AXIS == AX_COL) {
                const uint32_t w0 = bs[0].code | (bs[1].code << 8) | (bs[2].code << 16) | (bs[3].code << 24);
                *reinterpret_cast<uint32_t *>(scales0 + (r0 / RB) * cols + c0) = w0;
            } else if ((lane & 7) == 0) {
                scales0[(r0 / 32) * (cols / 32) + c0 / 32] = (uint8_t)bs[0].code;
            }
        }

        // per column: multiplier (bf16 bits for the power-of-two rules), the
        // nibble mask of flushed blocks, dequantization and reference factors
        uint32_t kb[4], zmask = 0xffffu;
        float inv[4], X[4], R[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const BlockScale &s = bs[(AXIS == AX_COL) ? j : 0];
            const bool flush = s.zero && !s.nan;
            // the scaled values s and their reference factor X (y = X s):
            // a flushed block is scaled by a power of two from its column's
            // maximum (its codes are zero), a non-finite one not at all
            const float2 pp = pow2_near_inv(a[j]);
            inv[j] = s.nan ? 1.0f : flush ? pp.x : s.inv;
            kb[j] = NEAR ? 0x3f80u : (__float_as_uint(inv[j]) >> 16);
            if (s.zero) zmask &= ~(0xfu << (4 * j));
            X[j] = s.nan ? __uint_as_float(0x7fc00000u) : flush ? pp.y : s.deq;
            R[j] = s.nan ? 1.0f : X[j];
        }

        float2 re2[2], rb2[2], sx2[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            re2[i] = make_float2(0.f, 0.f);
            rb2[i] = re2[i];
            sx2[i] = re2[i];
        }
        int qz = 0;
        uint8_t *const codes = codes0 + (r0 * cols + c0) / 2;
        const uint32_t zmask2 = zmask | (zmask << 16);
        // two rows a step: their eight codes share one word (row r in the low
        // half, row r + 1 in the high half), one mask, one decode and one
        // zero count
#pragma unroll 4
        for (int r = 0; r < RB; r += 2) {
            float s8[8];
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const uint2 u = b[(r + rr) * 32];
                const uint32_t v[2] = {u.x, u.y};
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    float2 sv = bfx_scale2(v[i], kb[2 * i], kb[2 * i + 1]);
                    if (NEAR) sv = __fmul2_rn(sv, make_float2(inv[2 * i], inv[2 * i + 1]));
                    s8[4 * rr + 2 * i] = sv.x;
                    s8[4 * rr + 2 * i + 1] = sv.y;
                }
            }
            const uint32_t word = cvt_e2m1x4x2(s8) & zmask2;
            if (ok) {
                *reinterpret_cast<uint16_t *>(codes + (int64_t)r * (cols / 2)) = (uint16_t)word;
                *reinterpret_cast<uint16_t *>(codes + (int64_t)(r + 1) * (cols / 2)) = (uint16_t)(word >> 16);
            }
            if (STATS) {
                uint32_t h[4];
                asm("{\n\t.reg .b8 c0, c1, c2, c3;\n\t"
                    "mov.b32 {c0, c1, c2, c3}, %4;\n\t"
                    "cvt.rn.f16x2.e2m1x2 %0, c0;\n\t"
                    "cvt.rn.f16x2.e2m1x2 %1, c1;\n\t"
                    "cvt.rn.f16x2.e2m1x2 %2, c2;\n\t"
                    "cvt.rn.f16x2.e2m1x2 %3, c3;\n\t}"
                    : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3]) : "r"(word));
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i = e & 1;                   // column pair
                    const float2 d = sub_f16x2_from(s8[2 * e], s8[2 * e + 1], h[e]);   // s - q
                    re2[i] = __ffma2_rn(d, d, re2[i]);
                    rb2[i] = __fadd2_rn(rb2[i], d);
                    const float2 sv = make_float2(s8[2 * e], s8[2 * e + 1]);
                    sx2[i] = __ffma2_rn(sv, sv, sx2[i]);                     // y = R s
                }
                qz += 8 - __popc(((word & 0x77777777u) + 0x77777777u) & 0x88888888u);
            }
        }
        if (STATS && ok) {
            // y - x_hat = X (s - q) per column; reference sums R^2 sum s^2
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int i = j >> 1;
                const float e = (j & 1) ? re2[i].y : re2[i].x, bb = (j & 1) ? rb2[i].y : rb2[i].x;
                const float sx = (j & 1) ? sx2[i].y : sx2[i].x;
                const double Xd = (double)X[j], Rd = (double)R[j];
                acc.e2 += (double)e * Xd * Xd;
                acc.e -= (double)bb * Xd;
                acc.x2 += (double)sx * Rd * Rd;
            }
            // exact zeros (rare), nonzero and flushed counts; NaN blocks
            // (all codes zero) are not flushes
            int xzt = 0, nanz = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                int xz = 0;
                if (mabs[j] == 0.0f)
#pragma unroll 1
                    for (int r = 0; r < RB; ++r) {
                        const uint2 u = b[r * 32];
                        const uint32_t vv = (j >> 1) ? u.y : u.x;
                        xz += ((vv >> (16 * (j & 1))) & 0x7fffu) == 0u;
                    }
                xzt += xz;
                nanz += bs[(AXIS == AX_COL) ? j : 0].nan ? RB : xz;
            }
            acc.nz += (double)(4 * RB - xzt);
            acc.ftz += (double)(qz - nanz);
        }
    }
    finish_launch(p, acc, cta, ncta);
}

template <int AXIS, bool STATS, bool NEAR, int RB>
int launch_colx_k(const QParams *ps, int n, cudaStream_t st)
{
    auto k = k_quant_colx<AXIS, STATS, NEAR, RB>;
    const size_t smem = (size_t)kColxWarps * 2 * kColxBufBytes;
    const int occ = cached_occupancy(reinterpret_cast<const void *>(k), kColxThreads, smem);
    ColxGroup g;
    memset(&g, 0, sizeof(g));
    uint64_t need[kFastGroupMax];
    for (int i = 0; i < n; ++i) {
        g.p[i] = ps[i];
        const int64_t items = (ps[i].rows / RB) * ((ps[i].cols + kColxCols - 1) / kColxCols);
        need[i] = (uint64_t)((items + kColxWarps - 1) / kColxWarps);     // CTAs with work
    }
    g.n = n;
    uint64_t total = (uint64_t)device_sm_count() * occ;
    if (total > (uint64_t)kMaxPartials) total = kMaxPartials;
    if (total < (uint64_t)n) total = n;
    split_ctas(need, n, total, g.cta0);
    k<<<g.cta0[n], kColxThreads, smem, st>>>(g);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

template <int AXIS, int RB>
int launch_colx_rb(const QParams *ps, int n, cudaStream_t st)
{
    const QParams &p = ps[0];
    const bool near = p.sd.fmt != S_E8M0 && p.sd.rule == R_NEAREST;
    bool stats = false;
    for (int i = 0; i < n; ++i) stats = stats || ps[i].partials != nullptr;
    if (stats)
        return near ? launch_colx_k<AXIS, true, true, RB>(ps, n, st) : launch_colx_k<AXIS, true, false, RB>(ps, n, st);
    return near ? launch_colx_k<AXIS, false, true, RB>(ps, n, st) : launch_colx_k<AXIS, false, false, RB>(ps, n, st);
}

template <int AXIS>
int launch_colx(const QParams *ps, int n, cudaStream_t st)
{
    if constexpr (AXIS == AX_2D) {
        return launch_colx_rb<AXIS, 32>(ps, n, st);
    } else {
        switch (ps[0].block) {
        case 8: return launch_colx_rb<AXIS, 8>(ps, n, st);
        case 16: return launch_colx_rb<AXIS, 16>(ps, n, st);
        case 32: return launch_colx_rb<AXIS, 32>(ps, n, st);
        default: return -1;
        }
    }
}

template <typename K>
int launch_k(K kernel, const QParams &p, int64_t work_warps, size_t smem, cudaStream_t st,
             int *grid_out)
{
    const int g = grid_for(kernel, work_warps, kColThreads, smem);
    kernel<<<g, kColThreads, smem, st>>>(p);
    if (grid_out) *grid_out = g;
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

template <typename InT, int CPT, int AXIS, bool FAST, bool HAD>
int launch_col_k(const QParams &p, cudaStream_t st, int *grid_out)
{
    const int RB = (AXIS == AX_2D) ? 32 : p.block;
    const int NB = (AXIS == AX_COL && p.mbs) ? 128 / RB : 1;
    const int64_t ncc = p.cols / CPT;
    const int64_t items = (p.rows / ((int64_t)RB * NB)) * ((ncc + 31) / 32);
    size_t smem = (size_t)kColWarps * 32 * 32 * 16;
    if (AXIS == AX_2D && p.mbs) smem += (size_t)kColWarps * 32 * 32 * 8;
    return launch_k(k_quant_col<InT, CPT, AXIS, FAST, HAD>, p, items, smem, st, grid_out);
}

template <typename InT, int AXIS>
int launch_axis(const QParams &p, int fast, cudaStream_t st, int *grid_out)
{
    // 8 bf16 columns per lane (16-byte rows) for 4-bit codes without a
    // rotation; otherwise 4 columns held as binary32
    if (p.had) {
        if (fast) return launch_col_k<InT, 4, AXIS, true, true>(p, st, grid_out);
        return launch_col_k<InT, 4, AXIS, false, true>(p, st, grid_out);
    }
    if constexpr (sizeof(InT) == 2) {
        // E2M1 nearest-even without a macro scale: the double-buffered kernel
        if (fast && !p.mbs && p.ed.elem == 0) {
            if (grid_out) *grid_out = 0;
            return launch_colx<AXIS>(&p, 1, st);
        }
        if (p.ed.code_bits == 4) {
            if (fast) return launch_col_k<InT, 8, AXIS, true, false>(p, st, grid_out);
            return launch_col_k<InT, 8, AXIS, false, false>(p, st, grid_out);
        }
    }
    if (fast) return launch_col_k<InT, 4, AXIS, true, false>(p, st, grid_out);
    return launch_col_k<InT, 4, AXIS, false, false>(p, st, grid_out);
}

}  // namespace

int launch_quantize_colx_group(const QParams *ps, int n, int axis, cudaStream_t st)
{
    if (n < 1 || n > kFastGroupMax) return -1;
    return axis == AX_COL ? launch_colx<AX_COL>(ps, n, st) : launch_colx<AX_2D>(ps, n, st);
}

int launch_quantize_col(const QParams &p, int axis, int in_fp32, int fast, cudaStream_t st,
                        int *grid_out)
{
    if (axis == AX_COL)
        return in_fp32 ? launch_axis<float, AX_COL>(p, fast, st, grid_out)
                       : launch_axis<__nv_bfloat16, AX_COL>(p, fast, st, grid_out);
    return in_fp32 ? launch_axis<float, AX_2D>(p, fast, st, grid_out)
                   : launch_axis<__nv_bfloat16, AX_2D>(p, fast, st, grid_out);
}

int launch_amax_col(const QParams &p, int in_fp32, cudaStream_t st)
{
    const int64_t items = (p.rows / p.block) * ((p.cols / 4 + 31) / 32);
    const size_t smem = (size_t)kColWarps * 32 * 32 * 16;
    if (in_fp32) return launch_k(k_amax_col<float>, p, items, smem, st, nullptr);
    return launch_k(k_amax_col<__nv_bfloat16>, p, items, smem, st, nullptr);
}

}  // namespace mxk
