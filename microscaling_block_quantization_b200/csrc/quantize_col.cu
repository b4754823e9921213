// sm_100a block quantizer kernels for column-wise (B x 1) and 2D (32 x 32)
// blocks (fmread summary of Yang et al.: column-wise blocks help activations,
// 2D blocks balance accuracy and efficiency).
//
// Each warp stages a tile of RB rows x (32 lanes x CPT columns) in shared
// memory with asynchronous 16-byte copies (all rows in flight at once), then
// every lane works down its own CPT columns: column axis -> CPT blocks per
// lane; 2D -> one 32 x 32 block per 32 / CPT lanes.  Loads and stores stay
// coalesced along rows; the reduction runs along columns out of shared memory.
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
        if (p.ed.code_bits == 4) {
            if (fast) return launch_col_k<InT, 8, AXIS, true, false>(p, st, grid_out);
            return launch_col_k<InT, 8, AXIS, false, false>(p, st, grid_out);
        }
    }
    if (fast) return launch_col_k<InT, 4, AXIS, true, false>(p, st, grid_out);
    return launch_col_k<InT, 4, AXIS, false, false>(p, st, grid_out);
}

}  // namespace

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
