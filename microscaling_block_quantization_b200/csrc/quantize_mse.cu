// MSE-optimal nearest-format block scales and the alternating optimisation
// of the global and group scales ("Bridging the Gap Between Promise and
// Performance for Microscaling FP4 Quantization", sec. 2.2: MSE-optimised
// grids, found per tensor by alternating between the global scale and the
// group scales).
//
// Group step: for a given tensor scale s_T every row block takes the scale
// code c with the smallest squared error
//   SSE(c) = sum_t (x_t - x_hat_t)^2,  x_hat_t = (q_t s_c) s_T,
// q_t the nearest-even E2M1 value of x_t * RN(1 / RN(s_c s_T)), over all
// finite codes of the format (127 for UE4M3, 255 for UE5M3), ties to the
// lower code.  Every SSE is a binary64 sum in element order of binary64
// squares of binary64 differences, each operation rounded on its own (no
// contraction), so the choice is the same wherever it is evaluated.
// Global step: with the codes and u_t = q_t s_c fixed, the least-squares
// s_T = sum x_t u_t / sum u_t^2 (binary64 sums, rounded once to binary32).
// Rounds: kMseRounds; the starting s_T is the amax rule's.
//
// One thread per block; every thread of a CTA walks the codes in the same
// order, reading each code's (s_c, RN(s_c s_T), reciprocal) from a table in
// shared memory.  Global-step passes reduce (sum x u, sum u^2) per CTA into
// the workspace records; the last CTA writes the next s_T.  The final pass
// writes codes, scales and the fused statistics.
#include "mx.h"
#include "quant_common.cuh"

namespace mxk {
namespace {

constexpr int kMseThreads = 128;
constexpr int kMseRounds = 4;
constexpr int kMaxCodes = 255;

struct MseArgs {
    const float *sT_in;     // the tensor scale of this pass (null: 1)
    float *sT_out;          // global-step passes: the next tensor scale
    int ncodes;             // finite scale codes
};

template <typename InT, int B>
__device__ __forceinline__ bool load_block(const QParams &p, int64_t b, float x[B])
{
    bool bad = false;
    if constexpr (sizeof(InT) == 2) {
        const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(p.x) + b * B);
#pragma unroll
        for (int k = 0; k < B / 8; ++k) {
            const uint4 u = __ldg(src + k);
            unpack_bf16x2(u.x, x[8 * k + 0], x[8 * k + 1]);
            unpack_bf16x2(u.y, x[8 * k + 2], x[8 * k + 3]);
            unpack_bf16x2(u.z, x[8 * k + 4], x[8 * k + 5]);
            unpack_bf16x2(u.w, x[8 * k + 6], x[8 * k + 7]);
        }
    } else {
        const float4 *src = reinterpret_cast<const float4 *>(static_cast<const float *>(p.x) + b * B);
#pragma unroll
        for (int k = 0; k < B / 4; ++k) {
            const float4 u = __ldg(src + k);
            x[4 * k + 0] = u.x; x[4 * k + 1] = u.y; x[4 * k + 2] = u.z; x[4 * k + 3] = u.w;
        }
    }
#pragma unroll
    for (int t = 0; t < B; ++t) bad |= nonfinite(x[t]);
    return bad;
}

// nearest-even E2M1 value (saturating) of two binary32 values
__device__ __forceinline__ float2 e2m1_round2(float a, float b)
{
    uint32_t r;
    asm("{\n\t.reg .b8 c;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 c, %2, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, c;\n\t}"
        : "=r"(r) : "f"(a), "f"(b));
    return __half22float2(*reinterpret_cast<__half2 *>(&r));
}

// squared error of the block under one code (binary64, element order)
template <int B>
__device__ __forceinline__ double block_sse(const float x[B], float sb, float inv, bool zero, float sT)
{
    double acc = 0.0;
#pragma unroll
    for (int t = 0; t < B; t += 2) {
        float xh0 = 0.0f, xh1 = 0.0f;
        if (!zero) {
            const float2 q = e2m1_round2(__fmul_rn(x[t], inv), __fmul_rn(x[t + 1], inv));
            xh0 = __fmul_rn(__fmul_rn(q.x, sb), sT);
            xh1 = __fmul_rn(__fmul_rn(q.y, sb), sT);
        }
        const double e0 = __dsub_rn((double)x[t], (double)xh0);
        acc = __dadd_rn(acc, __dmul_rn(e0, e0));
        const double e1 = __dsub_rn((double)x[t + 1], (double)xh1);
        acc = __dadd_rn(acc, __dmul_rn(e1, e1));
    }
    return acc;
}

template <typename InT, int B, bool WRITE>
__global__ void __launch_bounds__(kMseThreads) k_quant_mse(const QParams p, const MseArgs a)
{
    __shared__ float s_sb[kMaxCodes], s_inv[kMaxCodes];
    __shared__ unsigned char s_zero[kMaxCodes];
    const float sT = a.sT_in ? *a.sT_in : 1.0f;
    for (int c = threadIdx.x; c < a.ncodes; c += blockDim.x) {
        const float sb = ue_value(p.sd, (uint32_t)c);
        const float inv = __fdiv_rn(1.0f, __fmul_rn(sb, sT));
        s_sb[c] = sb;
        s_inv[c] = inv;
        s_zero[c] = (sb == 0.0f) || !(inv < __uint_as_float(0x7f800000u));
    }
    if (WRITE && p.ts_mode == TS_COMPUTE && blockIdx.x == 0 && threadIdx.x == 0) *p.tensor_scale = sT;
    __syncthreads();

    const int64_t nblk = p.rows * (p.cols / B);
    const uint32_t S = (uint32_t)(p.cols / B);
    double num = 0.0, den = 0.0;
    Acc acc = {0, 0, 0, 0, 0};
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblk; b += (int64_t)gridDim.x * blockDim.x) {
        float x[B];
        const bool bad = load_block<InT, B>(p, b, x);
        uint32_t code = (uint32_t)p.sd.ue_nan_code;
        float xh[B];
        uint32_t packed[B / 8];
#pragma unroll
        for (int k = 0; k < B / 8; ++k) packed[k] = 0u;
        if (!bad) {
            double best = __longlong_as_double(0x7ff0000000000000ll);
            int bc = 0;
            for (int c = 0; c < a.ncodes; ++c) {
                const double sse = block_sse<B>(x, s_sb[c], s_inv[c], s_zero[c] != 0, sT);
                if (sse < best) {
                    best = sse;
                    bc = c;
                }
            }
            code = (uint32_t)bc;
            const float sb = s_sb[bc], inv = s_inv[bc];
            const bool zero = s_zero[bc] != 0;
#pragma unroll
            for (int t = 0; t < B; t += 2) {
                float2 q = make_float2(0.0f, 0.0f);
                uint32_t byte = 0u;
                if (!zero) {
                    const float v0 = __fmul_rn(x[t], inv), v1 = __fmul_rn(x[t + 1], inv);
                    uint16_t c2;
                    asm("{\n\t.reg .b8 c;\n\t"
                        "cvt.rn.satfinite.e2m1x2.f32 c, %2, %1;\n\t"
                        "cvt.u16.u8 %0, c;\n\t}"
                        : "=h"(c2) : "f"(v0), "f"(v1));
                    byte = c2;
                    q = e2m1_round2(v0, v1);
                }
                packed[t >> 3] |= byte << (4 * (t & 7));
                const float u0 = __fmul_rn(q.x, sb), u1 = __fmul_rn(q.y, sb);
                xh[t] = __fmul_rn(u0, sT);
                xh[t + 1] = __fmul_rn(u1, sT);
                if (!WRITE) {
                    num = __dadd_rn(num, __dmul_rn((double)x[t], (double)u0));
                    num = __dadd_rn(num, __dmul_rn((double)x[t + 1], (double)u1));
                    den = __dadd_rn(den, __dmul_rn((double)u0, (double)u0));
                    den = __dadd_rn(den, __dmul_rn((double)u1, (double)u1));
                }
            }
        } else {
#pragma unroll
            for (int t = 0; t < B; ++t) xh[t] = __uint_as_float(0x7fc00000u);
        }
        if (WRITE) {
            uint8_t *dst = static_cast<uint8_t *>(p.codes) + b * (B / 2);
            if constexpr (B == 8) *reinterpret_cast<uint32_t *>(dst) = packed[0];
            else if constexpr (B == 16) *reinterpret_cast<uint2 *>(dst) = make_uint2(packed[0], packed[1]);
            else *reinterpret_cast<uint4 *>(dst) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
            if (p.sf_gemm) {
                const uint32_t r = (uint32_t)(b / S), j = (uint32_t)(b - (int64_t)r * S);
                p.scales[sf_chunk_index(r, j, S)] = (uint8_t)code;
            } else {
                p.scales[b] = (uint8_t)code;
            }
            if (p.partials) acc_add<B>(acc, x, xh);
        }
    }
    if (WRITE) {
        finish_launch(p, acc);
        return;
    }
    // global step: CTA sums of (sum x u, sum u^2) in a fixed order, then the
    // last CTA's fixed-order sum over the CTAs' records
    __shared__ double sh[kMseThreads / 32][2];
    __shared__ unsigned s_last;
    num = warp_sum(num);
    den = warp_sum(den);
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    if (lane == 0) {
        sh[w][0] = num;
        sh[w][1] = den;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double n0 = 0.0, d0 = 0.0;
        for (int k = 0; k < kMseThreads / 32; ++k) {
            n0 += sh[k][0];
            d0 += sh[k][1];
        }
        double *rec = p.partials + (int64_t)blockIdx.x * kPartialDoubles;
        rec[0] = n0;
        rec[1] = d0;
        __threadfence();
        s_last = atomicAdd(p.ticket, 1u) == gridDim.x - 1;
    }
    __syncthreads();
    if (!s_last || threadIdx.x >= 32) return;
    __threadfence();
    double n1 = 0.0, d1 = 0.0;
    for (unsigned i = threadIdx.x; i < gridDim.x; i += 32) {
        n1 += __ldcg(p.partials + (size_t)i * kPartialDoubles);
        d1 += __ldcg(p.partials + (size_t)i * kPartialDoubles + 1);
    }
    n1 = warp_sum(n1);
    d1 = warp_sum(d1);
    if (threadIdx.x == 0) {
        float next = sT;
        if (d1 > 0.0) {
            const float s = __double2float_rn(n1 / d1);
            if (s > 0.0f && s <= FLT_MAX) next = s;
        }
        *a.sT_out = next;
        *p.ticket = 0u;
    }
}

// s_T of the amax rule from the amax word (then cleared), into the chain
__global__ void k_mse_start(const QParams p, float *sT0)
{
    *sT0 = launch_tensor_scale(p);
    *p.amax_word = 0u;
}

template <typename InT, int B>
int launch_mse_b(const QParams &p, double *records, float *chain, cudaStream_t st)
{
    const int64_t nblk = p.rows * (p.cols / B);
    int64_t g = (nblk + kMseThreads - 1) / kMseThreads;
    const int64_t cap = (int64_t)device_sm_count() * 8;
    if (g > cap) g = cap;
    if (g > kMaxPartials) g = kMaxPartials;
    if (g < 1) g = 1;
    MseArgs a;
    a.ncodes = p.sd.ue_nan_code;
    if (p.ts_mode == TS_COMPUTE) {
        // global-step passes: records and ticket of the workspace
        QParams gp = p;
        gp.partials = records;
        k_mse_start<<<1, 1, 0, st>>>(p, chain);
        for (int r = 0; r < kMseRounds; ++r) {
            a.sT_in = chain + r;
            a.sT_out = chain + r + 1;
            k_quant_mse<InT, B, false><<<(unsigned)g, kMseThreads, 0, st>>>(gp, a);
        }
        a.sT_in = chain + kMseRounds;
    } else {
        a.sT_in = p.ts_mode == TS_GIVEN ? p.tensor_scale : nullptr;
    }
    a.sT_out = nullptr;
    k_quant_mse<InT, B, true><<<(unsigned)g, kMseThreads, 0, st>>>(p, a);
    if (cudaGetLastError() != cudaSuccess) return -1;
    // leave the header zero for the next user of the workspace
    if (p.ts_mode == TS_COMPUTE && cudaMemsetAsync(chain, 0, (kMseRounds + 1) * sizeof(float), st) != cudaSuccess)
        return -1;
    return 0;
}

}  // namespace

// Row-axis E2M1 blocks of 8, 16 or 32 with a UE4M3 / UE5M3 scale and the MSE
// rule.  records: the workspace's per-CTA records (the global-step passes
// reduce through them and p.ticket); chain: kMseRounds + 1 floats of the
// workspace header (the tensor scale of each round, cleared at the end).
int launch_quantize_mse(const QParams &p, double *records, float *chain, int in_fp32, cudaStream_t st)
{
    if (in_fp32) {
        switch (p.block) {
        case 8: return launch_mse_b<float, 8>(p, records, chain, st);
        case 16: return launch_mse_b<float, 16>(p, records, chain, st);
        case 32: return launch_mse_b<float, 32>(p, records, chain, st);
        default: return -1;
        }
    }
    switch (p.block) {
    case 8: return launch_mse_b<__nv_bfloat16, 8>(p, records, chain, st);
    case 16: return launch_mse_b<__nv_bfloat16, 16>(p, records, chain, st);
    case 32: return launch_mse_b<__nv_bfloat16, 32>(p, records, chain, st);
    default: return -1;
    }
}

}  // namespace mxk
