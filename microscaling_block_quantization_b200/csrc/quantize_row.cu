// sm_100a block quantizer kernels, row axis (the contiguous dimension).
//
// One pass over HBM per tensor: 128-bit vector loads, optional block
// Hadamard rotation, optional macro-block scale, optional offset, block
// statistic by warp shuffles, shared scale, element rounding, nibble packing
// and the fidelity sums of the dequantized values, all in registers.
//
// Method: "Unveiling the Potential of Quantization with MXFP4" (Sec.2 formats,
// Sec.4 OAS and MBS); "Is Finer Better?" (UE4M3/UE5M3 scales, per-tensor
// scale); "Bridging the Gap ... Microscaling FP4 Quantization" (sec. 2.2-2.3,
// rotation fused with quantization); fmread summary of Yang et al. (rounding
// modes, asymmetric scaling, row / column / 2D blocks).
#include <mutex>

#include "quant_common.cuh"

namespace mxk {

// ================================================================ row axis ==
// Thread = chunk of 8 consecutive elements of a row; a block of B elements is
// B/8 consecutive lanes; U chunks per lane in flight.
template <bool FAST>
__device__ __forceinline__ void row_chunk(const QParams &p, int64_t c, bool ok, float y[8],
                                          float sT, Acc &acc, int lane, bool stats)
{
    const int G = p.lanes_per_block;
    if (p.had) hadamard_chunk8(y, p.had, lane);
    if (p.rotated && ok) store8f(p.rotated, c * 8, y);

    float xq[8];
    float sm = 1.0f;
    if (p.mbs) {
        float m = 0.0f;
        int bad = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            bad |= nonfinite(y[j]);
            m = fmaxf(m, fabsf(y[j]));
        }
        m = grp_max(m, 16);
        bad = grp_or(bad, 16);
        uint32_t code = macro_code(p.ed, m, bad);
        sm = e4m3_value(code);
        const float inv = __fdiv_rn(1.0f, sm);
#pragma unroll
        for (int j = 0; j < 8; ++j) xq[j] = __fmul_rn(y[j], inv);
        if (ok && (lane & 15) == 0) p.macro[c >> 4] = (uint8_t)code;
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) xq[j] = y[j];
    }

    int bad = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) bad |= nonfinite(xq[j]);
    bad = grp_or(bad, G);

    float o = 0.0f;
    if (!FAST && p.asym) {
        float mn = xq[0], mx = xq[0];
#pragma unroll
        for (int j = 1; j < 8; ++j) {
            mn = fminf(mn, xq[j]);
            mx = fmaxf(mx, xq[j]);
        }
        mn = grp_min(mn, G);
        mx = grp_max(mx, G);
        if (!bad) o = p.ed.is_int ? bf16_round(mn) : bf16_round(__fmul_rn(__fadd_rn(mx, mn), 0.5f));
#pragma unroll
        for (int j = 0; j < 8; ++j) xq[j] = __fsub_rn(xq[j], o);
    }

    float alpha = 0.0f;
    const bool raw_max = !FAST && p.ed.is_int && p.asym;
#pragma unroll
    for (int j = 0; j < 8; ++j) alpha = fmaxf(alpha, raw_max ? xq[j] : fabsf(xq[j]));
    alpha = grp_max(alpha, G);
    const BlockScale bs = block_scale(p.ed, p.sd, alpha, bad, sT);

    float q[8];
    if constexpr (FAST) {
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = __fmul_rn(xq[j], bs.inv);
        const uint32_t pk = bs.zero ? 0u : cvt_e2m1x8(v);
        if (ok) reinterpret_cast<uint32_t *>(p.codes)[c] = pk;
        if (stats) e2m1x8_values(pk, q);
    } else {
        uint4 w0 = make_uint4(0, 0, 0, 0), w1 = w0;
        if (p.round_mode == RD_SR) {
            w0 = element_words(p.seed, (uint64_t)c * 2);
            w1 = element_words(p.seed, (uint64_t)c * 2 + 1);
        }
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t u = word_of(j < 4 ? w0 : w1, j & 3);
            uint32_t code = 0;
            q[j] = 0.0f;
            if (!bs.zero) code = encode_elem(p.ed, p.round_mode, __fmul_rn(xq[j], bs.inv), u, q[j]);
            if (p.ed.code_bits == 4) lo |= code << (4 * j);
            else if (j < 4) lo |= code << (8 * j);
            else hi |= code << (8 * (j - 4));
        }
        if (ok) {
            if (p.ed.code_bits == 4) reinterpret_cast<uint32_t *>(p.codes)[c] = lo;
            else reinterpret_cast<uint2 *>(p.codes)[c] = make_uint2(lo, hi);
        }
    }
    if (ok && (lane & (G - 1)) == 0) {
        const int64_t b = c / G;
        if (p.sf_gemm) {
            const int64_t S = p.cols / p.block;
            p.scales[sf_chunk_index(b / S, b - (b / S) * S, S)] = (uint8_t)bs.code;
        } else {
            p.scales[b] = (uint8_t)bs.code;
        }
        if (!FAST && p.asym) p.offsets[b] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
    }
    if (stats && ok) {
        float xh[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) xh[j] = deq_value(p, q[j], bs, sm, o, sT);
        acc_add<8>(acc, y, xh);
    }
}

template <typename InT, bool FAST>
__global__ void __launch_bounds__(kThreads) k_quant_row(const QParams p)
{
    constexpr int U = 2;
    const InT *x = static_cast<const InT *>(p.x);
    const int lane = threadIdx.x & 31;
    const int64_t nchunks = p.rows * p.cols / 8;
    const int64_t per_tile = 32 * U;
    const int64_t ntiles = (nchunks + per_tile - 1) / per_tile;
    const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const bool stats = p.partials != nullptr;
    const float sT = (p.ts_mode != TS_NONE) ? *p.tensor_scale : 1.0f;
    Acc acc = {0, 0, 0, 0, 0};
    for (int64_t t = gw; t < ntiles; t += nw) {
        float v[U][8];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t c = t * per_tile + u * 32 + lane;
            if (c < nchunks) load8(x, c * 8, v[u]);
            else
#pragma unroll
                for (int j = 0; j < 8; ++j) v[u][j] = 0.0f;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t c = t * per_tile + u * 32 + lane;
            row_chunk<FAST>(p, c, c < nchunks, v[u], sT, acc, lane, stats);
        }
    }
    if (stats) write_partials(p.partials, acc);
}

// Tensor absmax of y (NaN skipped) for the per-tensor scale, row chunks
// (rotation along rows: row and 2D layouts).
template <typename InT>
__global__ void __launch_bounds__(kThreads) k_amax_row(const QParams p)
{
    const InT *x = static_cast<const InT *>(p.x);
    const int lane = threadIdx.x & 31;
    const int64_t nchunks = p.rows * p.cols / 8;
    const int64_t ntiles = (nchunks + 31) / 32;
    const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    float m = 0.0f;
    for (int64_t t = gw; t < ntiles; t += nw) {
        const int64_t c = t * 32 + lane;
        float v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        if (c < nchunks) load8(x, c * 8, v);
        if (p.had) hadamard_chunk8(v, p.had, lane);
#pragma unroll
        for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(v[j]));
    }
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
    if (lane == 0 && m > 0.0f) atomicMax(p.amax_word, __float_as_uint(m));
}

// s_T = amax_T / (max_elem * max_scale); amax_T = 0 gives 1
__global__ void k_finalize_tensor_scale(const unsigned int *amax_word, float maxv, float smax,
                                        float *ts)
{
    const float amax = __uint_as_float(*amax_word);
    *ts = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, __fmul_rn(maxv, smax));
}

// Sum the per-CTA records in a fixed order and derive MSE, R-MSE, QSNR (Eq. (1)),
// bias and the flush-to-zero share.
__global__ void k_finalize_stats(const double *partials, int nparts, double count, double *stats)
{
    __shared__ double sh[256][5];
    double s[5] = {0, 0, 0, 0, 0};
    for (int i = threadIdx.x; i < nparts; i += blockDim.x)
        for (int k = 0; k < 5; ++k) s[k] += partials[(int64_t)i * kPartialDoubles + k];
    for (int k = 0; k < 5; ++k) sh[threadIdx.x][k] = s[k];
    __syncthreads();
    for (int w = blockDim.x / 2; w > 0; w >>= 1) {
        if ((int)threadIdx.x < w)
            for (int k = 0; k < 5; ++k) sh[threadIdx.x][k] += sh[threadIdx.x + w][k];
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        double x2 = sh[0][0], e2 = sh[0][1], e = sh[0][2], ftz = sh[0][3], nz = sh[0][4];
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
}

// ============================================================== launches ===
int cached_occupancy(const void *kernel, int threads, size_t smem)
{
    struct Entry { const void *k; int threads; size_t smem; int occ; };
    static Entry table[64];
    static int used = 0;
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i)
        if (table[i].k == kernel && table[i].threads == threads && table[i].smem == smem) return table[i].occ;
    if (smem > 48 * 1024) cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    int occ = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, threads, smem) != cudaSuccess || occ < 1) occ = 1;
    if (used < 64) table[used++] = Entry{kernel, threads, smem, occ};
    return occ;
}

static int g_sms = 0;
int device_sm_count()
{
    if (g_sms == 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess) return 148;
        if (cudaDeviceGetAttribute(&g_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) g_sms = 148;
    }
    return g_sms;
}

template <typename InT>
static int launch_row(const QParams &p, int fast, cudaStream_t st, int *grid_out)
{
    const int64_t tiles = (p.rows * p.cols / 8 + 63) / 64;
    if (fast) {
        const int g = grid_for(k_quant_row<InT, true>, tiles);
        k_quant_row<InT, true><<<g, kThreads, 0, st>>>(p);
        *grid_out = g;
    } else {
        const int g = grid_for(k_quant_row<InT, false>, tiles);
        k_quant_row<InT, false><<<g, kThreads, 0, st>>>(p);
        *grid_out = g;
    }
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

int launch_quantize(const QParams &p, int axis, int in_fp32, int fast, cudaStream_t st, int *grid_out)
{
    if (axis == AX_ROW)
        return in_fp32 ? launch_row<float>(p, fast, st, grid_out)
                       : launch_row<__nv_bfloat16>(p, fast, st, grid_out);
    return launch_quantize_col(p, axis, in_fp32, fast, st, grid_out);
}

int launch_tensor_amax(const QParams &p, int axis, int in_fp32, cudaStream_t st)
{
    if (cudaMemsetAsync(p.amax_word, 0, sizeof(unsigned int), st) != cudaSuccess) return -1;
    if (axis == AX_COL && p.had) {
        if (launch_amax_col(p, in_fp32, st)) return -1;
    } else {
        const int64_t tiles = (p.rows * p.cols / 8 + 31) / 32;
        if (in_fp32) {
            const int g = grid_for(k_amax_row<float>, tiles);
            k_amax_row<float><<<g, kThreads, 0, st>>>(p);
        } else {
            const int g = grid_for(k_amax_row<__nv_bfloat16>, tiles);
            k_amax_row<__nv_bfloat16><<<g, kThreads, 0, st>>>(p);
        }
    }
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

int launch_finalize_tensor_scale(const QParams &p, cudaStream_t st)
{
    k_finalize_tensor_scale<<<1, 1, 0, st>>>(p.amax_word, p.ed.maxv, p.sd.ue_maxv, p.tensor_scale);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

int launch_finalize_stats(const double *partials, int nparts, double count, double *stats,
                          cudaStream_t st)
{
    k_finalize_stats<<<1, 256, 0, st>>>(partials, nparts, count, stats);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace mxk
