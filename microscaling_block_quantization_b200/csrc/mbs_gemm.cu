// Macro Block Scaling operands for the block-scaled FP4 GEMM ("Unveiling the
// Potential of Quantization with MXFP4", Sec.4 MBS and its GEMM, Fig. 5).
//
// An MBS tensor carries, per 1 x 32 block, an E8M0 scale X = 2^k and, per
// 1 x 128 macro block, an E4M3 scale S_M; an element dequantizes to q X S_M.
// The product S_M X is an E4M3 significand times a power of two, so with a
// per-tensor power of two s_T it is exactly a UE4M3 value whenever it lands in
// UE4M3's normal range: the GEMM's nearest-scale (NVFP4) kind then consumes
// the MBS operand unchanged, with one 16-element scale (S_M X / s_T, written
// twice per 32-block) and s_T as the tensor scale.  Two launches: the largest
// folded exponent (atomic max), then the folded scales in the tcgen05 chunk
// layout.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "mx.h"
#include "mx_internal.h"

namespace mxk {
namespace {

constexpr int kFoldThreads = 256;
constexpr int kExpBias = 1024;      // folded exponents are stored biased (atomicMax on int)

// folded value S_M X of a block as significand m in [1, 2) and exponent;
// false for a NaN scale or macro scale, or a zero block (E8M0 code 0)
__device__ __forceinline__ bool fold_parts(uint32_t code, uint32_t mcode, float &m, int &e)
{
    if (code == 0xffu || (mcode & 0x7fu) == 0x7fu || code == 0u) return false;
    const float sm = e4m3_value(mcode);          // E4M3, positive
    if (!(sm > 0.0f)) return false;
    const uint32_t b = __float_as_uint(sm);
    m = __uint_as_float((b & 0x7fffffu) | 0x3f800000u);
    e = (int)(b >> 23) - 127 + (int)code - 127;  // normal E4M3 values only (S_M in [2/3, 4/3))
    return true;
}

__global__ void __launch_bounds__(kFoldThreads) k_mbs_fold_max(const uint8_t *scales, const uint8_t *macro,
                                                             int64_t nblk, int *emax_word)
{
    int best = -(1 << 30);
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblk; b += (int64_t)gridDim.x * blockDim.x) {
        float m;
        int e;
        if (fold_parts(scales[b], macro[b >> 2], m, e)) best = max(best, e);
    }
    for (int o = 16; o > 0; o >>= 1) best = max(best, __shfl_xor_sync(0xffffffffu, best, o));
    if ((threadIdx.x & 31) == 0 && best > -(1 << 30)) atomicMax(emax_word, best + kExpBias);
}

// one thread per 32-block: two UE4M3 codes (the two 16-element halves)
__global__ void __launch_bounds__(kFoldThreads) k_mbs_fold(const uint8_t *scales, const uint8_t *macro,
                                                         int64_t rows, int64_t cols, uint8_t *sf16,
                                                         const int *emax_word, float *ts)
{
    const int stored = *emax_word;
    // s_T = 2^t with the largest folded value m 2^emax below 2^8 after division
    const int t = stored == 0 ? 0 : stored - kExpBias - 7;
    if (blockIdx.x == 0 && threadIdx.x == 0) *ts = __uint_as_float((uint32_t)(127 + t) << 23);
    const int64_t s32 = cols / 32, s16 = cols / 16;
    const int64_t nblk = rows * s32;
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblk; b += (int64_t)gridDim.x * blockDim.x) {
        const uint32_t code = scales[b];
        const uint32_t mcode = macro[b >> 2];
        uint32_t u;
        float m;
        int e;
        if (code == 0xffu || (mcode & 0x7fu) == 0x7fu) u = 0x7fu;
        else if (!fold_parts(code, mcode, m, e)) u = 0u;
        else {
            const int ee = e - t;            // <= 7
            float v;
            if (ee >= -126) v = __uint_as_float(((uint32_t)(ee + 127) << 23) | (__float_as_uint(m) & 0x7fffffu));
            else v = 0.0f;                   // far below UE4M3's range
            uint16_t r;
            asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
            u = r & 0xffu;
        }
        const int64_t row = b / s32, j = (b - row * s32) * 2;
        sf16[sf_chunk_index((uint32_t)row, (uint32_t)j, (uint32_t)s16)] = (uint8_t)u;
        sf16[sf_chunk_index((uint32_t)row, (uint32_t)j + 1, (uint32_t)s16)] = (uint8_t)u;
    }
}

int grid_blocks(int64_t n)
{
    int64_t g = (n + kFoldThreads - 1) / kFoldThreads;
    const int64_t cap = (int64_t)device_sm_count() * 8;
    if (g > cap) g = cap;
    return (int)(g < 1 ? 1 : g);
}

}  // namespace
}  // namespace mxk

using namespace mxk;

extern "C" int mx_mbs_gemm_scales(const mx_config *cfg, const uint8_t *scales, const uint8_t *macro_scales,
                                  int64_t rows, int64_t cols, uint8_t *sf16, float *tensor_scale,
                                  void *workspace, int64_t workspace_bytes, void *stream)
{
    if (!cfg || !scales || !macro_scales || !sf16 || !tensor_scale || !workspace) return MX_ERR_INVALID;
    if (cfg->elem != MX_E2M1 || cfg->scale_fmt != MX_SCALE_E8M0 || cfg->block != 32 || cfg->macro_block != 128 ||
        cfg->axis != MX_AXIS_ROW || cfg->asymmetric || cfg->sf_layout != 0 || cfg->hadamard)
        return MX_ERR_UNSUPPORTED;
    if (rows <= 0 || cols <= 0 || rows % 128 || cols % 128) return MX_ERR_INVALID;
    if (rows > (kMaxElements - 1) / cols) return MX_ERR_INVALID;
    if (workspace_bytes < kWsHeader) return MX_ERR_WORKSPACE;
    if (((uintptr_t)workspace & 15u) || ((uintptr_t)sf16 & 15u) || ((uintptr_t)tensor_scale & 3u))
        return MX_ERR_ALIGN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int *emax_word = reinterpret_cast<int *>(static_cast<uint8_t *>(workspace) + 128);
    if (cudaMemsetAsync(emax_word, 0, sizeof(int), st) != cudaSuccess) return MX_ERR_CUDA;
    const int64_t nblk = rows * (cols / 32);
    const int g = grid_blocks(nblk);
    k_mbs_fold_max<<<g, kFoldThreads, 0, st>>>(scales, macro_scales, nblk, emax_word);
    k_mbs_fold<<<g, kFoldThreads, 0, st>>>(scales, macro_scales, rows, cols, sf16, emax_word, tensor_scale);
    if (cudaGetLastError() != cudaSuccess) return MX_ERR_CUDA;
    // leave the control word zero for the next user of the workspace
    if (cudaMemsetAsync(emax_word, 0, sizeof(int), st) != cudaSuccess) return MX_ERR_CUDA;
    return MX_OK;
}
