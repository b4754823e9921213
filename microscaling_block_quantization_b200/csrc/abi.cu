// C ABI entry points (include/mx.h): argument validation on the host, format
// descriptors, and the launch sequence of each call.  Nothing here computes
// on the CPU: every step of the method runs in the sm_100a kernels.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <new>

#include "mx.h"
#include "mx_internal.h"

using namespace mxk;

namespace {

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

bool make_elem(int elem, int asym, ElemDesc &d)
{
    memset(&d, 0, sizeof(d));
    d.elem = elem;
    d.asym = asym;
    switch (elem) {
    case MX_E2M1: d.mbits = 1; d.bias = 1; d.code_bits = 4; d.max_code = 7;  d.emax = 2; d.maxv = 6.0f;  break;
    case MX_E3M0: d.mbits = 0; d.bias = 3; d.code_bits = 4; d.max_code = 7;  d.emax = 4; d.maxv = 16.0f; break;
    case MX_E2M3: d.mbits = 3; d.bias = 1; d.code_bits = 6; d.max_code = 31; d.emax = 2; d.maxv = 7.5f;  break;
    case MX_E3M2: d.mbits = 2; d.bias = 3; d.code_bits = 6; d.max_code = 31; d.emax = 4; d.maxv = 28.0f; break;
    case MX_INT4:
        d.is_int = 1; d.code_bits = 4;
        if (asym) { d.max_code = 15; d.emax = 3; d.maxv = 15.0f; }
        else      { d.max_code = 7;  d.emax = 2; d.maxv = 7.0f; }
        break;
    default: return false;
    }
    if (!d.is_int) {
        d.sub_lim = ldexpf(1.0f, 1 - d.bias);
        d.sub_inv_q = ldexpf(1.0f, d.bias + d.mbits - 1);
    }
    return true;
}

bool make_scale(const mx_config *c, ScaleDesc &s)
{
    memset(&s, 0, sizeof(s));
    s.fmt = c->scale_fmt;
    s.rule = c->rule;
    s.tau = c->oas_tau;
    switch (c->scale_fmt) {
    case MX_SCALE_E8M0: s.kmin = -127; s.kmax = 127; break;
    case MX_SCALE_UE4M3:
        s.ue_bias = 7; s.ue_max_code = 0x7e; s.ue_nan_code = 0x7f; s.ue_maxv = 448.0f;
        s.kmin = -9; s.kmax = 8;
        break;
    case MX_SCALE_UE5M3:
        s.ue_bias = 15; s.ue_max_code = 0xfe; s.ue_nan_code = 0xff; s.ue_maxv = 114688.0f;
        s.kmin = -17; s.kmax = 16;
        break;
    default: return false;
    }
    return true;
}

bool is_pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

// Shape / combination checks shared by quantize and dequantize.
int check_config(const mx_config *c, int64_t rows, int64_t cols, bool want_had)
{
    if (!c) return MX_ERR_INVALID;
    if (rows < 0 || cols < 0) return MX_ERR_INVALID;
    if (c->sf_layout != 0 && c->sf_layout != 1) return MX_ERR_INVALID;
    if (c->sf_layout == 1 && c->axis != MX_AXIS_ROW) return MX_ERR_UNSUPPORTED;
    if (c->elem < MX_E2M1 || c->elem > MX_INT4) return MX_ERR_INVALID;
    if (c->scale_fmt < MX_SCALE_E8M0 || c->scale_fmt > MX_SCALE_UE5M3) return MX_ERR_INVALID;
    if (c->rule < MX_RULE_FLOOR || c->rule > MX_RULE_MSE) return MX_ERR_INVALID;
    // MSE rule: E8M0 blocks of 32 (any element type), or E2M1 with a nearest
    // scale format and blocks of 8 / 16 / 32 (the alternating optimisation
    // with a computed tensor scale); row axis, nearest-even elements
    if (c->rule == MX_RULE_MSE) {
        if (c->round != MX_ROUND_RTNE || c->axis != MX_AXIS_ROW || c->asymmetric || c->macro_block ||
            c->hadamard)
            return MX_ERR_UNSUPPORTED;
        if (c->scale_fmt == MX_SCALE_E8M0 && (c->block != 32 || c->tensor_scale != MX_TS_NONE))
            return MX_ERR_UNSUPPORTED;
        if (c->scale_fmt != MX_SCALE_E8M0 &&
            (c->elem != MX_E2M1 || !(c->block == 8 || c->block == 16 || c->block == 32) ||
             c->tensor_scale == MX_TS_AMAX))
            return MX_ERR_UNSUPPORTED;
    }
    if (c->round < MX_ROUND_RTNE || c->round > MX_ROUND_STOCHASTIC) return MX_ERR_INVALID;
    if (c->axis < MX_AXIS_ROW || c->axis > MX_AXIS_2D) return MX_ERR_INVALID;
    if (c->asymmetric != 0 && c->asymmetric != 1) return MX_ERR_INVALID;
    if (c->tensor_scale < MX_TS_NONE || c->tensor_scale > MX_TS_AMAX) return MX_ERR_INVALID;
    if (c->macro_block != 0 && c->macro_block != 128) return MX_ERR_INVALID;
    if (c->hadamard != 0 && c->hadamard != 16 && c->hadamard != 32) return MX_ERR_INVALID;
    if (want_had != (c->hadamard != 0)) return MX_ERR_INVALID;
    if (c->rule == MX_RULE_OAS && !(c->oas_tau > 0.0f && c->oas_tau < INFINITY)) return MX_ERR_INVALID;

    // block sizes per axis
    const int B = c->block;
    if (c->axis == MX_AXIS_ROW) {
        if (!(is_pow2(B) && B >= 8 && B <= 256)) return MX_ERR_UNSUPPORTED;
    } else if (c->axis == MX_AXIS_COL) {
        if (!(B == 8 || B == 16 || B == 32)) return MX_ERR_UNSUPPORTED;
    } else {
        if (B != 32) return MX_ERR_UNSUPPORTED;
    }

    // scale formats and rules
    if (c->scale_fmt == MX_SCALE_E8M0) {
        if (c->rule == MX_RULE_NEAREST) return MX_ERR_INVALID;
        if (c->tensor_scale != MX_TS_NONE) return MX_ERR_INVALID;
    } else {
        if (c->rule != MX_RULE_NEAREST && c->rule != MX_RULE_MSE && c->tensor_scale != MX_TS_NONE)
            return MX_ERR_UNSUPPORTED;
        if (c->asymmetric) return MX_ERR_UNSUPPORTED;
    }
    if (c->macro_block) {
        if (c->scale_fmt != MX_SCALE_E8M0 || c->asymmetric) return MX_ERR_UNSUPPORTED;
        if (c->axis != MX_AXIS_2D && B > 128) return MX_ERR_UNSUPPORTED;
    }

    // shapes
    if (rows == 0 || cols == 0) return MX_OK;
    // kernels walk rows in 32-element chunks (one per lane)
    if (cols % 32) return MX_ERR_INVALID;
    // fewer than 2^32 elements: 32-bit element, code-word and block indices
    if (rows > (kMaxElements - 1) / cols) return MX_ERR_INVALID;
    if (c->axis == MX_AXIS_ROW && cols % B) return MX_ERR_INVALID;
    if (c->sf_layout == 1 && (rows % 128 || (cols / B) % 4)) return MX_ERR_INVALID;
    if (c->axis == MX_AXIS_COL && rows % B) return MX_ERR_INVALID;
    if (c->axis == MX_AXIS_2D && (rows % 32 || cols % 32)) return MX_ERR_INVALID;
    if (c->macro_block) {
        if (c->axis == MX_AXIS_COL ? rows % 128 : cols % 128) return MX_ERR_INVALID;
    }
    if (c->hadamard) {
        const int n = c->hadamard;
        if (c->axis == MX_AXIS_COL) {
            if (B < n || rows % n) return MX_ERR_UNSUPPORTED;
        } else if (cols % n) {
            return MX_ERR_INVALID;
        }
    }
    return MX_OK;
}

int64_t nblocks_of(const mx_config *c, int64_t rows, int64_t cols)
{
    if (c->axis == MX_AXIS_ROW) return rows * (cols / c->block);
    if (c->axis == MX_AXIS_COL) return (rows / c->block) * cols;
    return (rows / 32) * (cols / 32);
}

int64_t nmacro_of(const mx_config *c, int64_t rows, int64_t cols)
{
    if (!c->macro_block) return 0;
    return c->axis == MX_AXIS_COL ? (rows / 128) * cols : rows * (cols / 128);
}

int64_t codes_bytes_of(const mx_config *c, int64_t rows, int64_t cols)
{
    // FP6: one byte per code, or 6 bits per code in the dense tensor-core form
    if (c->elem == MX_E2M3 || c->elem == MX_E3M2) return c->sf_layout == 1 ? rows * cols / 4 * 3 : rows * cols;
    return rows * cols / 2;
}

int cuda_ok(cudaError_t e) { return e == cudaSuccess ? MX_OK : MX_ERR_CUDA; }

// Validation and launch parameters of one tensor of a quantize call.  *empty:
// nothing to launch (the caller still writes the statistics of an empty
// tensor).
int prepare_quantize(const mx_config *cfg, const void *x, int32_t x_dtype, int64_t rows, int64_t cols,
                     void *codes, uint8_t *scales, float *tensor_scale, uint8_t *macro_scales,
                     uint16_t *offsets, double *stats, float *rotated, void *workspace,
                     int64_t workspace_bytes, bool want_had, bool amax_only, QParams &p, bool &empty)
{
    empty = false;
    int rc = check_config(cfg, rows, cols, want_had);
    if (rc != MX_OK) return rc;
    if (x_dtype != MX_DT_BF16 && x_dtype != MX_DT_FP32) return MX_ERR_INVALID;
    if (!amax_only) {
        if (cfg->tensor_scale != MX_TS_NONE && !tensor_scale) return MX_ERR_INVALID;
        if (cfg->macro_block && !macro_scales) return MX_ERR_INVALID;
        if (cfg->asymmetric && !offsets) return MX_ERR_INVALID;
    }
    const bool need_ws = stats != nullptr || cfg->tensor_scale == MX_TS_COMPUTE ||
                         cfg->tensor_scale == MX_TS_AMAX || amax_only;
    if (need_ws && (!workspace || workspace_bytes < kWorkspaceBytes)) return MX_ERR_WORKSPACE;
    const int64_t n = rows * cols;
    if (n == 0) {
        empty = true;
        return MX_OK;
    }
    if (!x || (!amax_only && (!codes || !scales))) return MX_ERR_INVALID;
    if (!aligned16(x) || (!amax_only && (!aligned16(codes) || !aligned16(scales)))) return MX_ERR_ALIGN;
    if ((macro_scales && !aligned16(macro_scales)) || (offsets && !aligned16(offsets)) ||
        (rotated && !aligned16(rotated)) || (workspace && !aligned16(workspace)) ||
        (stats && ((uintptr_t)stats & 7u)) || (tensor_scale && ((uintptr_t)tensor_scale & 3u)))
        return MX_ERR_ALIGN;

    memset(&p, 0, sizeof(p));
    p.x = x;
    p.rows = rows;
    p.cols = cols;
    p.codes = codes;
    p.scales = scales;
    p.tensor_scale = tensor_scale;
    p.macro = macro_scales;
    p.offsets = offsets;
    p.rotated = rotated;
    if (!make_elem(cfg->elem, cfg->asymmetric, p.ed)) return MX_ERR_INVALID;
    if (!make_scale(cfg, p.sd)) return MX_ERR_INVALID;
    p.block = cfg->block;
    p.lanes_per_block = cfg->block / 8;
    p.round_mode = cfg->round;
    p.asym = cfg->asymmetric;
    p.mbs = cfg->macro_block;
    p.had = cfg->hadamard;
    // a given amax (already in the workspace's amax word) is a computed
    // tensor scale without the pre-pass
    p.ts_mode = cfg->tensor_scale == MX_TS_AMAX ? (int)MX_TS_COMPUTE : cfg->tensor_scale;
    p.seed = cfg->seed;
    p.sf_gemm = cfg->sf_layout;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    p.amax_word = ws ? reinterpret_cast<unsigned int *>(ws) : nullptr;
    p.partials = (stats && ws) ? reinterpret_cast<double *>(ws + kWsHeader) : nullptr;
    p.stats = stats;
    p.count = (double)n;
    p.ticket = need_ws ? reinterpret_cast<unsigned int *>(ws + kWsTicket) : nullptr;
    return MX_OK;
}

// the element path of the fast (TMA ring) quantizer: E2M1, RTNE, symmetric,
// not the MSE rule
bool fast_elements(const mx_config *cfg)
{
    return cfg->elem == MX_E2M1 && cfg->round == MX_ROUND_RTNE && !cfg->asymmetric && cfg->rule != MX_RULE_MSE;
}

int quantize_impl(const mx_config *cfg, const void *x, int32_t x_dtype, int64_t rows, int64_t cols,
                  void *codes, uint8_t *scales, float *tensor_scale, uint8_t *macro_scales,
                  uint16_t *offsets, double *stats, float *rotated, void *workspace,
                  int64_t workspace_bytes, void *stream, bool want_had, bool amax_only = false)
{
    QParams p;
    bool empty;
    const int rc = prepare_quantize(cfg, x, x_dtype, rows, cols, codes, scales, tensor_scale, macro_scales,
                                    offsets, stats, rotated, workspace, workspace_bytes, want_had, amax_only,
                                    p, empty);
    if (rc != MX_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (empty) {
        if (amax_only) return MX_OK;
        if (stats) return launch_finalize_stats(nullptr, 0, 0.0, stats, st) ? MX_ERR_CUDA : MX_OK;
        return MX_OK;
    }
    const int in_fp32 = x_dtype == MX_DT_FP32;

    // the tensor-amax pre-pass; the quantizer derives s_T from its word
    if ((cfg->tensor_scale == MX_TS_COMPUTE || amax_only) && launch_tensor_amax(p, cfg->axis, in_fp32, st))
        return MX_ERR_CUDA;
    if (amax_only) return MX_OK;
    if (cfg->rule == MX_RULE_MSE && cfg->scale_fmt != MX_SCALE_E8M0) {
        // (a computed tensor scale: the global-step passes reduce through the
        // workspace records and ticket, which need_ws has required)
        uint8_t *ws = static_cast<uint8_t *>(workspace);
        float *chain = ws ? reinterpret_cast<float *>(ws + kWsMseChain) : nullptr;
        double *partials = ws ? reinterpret_cast<double *>(ws + kWsHeader) : nullptr;
        return launch_quantize_mse(p, partials, chain, in_fp32, st) ? MX_ERR_CUDA : MX_OK;
    }
    int grid = 0;
    if (launch_quantize(p, cfg->axis, in_fp32, fast_elements(cfg), st, &grid)) return MX_ERR_CUDA;
    return MX_OK;
}

// the configurations launch_quantize sends to the fast quantizer (without a
// rotated output)
bool groupable(const mx_config *cfg)
{
    return cfg->axis == MX_AXIS_ROW && fast_elements(cfg) &&
           ((!cfg->macro_block && !cfg->hadamard) || cfg->block == 16 || cfg->block == 32);
}

// the configurations launch_quantize_col sends to the double-buffered column /
// 2D quantizer
bool col_groupable(const mx_config *cfg, int32_t x_dtype)
{
    return cfg->axis != MX_AXIS_ROW && x_dtype == MX_DT_BF16 && fast_elements(cfg) && !cfg->macro_block &&
           !cfg->hadamard;
}

}  // namespace

extern "C" {

const char *mx_version(void) { return "mx-b200 0.1 (sm_100a)"; }

const char *mx_strerror(int code)
{
    switch (code) {
    case MX_OK: return "ok";
    case MX_ERR_INVALID: return "invalid argument, shape or combination";
    case MX_ERR_UNSUPPORTED: return "combination not supported by this library";
    case MX_ERR_ALIGN: return "pointer not 16-byte aligned";
    case MX_ERR_CUDA: return "CUDA launch or runtime error";
    case MX_ERR_WORKSPACE: return "workspace missing or too small";
    case MX_ERR_NO_DEVICE: return "no sm_100 device";
    case MX_ERR_TIMEOUT: return "a bounded in-kernel wait gave up";
    default: return "unknown status";
    }
}

int mx_query_sizes(const mx_config *cfg, int64_t rows, int64_t cols, mx_sizes *out)
{
    if (!cfg || !out) return MX_ERR_INVALID;
    int rc = check_config(cfg, rows, cols, cfg->hadamard != 0);
    if (rc != MX_OK) return rc;
    out->codes_bytes = codes_bytes_of(cfg, rows, cols);
    out->n_blocks = (rows && cols) ? nblocks_of(cfg, rows, cols) : 0;
    out->n_scales = out->n_blocks;
    out->n_macro = (rows && cols) ? nmacro_of(cfg, rows, cols) : 0;
    out->n_offsets = cfg->asymmetric ? out->n_blocks : 0;
    out->workspace_bytes = kWorkspaceBytes;
    return MX_OK;
}

int mx_quantize(const mx_config *cfg, const void *x, int32_t x_dtype, int64_t rows, int64_t cols,
                void *codes, uint8_t *scales, float *tensor_scale, uint8_t *macro_scales,
                uint16_t *offsets, double *stats, void *workspace, int64_t workspace_bytes,
                void *stream)
{
    return quantize_impl(cfg, x, x_dtype, rows, cols, codes, scales, tensor_scale, macro_scales,
                         offsets, stats, nullptr, workspace, workspace_bytes, stream, false);
}

int mx_hadamard_quantize(const mx_config *cfg, const void *x, int32_t x_dtype, int64_t rows,
                         int64_t cols, void *codes, uint8_t *scales, float *tensor_scale,
                         uint8_t *macro_scales, uint16_t *offsets, double *stats,
                         float *rotated, void *workspace, int64_t workspace_bytes, void *stream)
{
    return quantize_impl(cfg, x, x_dtype, rows, cols, codes, scales, tensor_scale, macro_scales,
                         offsets, stats, rotated, workspace, workspace_bytes, stream, true);
}

int mx_quantize_group(const mx_config *cfg, int32_t x_dtype, const mx_quantize_item *items, int32_t n,
                      void *stream)
{
    if (!cfg || !items || n < 1) return MX_ERR_INVALID;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    QParams *ps = new (std::nothrow) QParams[n];
    bool *empty = new (std::nothrow) bool[n];
    int rc = (ps && empty) ? MX_OK : MX_ERR_INVALID;
    // every item is checked before anything is queued
    for (int i = 0; i < n && rc == MX_OK; ++i) {
        const mx_quantize_item &it = items[i];
        rc = prepare_quantize(cfg, it.x, x_dtype, it.rows, it.cols, it.codes, it.scales, it.tensor_scale,
                              it.macro_scales, it.offsets, it.stats, nullptr, it.workspace, it.workspace_bytes,
                              cfg->hadamard != 0, false, ps[i], empty[i]);
    }
    // items that use their workspace must not share one
    const bool uses_ws = cfg->tensor_scale == MX_TS_COMPUTE || cfg->tensor_scale == MX_TS_AMAX;
    for (int i = 0; i < n && rc == MX_OK; ++i)
        for (int j = i + 1; j < n && rc == MX_OK; ++j) {
            const bool wi = items[i].stats || uses_ws, wj = items[j].stats || uses_ws;
            if (!wi || !wj || !items[i].workspace || !items[j].workspace) continue;
            const uintptr_t a0 = (uintptr_t)items[i].workspace, b0 = (uintptr_t)items[j].workspace;
            if (a0 < b0 + (uintptr_t)kWorkspaceBytes && b0 < a0 + (uintptr_t)kWorkspaceBytes) rc = MX_ERR_INVALID;
        }
    const int in_fp32 = x_dtype == MX_DT_FP32;
    const bool col = col_groupable(cfg, x_dtype);
    if (rc == MX_OK && !groupable(cfg) && !col) {
        // other configurations: one call per tensor, in order
        for (int i = 0; i < n && rc == MX_OK; ++i) {
            const mx_quantize_item &it = items[i];
            rc = quantize_impl(cfg, it.x, x_dtype, it.rows, it.cols, it.codes, it.scales, it.tensor_scale,
                               it.macro_scales, it.offsets, it.stats, nullptr, it.workspace, it.workspace_bytes,
                               stream, cfg->hadamard != 0);
        }
    } else if (rc == MX_OK) {
        // empty tensors: their statistics; the others in launches of up to
        // kFastGroupMax tensors (with the tensor-amax pre-pass of each launch's
        // tensors before it)
        QParams chunk[kFastGroupMax];
        int m = 0;
        for (int i = 0; i <= n && rc == MX_OK; ++i) {
            if (i < n && empty[i]) {
                if (items[i].stats && launch_finalize_stats(nullptr, 0, 0.0, items[i].stats, st)) rc = MX_ERR_CUDA;
                continue;
            }
            if (i < n) chunk[m++] = ps[i];
            if (m == kFastGroupMax || (i == n && m > 0)) {
                if (cfg->tensor_scale == MX_TS_COMPUTE) {
                    if (cfg->hadamard) {
                        for (int k = 0; k < m && rc == MX_OK; ++k)
                            if (launch_tensor_amax(chunk[k], cfg->axis, in_fp32, st)) rc = MX_ERR_CUDA;
                    } else if (launch_tensor_amax_group(chunk, m, in_fp32, st)) {
                        rc = MX_ERR_CUDA;
                    }
                }
                if (rc == MX_OK) {
                    const int e = col ? launch_quantize_colx_group(chunk, m, cfg->axis, st)
                                      : launch_quantize_fast_group(chunk, m, in_fp32, st);
                    if (e) rc = MX_ERR_CUDA;
                }
                m = 0;
            }
        }
    }
    delete[] ps;
    delete[] empty;
    return rc;
}

int mx_tensor_amax(const mx_config *cfg, const void *x, int32_t x_dtype, int64_t rows, int64_t cols,
                   void *workspace, int64_t workspace_bytes, void *stream)
{
    if (!cfg) return MX_ERR_INVALID;
    if (cfg->tensor_scale != MX_TS_AMAX) return MX_ERR_INVALID;
    return quantize_impl(cfg, x, x_dtype, rows, cols, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                         nullptr, workspace, workspace_bytes, stream, cfg->hadamard != 0, true);
}

int mx_stats_finalize(double *stats, void *stream)
{
    if (!stats) return MX_ERR_INVALID;
    if ((uintptr_t)stats & 7u) return MX_ERR_ALIGN;
    return launch_stats_refinalize(stats, static_cast<cudaStream_t>(stream)) ? MX_ERR_CUDA : MX_OK;
}

int mx_dequantize(const mx_config *cfg, const void *codes, const uint8_t *scales,
                  const float *tensor_scale, const uint8_t *macro_scales,
                  const uint16_t *offsets, int64_t rows, int64_t cols, void *out,
                  int32_t out_dtype, void *stream)
{
    int rc = check_config(cfg, rows, cols, cfg ? cfg->hadamard != 0 : false);
    if (rc != MX_OK) return rc;
    if (out_dtype != MX_DT_BF16 && out_dtype != MX_DT_FP32) return MX_ERR_INVALID;
    if (rows * cols == 0) return MX_OK;
    if (!codes || !scales || !out) return MX_ERR_INVALID;
    if (cfg->tensor_scale != MX_TS_NONE && !tensor_scale) return MX_ERR_INVALID;
    if (cfg->macro_block && !macro_scales) return MX_ERR_INVALID;
    if (cfg->asymmetric && !offsets) return MX_ERR_INVALID;
    if (!aligned16(codes) || !aligned16(scales) || !aligned16(out) ||
        (macro_scales && !aligned16(macro_scales)) || (offsets && !aligned16(offsets)))
        return MX_ERR_ALIGN;
    DParams p;
    memset(&p, 0, sizeof(p));
    p.codes = codes;
    p.scales = scales;
    p.tensor_scale = tensor_scale;
    p.macro = macro_scales;
    p.offsets = offsets;
    p.rows = rows;
    p.cols = cols;
    p.out = out;
    p.out_fp32 = out_dtype == MX_DT_FP32;
    if (!make_elem(cfg->elem, cfg->asymmetric, p.ed)) return MX_ERR_INVALID;
    if (!make_scale(cfg, p.sd)) return MX_ERR_INVALID;
    // an MSE-chosen nearest-format scale dequantizes like a nearest one
    if (p.sd.fmt != S_E8M0 && p.sd.rule == R_MSE) p.sd.rule = R_NEAREST;
    p.block = cfg->block;
    p.axis = cfg->axis;
    p.asym = cfg->asymmetric;
    p.mbs = cfg->macro_block;
    p.had = cfg->hadamard;
    p.ts_mode = cfg->tensor_scale;
    p.sf_gemm = cfg->sf_layout;
    return launch_dequantize(p, static_cast<cudaStream_t>(stream)) ? MX_ERR_CUDA : MX_OK;
}

int64_t mx_qsnr_workspace_bytes(int64_t rows, int64_t cols)
{
    (void)rows;
    (void)cols;
    return kWorkspaceBytes;
}

int mx_qsnr(const void *x, int32_t x_dtype, const void *x_hat, int32_t x_hat_dtype, int64_t rows,
            int64_t cols, int32_t block, int32_t axis, double *stats, float *per_block_mse,
            void *workspace, int64_t workspace_bytes, void *stream)
{
    if (rows < 0 || cols < 0 || !stats) return MX_ERR_INVALID;
    if (cols > 0 && rows > (kMaxElements - 1) / cols) return MX_ERR_INVALID;
    if ((x_dtype != MX_DT_BF16 && x_dtype != MX_DT_FP32) ||
        (x_hat_dtype != MX_DT_BF16 && x_hat_dtype != MX_DT_FP32))
        return MX_ERR_INVALID;
    if (axis < MX_AXIS_ROW || axis > MX_AXIS_2D) return MX_ERR_INVALID;
    if (!workspace || workspace_bytes < kWorkspaceBytes) return MX_ERR_WORKSPACE;
    if (((uintptr_t)stats & 7u) || !aligned16(workspace)) return MX_ERR_ALIGN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    double *partials = reinterpret_cast<double *>(static_cast<uint8_t *>(workspace) + kWsHeader);
    if (rows * cols == 0) return launch_finalize_stats(partials, 0, 0.0, stats, st) ? MX_ERR_CUDA : MX_OK;
    if (!x || !x_hat) return MX_ERR_INVALID;
    if (cols % 8) return MX_ERR_INVALID;
    if (per_block_mse) {
        if (axis == MX_AXIS_ROW && !(is_pow2(block) && block >= 8 && block <= 256 && cols % block == 0))
            return MX_ERR_INVALID;
        if (axis == MX_AXIS_COL && !((block == 8 || block == 16 || block == 32) && rows % block == 0))
            return MX_ERR_INVALID;
        if (axis == MX_AXIS_2D && (block != 32 || rows % 32 || cols % 32)) return MX_ERR_INVALID;
        if ((uintptr_t)per_block_mse & 3u) return MX_ERR_ALIGN;
    }
    if (!aligned16(x) || !aligned16(x_hat)) return MX_ERR_ALIGN;
    SParams p;
    memset(&p, 0, sizeof(p));
    p.x = x;
    p.xh = x_hat;
    p.x_fp32 = x_dtype == MX_DT_FP32;
    p.xh_fp32 = x_hat_dtype == MX_DT_FP32;
    p.rows = rows;
    p.cols = cols;
    p.block = per_block_mse ? block : 8;
    p.axis = axis;
    p.per_block_mse = per_block_mse;
    p.partials = partials;
    int grid = 0;
    if (launch_qsnr(p, st, &grid)) return MX_ERR_CUDA;
    return launch_finalize_stats(partials, grid, (double)(rows * cols), stats, st) ? MX_ERR_CUDA : MX_OK;
}

}  // extern "C"
