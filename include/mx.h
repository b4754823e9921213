/*
 * mx.h -- C ABI of the B200 (sm_100a) microscaling block-quantization library.
 *
 * Plain C: every argument is a pointer (host or device, as stated), an
 * integer or a float.  Every call is asynchronous on the CUDA stream passed
 * as `stream` (a cudaStream_t passed as void*, NULL = legacy default stream),
 * returns MX_OK (0) on success or a negative MX_ERR_* code, never prints and
 * never traps.  Arguments are validated on the host before any launch.
 *
 * Ownership: the caller owns every buffer.  The library allocates no device
 * memory; scratch space ("workspace") is passed in by the caller, sized by
 * mx_query_sizes() / mx_qsnr_workspace_bytes() / mx_gemm_workspace_bytes().
 * The first 256 bytes of a workspace are the library's control words (the
 * tensor-amax accumulator and a launch ticket): zero them once, before the
 * first call that uses the workspace (cudaMemset); every call leaves them
 * zero, so a workspace stays usable as long as calls sharing it are ordered
 * on one stream.
 * Buffers must stay alive until the stream reaches the end of the call.
 *
 * Sources (the pages this library follows):
 *   [MXFP4-OAS] "Unveiling the Potential of Quantization with MXFP4:
 *               Strategies for Quantization Error Reduction" (Qiita
 *               explainer / nubint review): Sec.2 MXFP4 and NVFP4 formats,
 *               Sec.3 QSNR Eq. (1) and Eq. (2), Sec.4 block granularity,
 *               Overflow-Aware Scaling (OAS), Macro Block Scaling (MBS),
 *               Fig. 5 (the AB^T product with macro scales).
 *   [FINER]     "Is Finer Better? The Limits of Microscaling Formats in
 *               Large Language Models": UE4M3 / UE5M3 block scales, FP32
 *               per-tensor scale, per-block and per-tensor MSE.
 *   [BRIDGING]  "Bridging the Gap Between Promise and Performance for
 *               Microscaling FP4 Quantization": block-wise Hadamard
 *               rotation fused with quantization (sec. 2.1-2.3), block-scaled
 *               FP4 GEMM on Blackwell (sec. 2.3).
 *   [MX-TRAIN]  fmread summary of Yang et al., MX quantization for LLM
 *               training (ARITH 2025): E2M1/E3M0/INT4 elements, RTNE / Ceil /
 *               stochastic rounding, asymmetric scaling, row-wise,
 *               column-wise and 2D blocks, R-MSE.
 */
#ifndef MX_H_
#define MX_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
#define MX_OK                0
#define MX_ERR_INVALID      -1   /* bad pointer, shape, enum value or combination */
#define MX_ERR_UNSUPPORTED  -2   /* valid per the pages but not implemented here */
#define MX_ERR_ALIGN        -3   /* a pointer is not 16-byte aligned */
#define MX_ERR_CUDA         -4   /* a CUDA launch or runtime call failed */
#define MX_ERR_WORKSPACE    -5   /* workspace missing or too small */
#define MX_ERR_NO_DEVICE    -6   /* no sm_100 device is current */
#define MX_ERR_TIMEOUT      -7   /* a bounded in-kernel wait gave up (device status) */

/* ---- element formats ([MXFP4-OAS] Sec.2, [MX-TRAIN]) -------------------- */
#define MX_E2M1 0   /* FP4: magnitudes {0,0.5,1,1.5,2,3,4,6}, sign-magnitude nibble */
#define MX_E3M0 1   /* FP4 exponent-only: {0, 2^-2 .. 2^4}, sign-magnitude nibble */
#define MX_E2M3 2   /* FP6 (OCP MXFP6), max 7.5, one code per byte (low 6 bits) */
#define MX_E3M2 3   /* FP6 (OCP MXFP6), max 28, one code per byte (low 6 bits) */
#define MX_INT4 4   /* symmetric: -7..7 two's-complement nibble; asymmetric: 0..15 */

/* ---- block-scale formats ([MXFP4-OAS] Sec.2, [FINER]) -------------------- */
#define MX_SCALE_E8M0  0   /* 2^(code-127); 0xFF = NaN */
#define MX_SCALE_UE4M3 1   /* unsigned E4M3, bias 7: 2^-9 .. 448; 0x7F = NaN */
#define MX_SCALE_UE5M3 2   /* unsigned E5M3, bias 15: 2^-17 .. 1.75*2^16; 0xFF = NaN */

/* ---- shared-scale rules ----------------------------------------------- */
/* FLOOR: 2^(floor(log2 amax) - emax_elem) (OCP MX).  CEIL: smallest power of
 * two with amax <= max_elem * 2^k (no overflow).  OAS: FLOOR, doubled when
 * amax / 2^k_floor > oas_tau ([MXFP4-OAS] Sec.4).  NEAREST: UE4M3/UE5M3 scale
 * = RTNE((amax / max_elem) / s_T), saturating (NVFP4-style).  FLOOR / CEIL /
 * OAS with a UE4M3 / UE5M3 format store power-of-two scales in that format
 * ([MXFP4-OAS] Sec.4: E4M3 used as power-of-two scales for block 16). */
#define MX_RULE_FLOOR   0
#define MX_RULE_CEIL    1
#define MX_RULE_OAS     2
#define MX_RULE_NEAREST 3
/* MSE: MSE-optimal block scales ([BRIDGING] sec. 2.2: MSE-optimised grids;
 * the pages name the objective, not the search).  Row axis, MX_ROUND_RTNE,
 * symmetric, no macro scale or rotation.
 *   E8M0 (block 32, any element type): the exponent among k_floor and
 *   k_floor + 1 whose nearest-even codes leave the smaller block squared
 *   error, 4^k sum (v - q)^2 with v = binary32(x 2^-k), each sum in binary64
 *   in element order, ties to k_floor.
 *   UE4M3 / UE5M3 (E2M1, blocks of 8, 16 or 32): for the tensor scale s_T
 *   (MX_TS_NONE: 1, MX_TS_GIVEN: *tensor_scale) every block takes the code
 *   c, over all finite codes, with the smallest sum (x - x_hat)^2, x_hat =
 *   (q s_c) s_T and q the nearest-even value of x * RN(1 / RN(s_c s_T));
 *   binary64 differences, squares and element-order sums, ties to the lower
 *   code.  With MX_TS_COMPUTE the global and the group scales alternate
 *   (four rounds from the amax rule's s_T): the group step above, then
 *   s_T = sum x u / sum u^2 with u = q s_c held fixed (binary64 sums rounded
 *   once to binary32); the final s_T is written to *tensor_scale.  Dequantize
 *   and GEMM read these scales like nearest ones. */
#define MX_RULE_MSE     4

/* ---- element rounding ([MX-TRAIN]) ------------------------------------- */
#define MX_ROUND_RTNE       0   /* nearest, ties to the even code, saturating */
#define MX_ROUND_CEIL       1   /* next grid point up in magnitude, saturating */
#define MX_ROUND_STOCHASTIC 2   /* up with probability (|v|-lo)/(hi-lo); Philox4x32-10 */

/* ---- block axis ([MX-TRAIN]: row-wise, column-wise, 2D) ----------------- */
#define MX_AXIS_ROW 0   /* 1 x B blocks along a row (the contiguous dimension) */
#define MX_AXIS_COL 1   /* B x 1 blocks along a column */
#define MX_AXIS_2D  2   /* 32 x 32 tiles */

/* ---- dtypes ------------------------------------------------------------- */
#define MX_DT_BF16 0
#define MX_DT_FP32 1

/* ---- per-tensor FP32 scale (NVFP4, UE*-S; [FINER]) ----------------------- */
#define MX_TS_NONE    0   /* s_T = 1 */
#define MX_TS_COMPUTE 1   /* s_T = amax_T / (max_elem * max_scale), written to *tensor_scale */
#define MX_TS_GIVEN   2   /* s_T read from *tensor_scale (device) */
#define MX_TS_AMAX    3   /* as MX_TS_COMPUTE, with amax_T taken from the workspace's amax
                             word (left there by mx_tensor_amax, then reduced across the
                             shards of a row-partitioned tensor) instead of a pre-pass */

typedef struct {
    int32_t elem;          /* MX_E2M1 ... MX_INT4 */
    int32_t scale_fmt;     /* MX_SCALE_* */
    int32_t rule;          /* MX_RULE_* */
    float   oas_tau;       /* OAS threshold on amax / 2^k_floor (E2M1: 6 = ceil, 8 = floor) */
    int32_t block;         /* elements per block along the axis: 8,16,32,64,128,256 (row);
                              8,16,32 (col); 32 (2D) */
    int32_t axis;          /* MX_AXIS_* */
    int32_t round;         /* MX_ROUND_* */
    int32_t asymmetric;    /* 1: per-block bf16 offset (INT4: min; FP: (max+min)/2) */
    int32_t tensor_scale;  /* MX_TS_* (UE4M3/UE5M3 with MX_RULE_NEAREST only) */
    int32_t macro_block;   /* 0 or 128: MBS macro scale per 1x128 along the axis */
    int32_t hadamard;      /* 0, 16 or 32: block Hadamard rotation (mx_hadamard_quantize) */
    int32_t sf_layout;     /* scales layout: 0 canonical (below); 1 tcgen05 chunks (row axis
                              only; rows % 128 == 0, (cols / block) % 4 == 0): for row r and
                              scale j of a row holding S = cols / block scales, byte
                              ((r/128)*(S/4) + j/4)*512 + (r%32)*16 + ((r/32)%4)*4 + j%4,
                              the layout mx_gemm copies into tensor memory.  With FP6
                              elements it also sets the code layout to the dense operand
                              form: every 16 codes of a row in 12 bytes (code i at bits
                              [6i, 6i+6) of the little-endian group), groups back to back,
                              6 bits per element; FP4 codes are unchanged */
    uint64_t seed;         /* stochastic-rounding key */
} mx_config;

typedef struct {
    int64_t codes_bytes;     /* packed element codes */
    int64_t n_scales;        /* one byte per block */
    int64_t n_macro;         /* one E4M3 byte per macro block (0 without MBS) */
    int64_t n_offsets;       /* one bf16 per block (0 unless asymmetric) */
    int64_t workspace_bytes; /* scratch for mx_quantize / mx_hadamard_quantize */
    int64_t n_blocks;
} mx_sizes;

/* Length of every `stats` buffer (binary64, device):
 * [0] sum x^2   [1] sum (x - x_hat)^2   [2] sum (x_hat - x)   [3] #flushed
 * (x != 0, x_hat == 0)   [4] #nonzero x   [5] MSE   [6] R-MSE   [7] QSNR dB
 * (Eq. (1) of [MXFP4-OAS] Sec.3)   [8] mean bias   [9] flush-to-zero share
 * [10] element count   [11..15] reserved (0).
 * A zero signal gives QSNR NaN; a zero error gives +inf. */
#define MX_STATS_LEN 16

/* Sizes of the outputs of mx_quantize for a rows x cols input. */
int mx_query_sizes(const mx_config *cfg, int64_t rows, int64_t cols, mx_sizes *out);

/*
 * mx_quantize -- block quantization of a row-major rows x cols tensor
 * ([MXFP4-OAS] Sec.2/Sec.4, [FINER], [MX-TRAIN]).
 *   x          device, bf16 or fp32 (x_dtype), row-major, 16-byte aligned.
 *   codes      device out.  4-bit formats: rows x cols/2 bytes, element (r, 2j)
 *              in the low nibble of byte (r, j); FP6: rows x cols bytes, or
 *              rows x cols x 3/4 in the dense form of cfg->sf_layout == 1.
 *              The layout is the same for every axis.
 *   scales     device out, one byte per block: row axis [rows][cols/B], column
 *              axis [rows/B][cols], 2D [rows/32][cols/32] (cfg->sf_layout == 0), or
 *              the tcgen05 chunk layout (cfg->sf_layout == 1, row axis).
 *   tensor_scale  device float: written (MX_TS_COMPUTE) or read (MX_TS_GIVEN);
 *              may be NULL with MX_TS_NONE.
 *   macro_scales  device out, E4M3 per 1x128 macro block along the axis
 *              (row / 2D: [rows][cols/128]; column: [rows/128][cols]); needed iff
 *              cfg->macro_block == 128.
 *   offsets    device out, bf16 bits per block (same layout as scales); needed
 *              iff cfg->asymmetric.
 *   stats      device out, MX_STATS_LEN doubles, or NULL: fidelity of the
 *              dequantized tensor against x, fused into the same pass.
 *   workspace  device scratch of sizes.workspace_bytes (needed when stats != NULL
 *              or cfg->tensor_scale == MX_TS_COMPUTE), control words zeroed
 *              before first use (see Ownership above).  The last CTA of the
 *              quantizer launch sums the statistics and clears the control
 *              words: one launch per call (two with a computed tensor scale:
 *              the amax pre-pass, then the quantizer).
 * Shapes: cols % 32 == 0 always (lanes walk rows in 32-element chunks),
 * rows * cols < 2^32, cols % block == 0 (row), rows % block == 0 (column),
 * rows % 32 == 0 (2D), % 128 along the axis for MBS.  Block non-finite
 * values give the NaN scale code and zero element codes.
 */
int mx_quantize(const mx_config *cfg, const void *x, int32_t x_dtype, int64_t rows, int64_t cols,
                void *codes, uint8_t *scales, float *tensor_scale, uint8_t *macro_scales,
                uint16_t *offsets, double *stats, void *workspace, int64_t workspace_bytes,
                void *stream);

/*
 * mx_quantize_noalloc -- mx_quantize for callers that cannot allocate device
 * memory: plain C callers holding no device allocator, code running while a
 * CUDA graph is being captured (cudaMalloc is not allowed there), services
 * that reserved all of HBM up front.  The pages have no counterpart: this is
 * an interface convenience, not part of the method.
 *   Same arguments and results as mx_quantize, without the workspace: the
 *   scratch lives in a fixed device array inside the library (262,400 bytes,
 *   the most mx_quantize can need: a 256-byte header and one 64-byte record
 *   for each of at most 4096 CTAs), held by every GPU that loads the library
 *   until the process exits.  A configuration needing more scratch is
 *   rejected with MX_ERR_WORKSPACE.  Nothing is allocated: no cudaMalloc, no
 *   cudaFree, no allocating library routine.
 *   The first call on a device resolves the array's device address (once per
 *   device, with that device current); make that first call before any stream
 *   capture.  Every call shares the one array (zero at load; every call
 *   leaves its control words zero), so calls that overlap on the
 *   GPU -- on different streams, or from different threads -- race: order them
 *   on one stream.  A call that returns MX_ERR_CUDA queues a reset of the
 *   array's control words on `stream` before it returns.  Rotation
 *   (cfg->hadamard != 0, the mx_hadamard_quantize entry) is not covered, nor
 *   MX_TS_AMAX (its amax word is in a caller's workspace): MX_ERR_UNSUPPORTED,
 *   checked on the host before anything is queued.
 */
int mx_quantize_noalloc(const mx_config *cfg, const void *x, int32_t x_dtype, int64_t rows,
                        int64_t cols, void *codes, uint8_t *scales, float *tensor_scale,
                        uint8_t *macro_scales, uint16_t *offsets, double *stats, void *stream);

/*
 * mx_hadamard_quantize -- mx_quantize preceded, in the same pass, by the
 * block Hadamard rotation y = x H_n / sqrt(n), n = cfg->hadamard in {16, 32},
 * over groups of n consecutive elements along the block axis (the row
 * direction for 2D) ([BRIDGING] sec. 2.1-2.3: fused online rotation).
 * Sylvester ordering, butterflies (a, b) -> (a + b, a - b) in binary32 with
 * stride 1, 2, 4, ..., then a multiply by binary32(1/sqrt(n)).
 * Everything (scales, stats, tensor scale) refers to y.  `rotated` (device,
 * fp32 rows x cols, nullable) receives y.
 */
int mx_hadamard_quantize(const mx_config *cfg, const void *x, int32_t x_dtype, int64_t rows,
                         int64_t cols, void *codes, uint8_t *scales, float *tensor_scale,
                         uint8_t *macro_scales, uint16_t *offsets, double *stats,
                         float *rotated, void *workspace, int64_t workspace_bytes, void *stream);

/* One tensor of mx_quantize_group: mx_quantize's per-tensor arguments. */
typedef struct {
    const void *x;            /* device input, rows x cols, row-major */
    int64_t rows, cols;
    void *codes;              /* device out, as mx_quantize */
    uint8_t *scales;          /* device out, as mx_quantize */
    float *tensor_scale;      /* device, as mx_quantize (this tensor's own s_T) */
    uint8_t *macro_scales;    /* device out or NULL, as mx_quantize */
    uint16_t *offsets;        /* device out or NULL, as mx_quantize */
    double *stats;            /* device out or NULL: this tensor's statistics */
    void *workspace;          /* device scratch of this tensor, as mx_quantize */
    int64_t workspace_bytes;
} mx_quantize_item;

/*
 * mx_quantize_group -- mx_quantize of n tensors that share one configuration
 * and input dtype (for instance the activation and the weight of a layer, or
 * the weights of several layers), each with its own outputs, tensor scale and
 * statistics: the results are those of n mx_quantize calls (mx_hadamard_quantize
 * without `rotated` when cfg->hadamard), bit for bit ([MXFP4-OAS] Sec.2: every
 * block, and every tensor, is quantized on its own).  Shapes may differ.
 *   For E2M1 round-to-nearest-even symmetric configurations (not the MSE
 *   rule) on the row axis (with a rotation or a macro scale, blocks of 16 or
 *   32), and on the column axis or 2D tiles with bf16 input (no rotation, no
 *   macro scale), the tensors share one quantizer launch, up to 4 tensors a
 *   launch, the CTAs split among the tensors in proportion to their sizes;
 *   with a computed tensor scale one tensor-amax launch comes before it.
 *   Other configurations run as n calls in order.
 *   Items that need a workspace (stats != NULL, MX_TS_COMPUTE, MX_TS_AMAX)
 *   must each have their own (MX_ERR_INVALID when two overlap).  Every item is
 *   checked before anything is queued; a failing item fails the call with
 *   that item's error.  n >= 1.
 */
int mx_quantize_group(const mx_config *cfg, int32_t x_dtype, const mx_quantize_item *items, int32_t n,
                      void *stream);

/*
 * mx_tensor_amax -- the tensor-amax pre-pass alone, for a tensor split by rows
 * over several devices (one process per GPU): amax_T = max |x| (of the rotated
 * y when cfg->hadamard), NaN ignored ([FINER] per-tensor scale), folded into
 * the workspace's amax word (byte 0, the binary32 bits of amax_T, a max with
 * what the word holds).  cfg->tensor_scale must be MX_TS_AMAX, and the word
 * must hold zero or a partial amax.  The word keeps amax_T: the caller may
 * reduce it across ranks (a max of the 32-bit words, which order like the
 * non-negative floats they hold), then call mx_quantize /
 * mx_hadamard_quantize with the same cfg and workspace, which derives
 * s_T = amax_T / (max_elem * max_scale) from the word, writes it to
 * *tensor_scale and clears the word.  Shapes and errors as mx_quantize; no
 * outputs other than the word.  The pages have no multi-device procedure:
 * this is how the per-tensor scale stays the one of the whole tensor.
 */
int mx_tensor_amax(const mx_config *cfg, const void *x, int32_t x_dtype, int64_t rows, int64_t cols,
                   void *workspace, int64_t workspace_bytes, void *stream);

/*
 * mx_stats_finalize -- recomputes the derived entries [5..9] of a `stats`
 * buffer (device, MX_STATS_LEN doubles) from its sums [0..4] and element count
 * [10]: after the sums of several shards' calls were added together (a sum
 * reduction across ranks), the buffer then holds the whole tensor's MSE,
 * R-MSE, QSNR, bias and flush share ([MXFP4-OAS] Sec.3 Eq. (1)).
 */
int mx_stats_finalize(double *stats, void *stream);

/*
 * mx_dequantize -- x_hat from codes and scales ([MX-TRAIN] fake quantization).
 * x_hat = (q * s_b) * s_T (NEAREST rule); q * 2^k (power-of-two rules), times
 * the macro scale with MBS, plus the offset when asymmetric; each step one
 * binary32 operation.  NaN scale codes give NaN.  With cfg->hadamard != 0 the
 * normalised rotation (its own inverse) is applied afterwards, returning to
 * the input space.  out: device, rows x cols, bf16 (RNE) or fp32 (out_dtype).
 */
int mx_dequantize(const mx_config *cfg, const void *codes, const uint8_t *scales,
                  const float *tensor_scale, const uint8_t *macro_scales,
                  const uint16_t *offsets, int64_t rows, int64_t cols, void *out,
                  int32_t out_dtype, void *stream);

/*
 * mx_qsnr -- fidelity reductions of x_hat against x ([MXFP4-OAS] Sec.3 Eq. (1);
 * [MX-TRAIN] R-MSE; [FINER] per-block MSE): stats as above, and when
 * per_block_mse != NULL the mean squared error of every block of the given
 * block size and axis (layout of `scales`).  x, x_hat: device, bf16 or fp32;
 * rows * cols < 2^32.  Reduction order is fixed: results are reproducible
 * run to run.
 */
int64_t mx_qsnr_workspace_bytes(int64_t rows, int64_t cols);
int mx_qsnr(const void *x, int32_t x_dtype, const void *x_hat, int32_t x_hat_dtype, int64_t rows,
            int64_t cols, int32_t block, int32_t axis, double *stats, float *per_block_mse,
            void *workspace, int64_t workspace_bytes, void *stream);

/*
 * mx_gemm -- block-scaled FP4 GEMM on the tcgen05 tensor cores,
 * C[M x N] = A^Q (B^Q)^T with FP32 accumulation ([BRIDGING] sec. 2.3;
 * [MXFP4-OAS] Fig. 5).  A^Q: M x K E2M1 codes, B^Q: N x K E2M1 codes, both
 * row-major along K as written by mx_quantize (row axis).  Scales in the
 * tcgen05 chunk layout (ca/cb->sf_layout = 1, as mx_quantize wrote them).
 * MXFP4: block 32, E8M0 (ca/cb rule FLOOR, CEIL or OAS).  NVFP4: block 16,
 * UE4M3 NEAREST with tensor scales tsA/tsB (device floats; used when
 * ca/cb->tensor_scale != MX_TS_NONE, else 1).  MXFP6 ([MX-TRAIN]'s MX6;
 * tcgen05 kind::mxf8f6f4): E2M3 and / or E3M2 codes in the dense form
 * mx_quantize writes with sf_layout = 1 (16 codes in 12 bytes), block 32,
 * E8M0; N % 256 == 0; the copy into shared memory widens them to the
 * kind's one byte per element.  The same kind takes one FP6 operand with
 * one MXFP4 operand (E2M1 + E8M0 / 32, packed codes): [MX-TRAIN]'s MX6
 * weights and activations against MX4 gradients.  On this kind both operand
 * pointers must be 32-byte aligned.  Operands rotated by mx_hadamard_quantize
 * are accepted when both carry the same rotation (cfg->hadamard), since
 * (A H)(B H)^T = A B^T ([BRIDGING] sec. 2.3: rotated operands into the FP4
 * GEMM).  Any other pair: MX_ERR_UNSUPPORTED.  C: device, bf16 or fp32
 * (c_dtype), row-major M x N.  M % 128 == 0, N % 128 == 0, K % 256 == 0.
 * Tiles: 128 x 256 per SM (persistent) when N % 256 == 0, else 128 x 128.
 */
int mx_gemm(const mx_config *ca, const mx_config *cb, const void *Aq, const uint8_t *Asf,
            const void *Bq, const uint8_t *Bsf, const float *tsA, const float *tsB, int64_t M,
            int64_t N, int64_t K, void *C, int32_t c_dtype, void *stream);

/*
 * mx_gemm_qsnr -- post-operation QSNR ([MXFP4-OAS] Sec.3 Eq. (2)):
 * 10 log10(||A B^T||_F^2 / ||A B^T - A^Q (B^Q)^T||_F^2) with A [M x K] and
 * B [N x K] bf16 (device).  One persistent kernel forms both products of
 * every 128 x 256 (N % 256 == 0, else 128 x 128) output tile on the tensor
 * cores -- the block-scaled one (operand pairs as mx_gemm), then bf16 with
 * FP32 accumulation -- and its epilogue reduces sum C_ref^2 and
 * sum (C_ref - C_q)^2 (binary32 over 32 columns, then binary64) without
 * writing C; a second launch adds the per-CTA records in a fixed order.
 * stats: device, 3 doubles [sum C_ref^2, sum (C_ref - C_q)^2, QSNR dB].
 * workspace: mx_gemm_workspace_bytes() bytes (a fixed 16,640: the per-CTA
 * records, independent of the shape).  Shapes as mx_gemm.
 */
int64_t mx_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);
int mx_gemm_qsnr(const mx_config *ca, const mx_config *cb, const void *A, const void *B, int64_t M,
                 int64_t N, int64_t K, const void *Aq, const uint8_t *Asf, const void *Bq,
                 const uint8_t *Bsf, const float *tsA, const float *tsB, double *stats,
                 void *workspace, int64_t workspace_bytes, void *stream);

/*
 * mx_gemm_qsnr_finalize -- recomputes entry [2] (QSNR dB, [MXFP4-OAS] Sec.3
 * Eq. (2)) of a 3-double mx_gemm_qsnr stats buffer (device) from its two sums
 * [0] and [1]: after the sums of several row bands of A (each band's
 * mx_gemm_qsnr against the same B) were added together across ranks, the
 * buffer then holds the whole product's QSNR.  A zero reference gives NaN, a
 * zero error +inf.  The pages have no multi-device procedure: this is how
 * QSNR(AB) stays the one of the whole product when A is split by rows.
 */
int mx_gemm_qsnr_finalize(double *stats, void *stream);

/*
 * mx_mbs_gemm_scales -- an MBS operand ([MXFP4-OAS] Sec.4 Macro Block
 * Scaling: E2M1 codes, E8M0 scale X per 1 x 32 block, E4M3 macro scale S_M per
 * 1 x 128, x_hat = q X S_M) as an operand of mx_gemm's NVFP4 kind.  The pages
 * give MBS's GEMM (Fig. 5) but no data path for it; this is one: S_M X is an
 * E4M3 significand times a power of two, so with a per-tensor power of two
 * s_T = 2^t it is exactly a UE4M3 value when it falls in UE4M3's normal range.
 *   cfg          the MBS configuration the operand was quantized with (E2M1,
 *                E8M0, block 32, macro_block 128, row axis, canonical scales).
 *   scales       device, rows x cols/32 E8M0 codes (canonical).
 *   macro_scales device, rows x cols/128 E4M3 codes.
 *   sf16         device out, rows x cols/16 UE4M3 codes in the tcgen05 chunk
 *                layout: code(S_M X / s_T) for both 16-element halves of every
 *                32-block (round to nearest even; NaN scale -> 0x7F; zero
 *                block -> 0).
 *   tensor_scale device out, one float: s_T, with t chosen so that the largest
 *                folded value is below 2^8; values more than 13 binades below
 *                it are rounded into UE4M3's subnormals (inexact).
 *   workspace    control words as for mx_quantize (the first 256 bytes).
 * Then mx_gemm / mx_gemm_qsnr with an NVFP4 configuration (block 16, UE4M3,
 * NEAREST, sf_layout 1, tensor_scale MX_TS_GIVEN) on the same codes, sf16
 * and tensor_scale.  rows % 128 == 0, cols % 128 == 0.  Two launches.
 */
int mx_mbs_gemm_scales(const mx_config *cfg, const uint8_t *scales, const uint8_t *macro_scales,
                       int64_t rows, int64_t cols, uint8_t *sf16, float *tensor_scale,
                       void *workspace, int64_t workspace_bytes, void *stream);

/*
 * mx_tensor_peak -- tensor-core ceiling probe for the roofline of mx_gemm (the
 * pages have no counterpart; it measures the device, not the method).  One
 * CTA per SM issues `iters` stages of four 128 x 256 x K block-scaled MMAs of
 * a kind -- 1: kind::mxf4 (K = 64), 2: kind::mxf4nvf4 (K = 64), 3:
 * kind::mxf8f6f4 (K = 32) -- on operands held in shared memory (zero codes,
 * unit scales), with no global memory traffic; sf_copies 1 adds the
 * per-stage scale copies into tensor memory that mx_gemm's stages make (into
 * one slot of columns), 2 the same copies rotating over four slots as
 * mx_gemm's stages do.
 * *flops (host) receives the launch's flop count: time the launch on
 * `stream` (CUDA events) for the throughput.  1 <= iters <= 2^22.
 * Asynchronous like the other calls.
 */
int mx_tensor_peak(int32_t kind, int64_t iters, int32_t sf_copies, double *flops, void *stream);

/* Status words of the bounded in-kernel waits: reads and clears them
 * (synchronises `stream`).  *status = 0 when no wait gave up, else the code of
 * the first wait that did: 1-3 and 11-14 the GEMM pipelines (128 x 128 and
 * persistent 128 x 256 tiles), 15-19 the fused QSNR(AB) kernel, 20 the
 * tensor-core probe, 21-22 the E2M1 nearest-even quantizer's TMA ring, 31-32
 * the other element types' ring.  A
 * kernel whose wait gave up has left its loop early, so its outputs are
 * incomplete; the library has no counterpart on the pages. */
int mx_device_status(void *stream, int32_t *status);

/* Human-readable text of a status code. */
const char *mx_strerror(int code);

/* Library version string. */
const char *mx_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MX_H_ */
