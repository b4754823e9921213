"""B200 (sm_100a) microscaling block quantization.

Thin Python binding over the C ABI of ``include/mx.h`` (``libmx_b200.so``):
argument marshalling only.  Every step of the method runs in the library's
CUDA kernels; torch provides device memory and streams.  There is no CPU
fallback: if the library is missing, every call raises.

Low-level functions carry the C names (``mx_quantize``, ``mx_dequantize``,
``mx_hadamard_quantize``, ``mx_qsnr``, ``mx_gemm``, ``mx_gemm_qsnr``, ...)
and take raw device pointers; the high-level helpers (``quantize``,
``dequantize``, ``qsnr``, ``gemm``, ``gemm_qsnr``) allocate the outputs with
torch and call them.
"""
from __future__ import annotations

import ctypes as C
import dataclasses
import os

import torch

from . import inputs  # noqa: F401  (seeded synthetic workloads)

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libmx_b200.so")

# ---- constants of include/mx.h ------------------------------------------
MX_OK = 0
E2M1, E3M0, E2M3, E3M2, INT4 = 0, 1, 2, 3, 4
SCALE_E8M0, SCALE_UE4M3, SCALE_UE5M3 = 0, 1, 2
RULE_FLOOR, RULE_CEIL, RULE_OAS, RULE_NEAREST, RULE_MSE = 0, 1, 2, 3, 4
ROUND_RTNE, ROUND_CEIL, ROUND_STOCHASTIC = 0, 1, 2
AXIS_ROW, AXIS_COL, AXIS_2D = 0, 1, 2
DT_BF16, DT_FP32 = 0, 1
TS_NONE, TS_COMPUTE, TS_GIVEN, TS_AMAX = 0, 1, 2, 3
STATS_LEN = 16
STAT_NAMES = ["sum_x2", "sum_e2", "sum_e", "n_ftz", "n_nonzero", "mse", "rmse", "qsnr_db",
              "bias", "ftz_frac", "count"]

FP6 = (E2M3, E3M2)


class mx_config(C.Structure):
    _fields_ = [("elem", C.c_int32), ("scale_fmt", C.c_int32), ("rule", C.c_int32),
                ("oas_tau", C.c_float), ("block", C.c_int32), ("axis", C.c_int32),
                ("round", C.c_int32), ("asymmetric", C.c_int32), ("tensor_scale", C.c_int32),
                ("macro_block", C.c_int32), ("hadamard", C.c_int32), ("sf_layout", C.c_int32),
                ("seed", C.c_uint64)]


class mx_quantize_item(C.Structure):
    _fields_ = [("x", C.c_void_p), ("rows", C.c_int64), ("cols", C.c_int64), ("codes", C.c_void_p),
                ("scales", C.c_void_p), ("tensor_scale", C.c_void_p), ("macro_scales", C.c_void_p),
                ("offsets", C.c_void_p), ("stats", C.c_void_p), ("workspace", C.c_void_p),
                ("workspace_bytes", C.c_int64)]


class mx_sizes(C.Structure):
    _fields_ = [("codes_bytes", C.c_int64), ("n_scales", C.c_int64), ("n_macro", C.c_int64),
                ("n_offsets", C.c_int64), ("workspace_bytes", C.c_int64), ("n_blocks", C.c_int64)]


@dataclasses.dataclass(frozen=True)
class Config:
    """One quantization configuration (fields of ``mx_config``)."""
    elem: int = E2M1
    scale_fmt: int = SCALE_E8M0
    rule: int = RULE_FLOOR
    oas_tau: float = 7.0
    block: int = 32
    axis: int = AXIS_ROW
    round: int = ROUND_RTNE
    asymmetric: int = 0
    tensor_scale: int = TS_NONE
    macro_block: int = 0
    hadamard: int = 0
    seed: int = 0
    sf_layout: int = 0

    def c(self) -> mx_config:
        return mx_config(self.elem, self.scale_fmt, self.rule, self.oas_tau, self.block,
                         self.axis, self.round, self.asymmetric, self.tensor_scale,
                         self.macro_block, self.hadamard, self.sf_layout, self.seed)


MXFP4 = Config()
NVFP4 = Config(block=16, scale_fmt=SCALE_UE4M3, rule=RULE_NEAREST, tensor_scale=TS_COMPUTE)


class MXError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {code} ({mx_strerror(code)})")
        self.code = code


_lib = None


def lib() -> C.CDLL:
    """The loaded CUDA library; raises when it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -c 'import __graft_entry__ as g; g.build()'`")
        L = C.CDLL(LIB_PATH)
        P, i32, i64 = C.c_void_p, C.c_int32, C.c_int64
        cfgp = C.POINTER(mx_config)
        L.mx_query_sizes.argtypes = [cfgp, i64, i64, C.POINTER(mx_sizes)]
        L.mx_quantize.argtypes = [cfgp, P, i32, i64, i64, P, P, P, P, P, P, P, i64, P]
        L.mx_hadamard_quantize.argtypes = [cfgp, P, i32, i64, i64, P, P, P, P, P, P, P, P, i64, P]
        L.mx_quantize_noalloc.argtypes = [cfgp, P, i32, i64, i64, P, P, P, P, P, P, P]
        L.mx_quantize_group.argtypes = [cfgp, i32, C.POINTER(mx_quantize_item), i32, P]
        L.mx_dequantize.argtypes = [cfgp, P, P, P, P, P, i64, i64, P, i32, P]
        L.mx_qsnr_workspace_bytes.argtypes = [i64, i64]
        L.mx_qsnr_workspace_bytes.restype = i64
        L.mx_qsnr.argtypes = [P, i32, P, i32, i64, i64, i32, i32, P, P, P, i64, P]
        L.mx_gemm_workspace_bytes.argtypes = [i64, i64, i64]
        L.mx_gemm_workspace_bytes.restype = i64
        L.mx_gemm.argtypes = [cfgp, cfgp, P, P, P, P, P, P, i64, i64, i64, P, i32, P]
        L.mx_gemm_qsnr.argtypes = [cfgp, cfgp, P, P, i64, i64, i64, P, P, P, P, P, P, P, P, i64, P]
        L.mx_mbs_gemm_scales.argtypes = [cfgp, P, P, i64, i64, P, P, P, i64, P]
        L.mx_device_status.argtypes = [P, C.POINTER(i32)]
        L.mx_tensor_amax.argtypes = [cfgp, P, i32, i64, i64, P, i64, P]
        L.mx_stats_finalize.argtypes = [P, P]
        L.mx_gemm_qsnr_finalize.argtypes = [P, P]
        L.mx_tensor_peak.argtypes = [i32, i64, i32, C.POINTER(C.c_double), P]
        L.mx_strerror.argtypes = [C.c_int]
        L.mx_strerror.restype = C.c_char_p
        L.mx_version.restype = C.c_char_p
        for f in ("mx_query_sizes", "mx_quantize", "mx_quantize_group", "mx_quantize_noalloc",
                  "mx_hadamard_quantize", "mx_dequantize",
                  "mx_qsnr", "mx_gemm", "mx_gemm_qsnr", "mx_mbs_gemm_scales", "mx_device_status",
                  "mx_tensor_amax", "mx_stats_finalize", "mx_gemm_qsnr_finalize", "mx_tensor_peak"):
            getattr(L, f).restype = C.c_int
        _lib = L
    return _lib


def mx_strerror(code: int) -> str:
    return lib().mx_strerror(code).decode()


def mx_version() -> str:
    return lib().mx_version().decode()


# ---- marshalling helpers --------------------------------------------------
def _p(t: torch.Tensor | None):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream) -> C.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return DT_BF16
    if t.dtype == torch.float32:
        return DT_FP32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _check(fn: str, rc: int) -> None:
    if rc != MX_OK:
        raise MXError(fn, rc)


def _cuda2d(x: torch.Tensor, name: str) -> None:
    if not x.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if x.dim() != 2 or not x.is_contiguous():
        raise ValueError(f"{name} must be a contiguous 2-D tensor")


def query_sizes(cfg: Config, rows: int, cols: int) -> mx_sizes:
    s = mx_sizes()
    c = cfg.c()
    _check("mx_query_sizes", lib().mx_query_sizes(C.byref(c), rows, cols, C.byref(s)))
    return s


# ---- low-level calls (C names) -------------------------------------------
def mx_quantize(cfg: Config, x, x_dtype, rows, cols, codes, scales, tensor_scale, macro, offsets,
                stats, workspace, workspace_bytes, stream) -> int:
    c = cfg.c()
    return lib().mx_quantize(C.byref(c), x, x_dtype, rows, cols, codes, scales, tensor_scale,
                             macro, offsets, stats, workspace, workspace_bytes, stream)


def mx_quantize_group(cfg: Config, x_dtype, items, n, stream) -> int:
    """``items``: a ctypes array of ``mx_quantize_item``."""
    c = cfg.c()
    return lib().mx_quantize_group(C.byref(c), x_dtype, items, n, stream)


def mx_tensor_amax(cfg: Config, x, x_dtype, rows, cols, workspace, workspace_bytes, stream) -> int:
    c = cfg.c()
    return lib().mx_tensor_amax(C.byref(c), x, x_dtype, rows, cols, workspace, workspace_bytes, stream)


def mx_stats_finalize(stats, stream) -> int:
    return lib().mx_stats_finalize(stats, stream)


def mx_gemm_qsnr_finalize(stats, stream) -> int:
    return lib().mx_gemm_qsnr_finalize(stats, stream)


def mx_quantize_noalloc(cfg: Config, x, x_dtype, rows, cols, codes, scales, tensor_scale, macro,
                        offsets, stats, stream) -> int:
    """mx_quantize without a workspace argument, for callers that cannot
    allocate device memory; its scratch is a fixed array inside the library
    shared by all calls (order the calls on one stream)."""
    c = cfg.c()
    return lib().mx_quantize_noalloc(C.byref(c), x, x_dtype, rows, cols, codes, scales,
                                     tensor_scale, macro, offsets, stats, stream)


def mx_hadamard_quantize(cfg: Config, x, x_dtype, rows, cols, codes, scales, tensor_scale, macro,
                         offsets, stats, rotated, workspace, workspace_bytes, stream) -> int:
    c = cfg.c()
    return lib().mx_hadamard_quantize(C.byref(c), x, x_dtype, rows, cols, codes, scales,
                                      tensor_scale, macro, offsets, stats, rotated, workspace,
                                      workspace_bytes, stream)


def mx_dequantize(cfg: Config, codes, scales, tensor_scale, macro, offsets, rows, cols, out,
                  out_dtype, stream) -> int:
    c = cfg.c()
    return lib().mx_dequantize(C.byref(c), codes, scales, tensor_scale, macro, offsets, rows, cols,
                               out, out_dtype, stream)


def mx_qsnr(x, x_dtype, xh, xh_dtype, rows, cols, block, axis, stats, per_block_mse, workspace,
            workspace_bytes, stream) -> int:
    return lib().mx_qsnr(x, x_dtype, xh, xh_dtype, rows, cols, block, axis, stats, per_block_mse,
                         workspace, workspace_bytes, stream)


def mx_gemm(ca: Config, cb: Config, Aq, Asf, Bq, Bsf, tsA, tsB, M, N, K, C_out, c_dtype,
            stream) -> int:
    a, b = ca.c(), cb.c()
    return lib().mx_gemm(C.byref(a), C.byref(b), Aq, Asf, Bq, Bsf, tsA, tsB, M, N, K, C_out,
                         c_dtype, stream)


def mx_gemm_qsnr(ca: Config, cb: Config, A, B, M, N, K, Aq, Asf, Bq, Bsf, tsA, tsB, stats,
                 workspace, workspace_bytes, stream) -> int:
    a, b = ca.c(), cb.c()
    return lib().mx_gemm_qsnr(C.byref(a), C.byref(b), A, B, M, N, K, Aq, Asf, Bq, Bsf, tsA, tsB,
                              stats, workspace, workspace_bytes, stream)


def mx_mbs_gemm_scales(cfg: Config, scales, macro, rows, cols, sf16, tensor_scale, workspace,
                       workspace_bytes, stream) -> int:
    c = cfg.c()
    return lib().mx_mbs_gemm_scales(C.byref(c), scales, macro, rows, cols, sf16, tensor_scale, workspace,
                                    workspace_bytes, stream)


def mx_device_status(stream=None) -> int:
    st = C.c_int32(0)
    _check("mx_device_status", lib().mx_device_status(_stream(stream), C.byref(st)))
    return st.value


# ---- high-level helpers ----------------------------------------------------
@dataclasses.dataclass
class Quantized:
    """Outputs of one quantize call (device tensors)."""
    cfg: Config
    rows: int
    cols: int
    codes: torch.Tensor          # uint8, packed
    scales: torch.Tensor         # uint8, one per block
    tensor_scale: torch.Tensor   # float32[1]
    macro: torch.Tensor | None   # uint8 E4M3 per macro block
    offsets: torch.Tensor | None  # int16 (bf16 bits) per block
    stats: torch.Tensor | None   # float64[16]
    rotated: torch.Tensor | None = None


class Workspace:
    """Caller-owned scratch buffer, reused across calls.  Allocated zeroed: its
    first 256 bytes are the library's control words, which must be zero before
    the first call and which every call leaves zero."""

    def __init__(self, device=None):
        self.device = device
        self.buf: torch.Tensor | None = None

    def get(self, nbytes: int, device) -> torch.Tensor:
        if self.buf is None or self.buf.numel() < nbytes or self.buf.device != device:
            self.buf = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)
        return self.buf


_default_ws: dict = {}


def _ws(nbytes: int, device) -> torch.Tensor:
    w = _default_ws.setdefault(str(device), Workspace())
    return w.get(nbytes, device)


def alloc_outputs(cfg: Config, rows: int, cols: int, device, stats: bool = True,
                  rotated: bool = False, tensor_scale: torch.Tensor | None = None) -> Quantized:
    s = query_sizes(cfg, rows, cols)
    codes = torch.empty(max(s.codes_bytes, 16), dtype=torch.uint8, device=device)
    scales = torch.empty(max(s.n_scales, 16), dtype=torch.uint8, device=device)
    ts = tensor_scale if tensor_scale is not None else torch.ones(1, dtype=torch.float32, device=device)
    macro = torch.empty(max(s.n_macro, 16), dtype=torch.uint8, device=device) if cfg.macro_block else None
    offs = torch.empty(max(s.n_offsets, 8), dtype=torch.int16, device=device) if cfg.asymmetric else None
    st = torch.empty(STATS_LEN, dtype=torch.float64, device=device) if stats else None
    rot = torch.empty((rows, cols), dtype=torch.float32, device=device) if rotated else None
    return Quantized(cfg, rows, cols, codes[: s.codes_bytes], scales[: s.n_scales], ts,
                     None if macro is None else macro[: s.n_macro],
                     None if offs is None else offs[: s.n_offsets], st, rot)


def quantize(x: torch.Tensor, cfg: Config = MXFP4, *, stats: bool = True,
             tensor_scale: torch.Tensor | None = None, rotated: bool = False,
             out: Quantized | None = None, stream=None,
             workspace: torch.Tensor | None = None) -> Quantized:
    """Block-quantize a 2-D bf16/fp32 CUDA tensor (``mx_quantize``, or
    ``mx_hadamard_quantize`` when ``cfg.hadamard`` is set).  ``workspace``:
    a caller's scratch (uint8, at least ``query_sizes(...).workspace_bytes``,
    control words zero), needed with ``TS_AMAX`` to carry the amax.  Without
    it the call uses one scratch per device, so calls that may run at the
    same time on different streams must each pass their own."""
    _cuda2d(x, "x")
    rows, cols = x.shape
    q = out if out is not None else alloc_outputs(cfg, rows, cols, x.device, stats, rotated,
                                                  tensor_scale)
    ws = workspace if workspace is not None else _ws(query_sizes(cfg, rows, cols).workspace_bytes, x.device)
    st = _stream(stream)
    if cfg.hadamard:
        rc = mx_hadamard_quantize(cfg, _p(x), _dtype_code(x), rows, cols, _p(q.codes), _p(q.scales),
                                  _p(q.tensor_scale), _p(q.macro), _p(q.offsets), _p(q.stats),
                                  _p(q.rotated), _p(ws), ws.numel(), st)
        _check("mx_hadamard_quantize", rc)
    else:
        rc = mx_quantize(cfg, _p(x), _dtype_code(x), rows, cols, _p(q.codes), _p(q.scales),
                         _p(q.tensor_scale), _p(q.macro), _p(q.offsets), _p(q.stats), _p(ws),
                         ws.numel(), st)
        _check("mx_quantize", rc)
    return q


def quantize_group(xs, cfg: Config = MXFP4, *, stats: bool = True, outs=None, stream=None,
                   workspaces=None) -> list:
    """Block-quantize several 2-D CUDA tensors of one dtype with one
    configuration (``mx_quantize_group``): the same results as one
    ``quantize`` per tensor, with the tensors sharing launches.  ``outs`` /
    ``workspaces``: optional lists with one entry per tensor (each tensor that
    needs scratch gets its own; by default one scratch per position and
    device)."""
    xs = list(xs)
    if not xs:
        return []
    for i, x in enumerate(xs):
        _cuda2d(x, f"xs[{i}]")
    dt = _dtype_code(xs[0])
    if any(_dtype_code(x) != dt for x in xs):
        raise TypeError("every tensor of a group has the same dtype")
    qs = list(outs) if outs is not None else [alloc_outputs(cfg, *x.shape, x.device, stats) for x in xs]
    items = (mx_quantize_item * len(xs))()
    keep = []
    for i, (x, q) in enumerate(zip(xs, qs)):
        rows, cols = x.shape
        if workspaces is not None:
            ws = workspaces[i]
        else:
            nbytes = query_sizes(cfg, rows, cols).workspace_bytes
            w = _default_ws.setdefault(str(x.device) if i == 0 else f"{x.device}#{i}", Workspace())
            ws = w.get(nbytes, x.device)
        keep.append(ws)
        items[i] = mx_quantize_item(x.data_ptr(), rows, cols, q.codes.data_ptr(), q.scales.data_ptr(),
                                    q.tensor_scale.data_ptr(), _ptr_or_none(q.macro), _ptr_or_none(q.offsets),
                                    _ptr_or_none(q.stats), ws.data_ptr(), ws.numel())
    _check("mx_quantize_group", mx_quantize_group(cfg, dt, items, len(xs), _stream(stream)))
    return qs


def _ptr_or_none(t: torch.Tensor | None):
    return None if t is None else t.data_ptr()


def tensor_amax(x: torch.Tensor, cfg: Config, workspace: torch.Tensor, stream=None) -> None:
    """Fold max |x| (of the rotated tensor with ``cfg.hadamard``) into the
    amax word at byte 0 of ``workspace`` (``mx_tensor_amax``; ``cfg`` with
    ``tensor_scale=TS_AMAX``)."""
    _cuda2d(x, "x")
    rows, cols = x.shape
    rc = mx_tensor_amax(cfg, _p(x), _dtype_code(x), rows, cols, _p(workspace), workspace.numel(),
                        _stream(stream))
    _check("mx_tensor_amax", rc)


def stats_finalize(stats: torch.Tensor, stream=None) -> torch.Tensor:
    """Recompute MSE / R-MSE / QSNR / bias / flush share of a stats buffer from
    its sums and count, in place (``mx_stats_finalize``)."""
    _check("mx_stats_finalize", mx_stats_finalize(_p(stats), _stream(stream)))
    return stats


def tensor_peak(kind: int, iters: int, sf_copies: int = 0, stream=None) -> float:
    """Launch the tensor-core ceiling probe (``mx_tensor_peak``; kind 1
    kind::mxf4, 2 kind::mxf4nvf4, 3 kind::mxf8f6f4) on ``stream`` and return
    the launch's flop count; the caller times the launch."""
    f = C.c_double(0.0)
    _check("mx_tensor_peak", lib().mx_tensor_peak(kind, iters, int(sf_copies), C.byref(f), _stream(stream)))
    return f.value


def gemm_qsnr_finalize(stats: torch.Tensor, stream=None) -> torch.Tensor:
    """Recompute the dB entry of a QSNR(AB) stats buffer (float64[3] on the
    device) from its two sums, in place (``mx_gemm_qsnr_finalize``)."""
    _check("mx_gemm_qsnr_finalize", mx_gemm_qsnr_finalize(_p(stats), _stream(stream)))
    return stats


def new_workspace(cfg: Config, rows: int, cols: int, device) -> torch.Tensor:
    """A zeroed scratch buffer for ``quantize`` / ``tensor_amax``."""
    return torch.zeros(query_sizes(cfg, rows, cols).workspace_bytes, dtype=torch.uint8, device=device)


def dequantize(q: Quantized, out_dtype: torch.dtype = torch.float32, stream=None,
               out: torch.Tensor | None = None) -> torch.Tensor:
    """x_hat from a ``Quantized`` (``mx_dequantize``); with a rotation the
    result is rotated back to the input space."""
    cfg = q.cfg
    if out is None:
        out = torch.empty((q.rows, q.cols), dtype=out_dtype, device=q.codes.device)
    rc = mx_dequantize(cfg, _p(q.codes), _p(q.scales), _p(q.tensor_scale), _p(q.macro),
                       _p(q.offsets), q.rows, q.cols, _p(out), _dtype_code(out), _stream(stream))
    _check("mx_dequantize", rc)
    return out


def qsnr(x: torch.Tensor, x_hat: torch.Tensor, block: int = 0, axis: int = AXIS_ROW,
         per_block: bool = False, stream=None):
    """Fidelity statistics of x_hat against x (``mx_qsnr``): float64[16] on
    the device, and the per-block MSE when ``per_block``."""
    _cuda2d(x, "x")
    _cuda2d(x_hat, "x_hat")
    rows, cols = x.shape
    st = torch.empty(STATS_LEN, dtype=torch.float64, device=x.device)
    pb = None
    if per_block:
        if axis == AXIS_ROW:
            nb = rows * (cols // block)
        elif axis == AXIS_COL:
            nb = (rows // block) * cols
        else:
            nb = (rows // 32) * (cols // 32)
        pb = torch.empty(nb, dtype=torch.float32, device=x.device)
    ws = _ws(lib().mx_qsnr_workspace_bytes(rows, cols), x.device)
    rc = mx_qsnr(_p(x), _dtype_code(x), _p(x_hat), _dtype_code(x_hat), rows, cols,
                 block if per_block else 0, axis, _p(st), _p(pb), _p(ws), ws.numel(),
                 _stream(stream))
    _check("mx_qsnr", rc)
    return st, pb


def gemm(qa: Quantized, qb: Quantized, out_dtype: torch.dtype = torch.bfloat16,
         stream=None, out: torch.Tensor | None = None) -> torch.Tensor:
    """C = A^Q (B^Q)^T on the tcgen05 tensor cores (``mx_gemm``)."""
    M, K = qa.rows, qa.cols
    N = qb.rows
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=qa.codes.device)
    rc = mx_gemm(qa.cfg, qb.cfg, _p(qa.codes), _p(qa.scales), _p(qb.codes), _p(qb.scales),
                 _p(qa.tensor_scale), _p(qb.tensor_scale), M, N, K, _p(out), _dtype_code(out),
                 _stream(stream))
    _check("mx_gemm", rc)
    return out


def mbs_gemm_operand(q: Quantized, stream=None) -> Quantized:
    """An MBS-quantized tensor (block 32, E8M0, macro_block 128, canonical
    scales) as an operand of the NVFP4 GEMM kind (``mx_mbs_gemm_scales``):
    same codes, UE4M3 16-element scales S_M X / s_T in the tcgen05 chunk
    layout and the power-of-two tensor scale s_T."""
    if not q.cfg.macro_block or q.macro is None:
        raise ValueError("not an MBS-quantized tensor")
    dev = q.codes.device
    sf16 = torch.empty(max(q.rows * q.cols // 16, 16), dtype=torch.uint8, device=dev)
    ts = torch.empty(1, dtype=torch.float32, device=dev)
    ws = _ws(256, dev)
    rc = mx_mbs_gemm_scales(q.cfg, _p(q.scales), _p(q.macro), q.rows, q.cols, _p(sf16), _p(ts), _p(ws),
                            ws.numel(), _stream(stream))
    _check("mx_mbs_gemm_scales", rc)
    cfg = Config(block=16, scale_fmt=SCALE_UE4M3, rule=RULE_NEAREST, tensor_scale=TS_GIVEN, sf_layout=1)
    return Quantized(cfg, q.rows, q.cols, q.codes, sf16[: q.rows * q.cols // 16], ts, None, None, None)


def gemm_qsnr(A: torch.Tensor, B: torch.Tensor, qa: Quantized, qb: Quantized,
              stream=None) -> torch.Tensor:
    """QSNR(AB) of Eq. (2) with A [M x K], B [N x K] bf16 (``mx_gemm_qsnr``):
    float64[3] = [sum C_ref^2, sum (C_ref - C_q)^2, dB] on the device."""
    _cuda2d(A, "A")
    _cuda2d(B, "B")
    M, K = A.shape
    N = B.shape[0]
    st = torch.empty(3, dtype=torch.float64, device=A.device)
    nbytes = lib().mx_gemm_workspace_bytes(M, N, K)
    ws = _ws(nbytes, A.device)
    rc = mx_gemm_qsnr(qa.cfg, qb.cfg, _p(A), _p(B), M, N, K, _p(qa.codes), _p(qa.scales),
                      _p(qb.codes), _p(qb.scales), _p(qa.tensor_scale), _p(qb.tensor_scale),
                      _p(st), _p(ws), ws.numel(), _stream(stream))
    _check("mx_gemm_qsnr", rc)
    return st
