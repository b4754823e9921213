"""CPU oracle for microscaling block quantization -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product path (the CUDA library and its Python binding) never does, and this
package never imports the product path.

All arithmetic lives in ``mx_oracle.c`` (plain scalar C, see the header there
for the page citations and the readings taken).  This module only marshals
numpy arrays through ctypes.
"""
from __future__ import annotations

import ctypes as C
import dataclasses

import numpy as np

from . import build as _build

# enumeration values (the library's interface convention)
E2M1, E3M0, E2M3, E3M2, INT4 = 0, 1, 2, 3, 4
E8M0, UE4M3, UE5M3 = 0, 1, 2
FLOOR, CEIL, OAS, NEAREST, MSE = 0, 1, 2, 3, 4
RTNE, RCEIL, SR = 0, 1, 2
ROW, COL, TWO_D = 0, 1, 2
BF16, FP32 = 0, 1
TS_NONE, TS_COMPUTE, TS_GIVEN = 0, 1, 2


class _Cfg(C.Structure):
    _fields_ = [("elem", C.c_int32), ("scale_fmt", C.c_int32), ("rule", C.c_int32),
                ("oas_tau", C.c_float), ("block", C.c_int32), ("axis", C.c_int32),
                ("round_mode", C.c_int32), ("asymmetric", C.c_int32),
                ("tensor_scale", C.c_int32), ("macro_block", C.c_int32),
                ("hadamard", C.c_int32), ("reserved", C.c_int32), ("seed", C.c_uint64)]


@dataclasses.dataclass
class Cfg:
    elem: int = E2M1
    scale_fmt: int = E8M0
    rule: int = FLOOR
    oas_tau: float = 7.0
    block: int = 32
    axis: int = ROW
    round_mode: int = RTNE
    asymmetric: int = 0
    tensor_scale: int = TS_NONE
    macro_block: int = 0
    hadamard: int = 0
    seed: int = 0

    def c(self) -> _Cfg:
        return _Cfg(self.elem, self.scale_fmt, self.rule, self.oas_tau, self.block, self.axis,
                    self.round_mode, self.asymmetric, self.tensor_scale, self.macro_block,
                    self.hadamard, 0, self.seed)


_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        P = C.c_void_p
        i64 = C.c_int64
        L.orc_quantize.argtypes = [C.POINTER(_Cfg), P, C.c_int, i64, i64, P, P, P, P, P, P]
        L.orc_quantize.restype = C.c_int
        L.orc_dequantize.argtypes = [C.POINTER(_Cfg), P, P, P, P, P, i64, i64, C.c_int, P]
        L.orc_dequantize.restype = C.c_int
        L.orc_pack.argtypes = [C.c_int, P, i64, i64, P]
        L.orc_unpack.argtypes = [C.c_int, P, i64, i64, P]
        L.orc_pack_tc.argtypes = [C.c_int, P, i64, i64, P]
        L.orc_unpack_tc.argtypes = [C.c_int, P, i64, i64, P]
        L.orc_packed_bytes.argtypes = [C.c_int, i64, i64]
        L.orc_packed_bytes.restype = i64
        L.orc_stats.argtypes = [P, P, i64, i64, C.c_int, C.c_int, P, P]
        L.orc_finalize_stats.argtypes = [P]
        L.orc_philox4x32_10.argtypes = [P, P, P]
        L.orc_encode_elem.argtypes = [C.c_int, C.c_int, C.c_int, C.c_float, C.c_uint32]
        L.orc_encode_elem.restype = C.c_uint8
        L.orc_decode_elem.argtypes = [C.c_int, C.c_int, C.c_uint8]
        L.orc_decode_elem.restype = C.c_float
        L.orc_scale_decode.argtypes = [C.c_int, C.c_uint8]
        L.orc_scale_decode.restype = C.c_float
        L.orc_scale_encode_nearest.argtypes = [C.c_int, C.c_float]
        L.orc_scale_encode_nearest.restype = C.c_uint8
        L.orc_fwht.argtypes = [C.c_int, P, C.c_int]
        L.orc_packed_tc_bytes.argtypes = [C.c_int, i64, i64]
        L.orc_packed_tc_bytes.restype = i64
        L.orc_tensor_scale.argtypes = [C.c_int, C.c_int, P, i64]
        L.orc_tensor_scale.restype = C.c_float
        L.orc_mse_grid_trace.argtypes = [C.c_int, C.c_int, P, C.c_int, i64, i64, C.c_int, P, P]
        L.orc_mse_grid_trace.restype = C.c_float
        L.orc_gemm.argtypes = [P, P, i64, i64, i64, P]
        L.orc_gemm_qsnr.argtypes = [P, P, P, P, i64, i64, i64, P]
        L.orc_bf16_to_f32.argtypes = [C.c_uint16]
        L.orc_bf16_to_f32.restype = C.c_float
        L.orc_f32_to_bf16.argtypes = [C.c_float]
        L.orc_f32_to_bf16.restype = C.c_uint16
        _lib = L
    return _lib


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def as_input(x) -> tuple[np.ndarray, int]:
    """numpy/torch input -> (contiguous array, dtype code).  bf16 tensors are
    passed as their raw 16-bit patterns."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), BF16
            if x.dtype == torch.float32:
                return x.numpy(), FP32
            raise TypeError(f"unsupported dtype {x.dtype}")
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return x, BF16
    if x.dtype == np.float32:
        return x, FP32
    raise TypeError(f"unsupported dtype {x.dtype}")


def n_blocks(cfg: Cfg, rows: int, cols: int) -> int:
    B = cfg.block
    if cfg.axis == ROW:
        return rows * (cols // B)
    if cfg.axis == COL:
        return (rows // B) * cols
    return (rows // B) * (cols // B)


def n_macro(cfg: Cfg, rows: int, cols: int) -> int:
    if not cfg.macro_block:
        return 0
    return (rows // 128) * cols if cfg.axis == COL else rows * (cols // 128)


def quantize(cfg: Cfg, x, tensor_scale: float | None = None) -> dict:
    """Run the oracle quantizer.  Returns codes (one per element), packed
    bytes, scale codes, tensor scale, macro-scale codes, bf16 offsets and the
    reference tensor y (the input, rotated when cfg.hadamard is set)."""
    arr, dt = as_input(x)
    rows, cols = arr.shape
    codes = np.zeros((rows, cols), np.uint8)
    scales = np.zeros(n_blocks(cfg, rows, cols), np.uint8)
    ts = np.array([tensor_scale if tensor_scale is not None else 1.0], np.float32)
    nm = n_macro(cfg, rows, cols)
    macro = np.zeros(max(nm, 1), np.uint8)
    offsets = np.zeros(n_blocks(cfg, rows, cols), np.uint16)
    y = np.zeros((rows, cols), np.float32)
    c = cfg.c()
    rc = lib().orc_quantize(C.byref(c), _ptr(arr), dt, rows, cols, _ptr(codes), _ptr(scales),
                            _ptr(ts), _ptr(macro) if nm else None,
                            _ptr(offsets), _ptr(y))
    if rc != 0:
        raise RuntimeError("oracle quantize failed")
    packed = pack(cfg.elem, codes)
    return dict(codes=codes, packed=packed, scales=scales, tensor_scale=float(ts[0]),
                macro=macro[:nm], offsets=offsets, y=y)


def pack(elem: int, codes: np.ndarray) -> np.ndarray:
    rows, cols = codes.shape
    nbytes = lib().orc_packed_bytes(elem, rows, cols)
    out = np.zeros(nbytes, np.uint8)
    lib().orc_pack(elem, _ptr(np.ascontiguousarray(codes)), rows, cols, _ptr(out))
    return out.reshape(rows, -1)


def pack_tc(elem: int, codes: np.ndarray) -> np.ndarray:
    """Codes in the tensor-core operand form (FP6: every 16 codes in 12
    bytes, 6 bits each; FP4 as `pack`)."""
    rows, cols = codes.shape
    nbytes = lib().orc_packed_tc_bytes(elem, rows, cols)
    out = np.zeros(nbytes, np.uint8)
    lib().orc_pack_tc(elem, _ptr(np.ascontiguousarray(codes)), rows, cols, _ptr(out))
    return out.reshape(rows, -1)


def unpack_tc(elem: int, packed: np.ndarray, rows: int, cols: int) -> np.ndarray:
    out = np.zeros((rows, cols), np.uint8)
    lib().orc_unpack_tc(elem, _ptr(np.ascontiguousarray(packed)), rows, cols, _ptr(out))
    return out


def unpack(elem: int, packed: np.ndarray, rows: int, cols: int) -> np.ndarray:
    out = np.zeros((rows, cols), np.uint8)
    lib().orc_unpack(elem, _ptr(np.ascontiguousarray(packed)), rows, cols, _ptr(out))
    return out


def dequantize(cfg: Cfg, packed, scales, tensor_scale, macro, offsets, rows: int, cols: int,
               unrotate: bool = False) -> np.ndarray:
    out = np.zeros((rows, cols), np.float32)
    ts = np.array([1.0 if tensor_scale is None else tensor_scale], np.float32)
    macro = None if macro is None or len(macro) == 0 else np.ascontiguousarray(macro, np.uint8)
    offsets = None if offsets is None else np.ascontiguousarray(offsets, np.uint16)
    c = cfg.c()
    rc = lib().orc_dequantize(C.byref(c), _ptr(np.ascontiguousarray(packed, np.uint8)),
                              _ptr(np.ascontiguousarray(scales, np.uint8)), _ptr(ts),
                              _ptr(macro), _ptr(offsets), rows, cols, int(unrotate), _ptr(out))
    if rc != 0:
        raise RuntimeError("oracle dequantize failed")
    return out


def stats(ref: np.ndarray, xhat: np.ndarray, block: int = 0, axis: int = ROW):
    """binary64 fidelity statistics (see mx_oracle.c for the layout) and, when
    block > 0, the per-block MSE."""
    ref = np.ascontiguousarray(ref, np.float32)
    xhat = np.ascontiguousarray(xhat, np.float32)
    rows, cols = ref.shape
    st = np.zeros(16, np.float64)
    pb = None
    if block:
        pb = np.zeros(n_blocks(Cfg(block=block, axis=axis), rows, cols), np.float32)
    lib().orc_stats(_ptr(ref), _ptr(xhat), rows, cols, block, axis, _ptr(st), _ptr(pb))
    return st, pb


def finalize_stats(st: np.ndarray) -> np.ndarray:
    st = np.ascontiguousarray(st, np.float64).copy()
    lib().orc_finalize_stats(_ptr(st))
    return st


def philox(ctr, key) -> list[int]:
    c = np.array(ctr, np.uint32)
    k = np.array(key, np.uint32)
    o = np.zeros(4, np.uint32)
    lib().orc_philox4x32_10(_ptr(c), _ptr(k), _ptr(o))
    return [int(v) for v in o]


def encode_elem(elem: int, v: float, mode: int = RTNE, u: int = 0, asym: int = 0) -> int:
    return int(lib().orc_encode_elem(elem, asym, mode, v, u))


def decode_elem(elem: int, code: int, asym: int = 0) -> float:
    return float(lib().orc_decode_elem(elem, asym, code))


def scale_decode(fmt: int, code: int) -> float:
    return float(lib().orc_scale_decode(fmt, code))


def scale_encode_nearest(fmt: int, x: float) -> int:
    return int(lib().orc_scale_encode_nearest(fmt, x))


def mse_grid_trace(scale_fmt: int, block: int, x, rounds: int = 4):
    """The alternating global / group scale optimisation of the MSE rule with
    a nearest scale format (row blocks): final s_T, the s_T before each group
    step and the squared error after it (rounds + 1 entries each)."""
    arr, dt = as_input(x)
    rows, cols = arr.shape
    st = np.zeros(rounds + 1, np.float32)
    se = np.zeros(rounds + 1, np.float64)
    s = lib().orc_mse_grid_trace(scale_fmt, block, _ptr(arr), dt, rows, cols, rounds, _ptr(st), _ptr(se))
    return float(s), st, se


def fwht(v: np.ndarray, normalise: bool = True) -> np.ndarray:
    v = np.array(v, np.float32).copy()
    lib().orc_fwht(len(v), _ptr(v), int(normalise))
    return v


def tensor_scale(elem: int, fmt: int, y: np.ndarray) -> float:
    y = np.ascontiguousarray(y, np.float32)
    return float(lib().orc_tensor_scale(elem, fmt, _ptr(y), y.size))


def gemm(A: np.ndarray, B: np.ndarray) -> np.ndarray:
    """C = A B^T in binary64 by the triple loop (small shapes only)."""
    A = np.ascontiguousarray(A, np.float32)
    B = np.ascontiguousarray(B, np.float32)
    M, K = A.shape
    N = B.shape[0]
    out = np.zeros((M, N), np.float64)
    lib().orc_gemm(_ptr(A), _ptr(B), M, N, K, _ptr(out))
    return out


def gemm_qsnr(A, B, Ah, Bh) -> np.ndarray:
    """[sum C_ref^2, sum (C_ref - C_q)^2, QSNR(AB) dB] by the triple loop."""
    A = np.ascontiguousarray(A, np.float32)
    B = np.ascontiguousarray(B, np.float32)
    Ah = np.ascontiguousarray(Ah, np.float32)
    Bh = np.ascontiguousarray(Bh, np.float32)
    M, K = A.shape
    N = B.shape[0]
    out = np.zeros(3, np.float64)
    lib().orc_gemm_qsnr(_ptr(A), _ptr(B), _ptr(Ah), _ptr(Bh), M, N, K, _ptr(out))
    return out


def gemm_qsnr_blas(A, B, Ah, Bh, row_chunk: int = 1024) -> np.ndarray:
    """Same quantities for large shapes with a binary64 BLAS product (a
    library routine) over the dequantized operands, in row chunks."""
    A = np.asarray(A, np.float64)
    B = np.asarray(B, np.float64)
    Ah = np.asarray(Ah, np.float64)
    Bh = np.asarray(Bh, np.float64)
    sr = 0.0
    se = 0.0
    for m0 in range(0, A.shape[0], row_chunk):
        cr = A[m0:m0 + row_chunk] @ B.T
        cq = Ah[m0:m0 + row_chunk] @ Bh.T
        sr += float(np.sum(cr * cr))
        se += float(np.sum((cr - cq) ** 2))
    q = float("nan") if sr == 0 else (float("inf") if se == 0 else 10.0 * np.log10(sr / se))
    return np.array([sr, se, q])


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (a pure bit shift)."""
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def input_f32(x) -> np.ndarray:
    arr, dt = as_input(x)
    return bf16_bits_to_f32(arr) if dt == BF16 else arr.astype(np.float32)


__all__ = [n for n in dir() if not n.startswith("_")]
