"""Row-partitioned quantization of one tensor over several GPUs.

One process per GPU (``torch.distributed``; NCCL on GPUs, gloo for the CPU
tests).  Blocks are independent ("Unveiling the Potential of Quantization
with MXFP4", Sec.2: one shared scale per block), so each rank quantizes a band
of whole rows on its own GPU and keeps its own codes and scales.  Two results
are properties of the whole tensor, and each costs one small exchange:

* a computed per-tensor scale ("Is Finer Better? The Limits of Microscaling
  Formats in LLMs", per-tensor FP32 scale; NVFP4 in "Bridging the Gap Between
  Promise and Performance for Microscaling FP4 Quantization", Sec.1):
  s_T = amax_T / (max_elem * max_scale) needs the amax of every band.  Each
  rank folds its band's amax into its workspace's amax word
  (``mx_tensor_amax``), the ranks take the max of the words, and the quantizer
  derives s_T from the word (``TS_AMAX``).  Float bits of non-negative values
  order like the 32-bit integers, so the max of the words is the word of the
  max.
* the fidelity statistics (Sec.3 Eq. (1) of the first page): the sums and the
  element count add over bands; the derived MSE / R-MSE / QSNR / bias / flush
  share are recomputed on the device from the summed buffer
  (``mx_stats_finalize``).

Bands follow the block geometry along rows so that no block straddles ranks:
column blocks of B rows, 2D blocks of 32 rows, 128 rows for the tcgen05 scale
layout and for column-axis macro blocks.

QSNR(AB) of a product split by the rows of A (Sec.3 Eq. (2) of the first
page): each rank holds a band of A's rows (bf16 and quantized) and the whole
B (bf16 and quantized); both sums of Eq. (2) add over the bands, so one sum
reduction of two numbers gives the whole product's QSNR.
"""
from __future__ import annotations

import dataclasses
import math

import torch
import torch.distributed as dist

from . import (AXIS_2D, AXIS_COL, TS_AMAX, TS_COMPUTE, Config, Quantized, gemm_qsnr, gemm_qsnr_finalize,
               new_workspace, quantize, stats_finalize, tensor_amax)

# entries of a stats buffer that add over bands: the five sums and the count
SUM_ENTRIES = (0, 1, 2, 3, 4, 10)


def row_align(cfg: Config) -> int:
    """Row granularity of a band: a multiple of every block extent along rows."""
    a = 1
    if cfg.axis == AXIS_COL:
        a = cfg.block
        if cfg.macro_block:
            a = math.lcm(a, 128)
        if cfg.hadamard:
            a = math.lcm(a, cfg.hadamard)
    elif cfg.axis == AXIS_2D:
        a = 32
    if cfg.sf_layout == 1:
        a = math.lcm(a, 128)
    return a


def row_band(rows: int, world: int, rank: int, align: int) -> tuple[int, int]:
    """Rows [r0, r1) of `rank`: the rows in units of `align`, split as evenly
    as the units allow (the first ranks take one unit more).  `rows` must be a
    multiple of `align`; a rank may get an empty band."""
    if rows % align:
        raise ValueError(f"rows ({rows}) must be a multiple of the band unit ({align})")
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    units = rows // align
    base, extra = divmod(units, world)
    u0 = rank * base + min(rank, extra)
    u1 = u0 + base + (1 if rank < extra else 0)
    return u0 * align, u1 * align


def reduce_amax_word(workspace: torch.Tensor, group=None) -> None:
    """Max of the ranks' amax words (byte 0 of each workspace), in place."""
    word = workspace[:4].view(torch.int32)
    dist.all_reduce(word, op=dist.ReduceOp.MAX, group=group)


def reduce_stats(stats: torch.Tensor, group=None) -> None:
    """Sum of the ranks' sums and counts, in place (the derived entries are
    left for ``stats_finalize``)."""
    idx = torch.tensor(SUM_ENTRIES, device=stats.device)
    part = stats.index_select(0, idx)
    dist.all_reduce(part, op=dist.ReduceOp.SUM, group=group)
    stats.index_copy_(0, idx, part)


def quantize_sharded(x_band: torch.Tensor, cfg: Config, *, stats: bool = True, group=None,
                     rotated: bool = False, workspace: torch.Tensor | None = None,
                     stream=None) -> Quantized:
    """Quantize this rank's band of rows of a row-partitioned tensor.  Codes,
    scales and offsets are the band's rows of the whole tensor's; the tensor
    scale and the statistics are the whole tensor's.  Every rank of `group`
    must call it with the same `cfg` and `stats` (the collectives run in the
    same order everywhere)."""
    rows, cols = x_band.shape
    ws = workspace if workspace is not None else new_workspace(cfg, max(rows, 1), cols, x_band.device)
    c = cfg
    if cfg.tensor_scale == TS_COMPUTE:
        c = dataclasses.replace(cfg, tensor_scale=TS_AMAX)
        tensor_amax(x_band, c, ws, stream=stream)
        reduce_amax_word(ws, group)
    q = quantize(x_band, c, stats=stats, rotated=rotated, workspace=ws, stream=stream)
    if stats:
        reduce_stats(q.stats, group)
        stats_finalize(q.stats, stream=stream)
    return q


def reduce_qsnr_sums(stats: torch.Tensor, group=None) -> None:
    """Sum of the ranks' [sum C_ref^2, sum (C_ref - C_q)^2], in place (the dB
    entry is left for ``gemm_qsnr_finalize``)."""
    dist.all_reduce(stats[:2], op=dist.ReduceOp.SUM, group=group)


def gemm_qsnr_sharded(A_band: torch.Tensor, B: torch.Tensor, qa_band: Quantized, qb: Quantized, *,
                      group=None, stream=None) -> torch.Tensor:
    """QSNR(AB) of a product whose A is split by rows over the ranks: this
    rank's band of A (bf16 rows and their quantized form, rows in units of
    128) against the replicated B; returns the whole product's float64[3]
    [sum C_ref^2, sum (C_ref - C_q)^2, dB].  An empty band contributes zeros.
    Every rank of `group` must call it (one collective)."""
    if A_band.shape[0] == 0:
        st = torch.zeros(3, dtype=torch.float64, device=B.device)
    else:
        st = gemm_qsnr(A_band, B, qa_band, qb, stream=stream)
    reduce_qsnr_sums(st, group)
    gemm_qsnr_finalize(st, stream=stream)
    return st
