"""Row-partitioned quantization over ranks, host side, on CPU.

Two gloo ranks each take a band of rows of one tensor.  The per-rank work is
the oracle's (no GPU here); what is under test is the partition and the two
exchanges of ``parallel``: the max of the amax words and the sum of the
statistics.  With them the bands' codes, scales and tensor scale are exactly
the whole tensor's, and the combined statistics are the whole tensor's.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from microscaling_block_quantization_b200 import inputs, parallel
import microscaling_block_quantization_b200 as mx
import oracle as orc

# (library config, oracle config fields, rows, cols)
CASES = {
    "nvfp4_row": (dict(block=16, scale_fmt=mx.SCALE_UE4M3, rule=mx.RULE_NEAREST, tensor_scale=mx.TS_COMPUTE),
                  dict(block=16, scale_fmt=orc.UE4M3, rule=orc.NEAREST), 96, 256),
    "ue5m3_row_b8": (dict(block=8, scale_fmt=mx.SCALE_UE5M3, rule=mx.RULE_NEAREST, tensor_scale=mx.TS_COMPUTE),
                     dict(block=8, scale_fmt=orc.UE5M3, rule=orc.NEAREST), 64, 128),
    "mxfp4_col": (dict(axis=mx.AXIS_COL), dict(axis=orc.COL), 96, 128),
    "mxfp4_2d": (dict(axis=mx.AXIS_2D), dict(axis=orc.TWO_D), 160, 96),
}


def test_row_band_partition():
    for rows, align in ((96, 32), (256, 128), (4096, 16), (32, 32), (0, 32)):
        for world in (1, 2, 3, 4, 8):
            bands = [parallel.row_band(rows, world, r, align) for r in range(world)]
            assert bands[0][0] == 0 and bands[-1][1] == rows
            for (a0, a1), (b0, b1) in zip(bands, bands[1:]):
                assert a1 == b0
            sizes = [b - a for a, b in bands]
            assert all(a % align == 0 and s % align == 0 for (a, _), s in zip(bands, sizes))
            assert max(sizes) - min(sizes) <= align
    with pytest.raises(ValueError):
        parallel.row_band(100, 2, 0, 32)


def test_row_align_follows_block_geometry():
    assert parallel.row_align(mx.Config()) == 1
    assert parallel.row_align(mx.Config(axis=mx.AXIS_COL, block=16)) == 16
    assert parallel.row_align(mx.Config(axis=mx.AXIS_COL, block=32, macro_block=128)) == 128
    assert parallel.row_align(mx.Config(axis=mx.AXIS_2D)) == 32
    assert parallel.row_align(mx.Config(sf_layout=1)) == 128


def _input(rows, cols):
    # the lower half of the rows 4x larger, so the two bands' amax differ
    x = inputs.laplace_outlier_cols(rows, cols, seed=4, n_outlier_cols=4)
    x[rows // 2:] *= 4
    return x


def _whole(case):
    cfg_kw, ocfg, rows, cols = CASES[case]
    x = _input(rows, cols)
    ts_mode = orc.TS_COMPUTE if cfg_kw.get("tensor_scale") else orc.TS_NONE
    oc = orc.Cfg(tensor_scale=ts_mode, **ocfg)
    return x, oc, orc.quantize(oc, x)


def _rank(rank, world, port, case, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        cfg_kw, ocfg, rows, cols = CASES[case]
        cfg = mx.Config(**cfg_kw)
        x = _input(rows, cols)
        r0, r1 = parallel.row_band(rows, world, rank, parallel.row_align(cfg))
        band = x[r0:r1]
        sT = None
        if cfg.tensor_scale == mx.TS_COMPUTE:
            # this rank's amax word, as the device pre-pass leaves it
            amax = np.float32(np.nanmax(np.abs(orc.input_f32(band)))) if r1 > r0 else np.float32(0)
            ws = torch.zeros(256, dtype=torch.uint8)
            ws[:4].view(torch.int32)[0] = int(amax.view(np.int32))
            parallel.reduce_amax_word(ws)
            amax_t = np.array([ws[:4].view(torch.float32).item()], np.float32)
            sT = orc.tensor_scale(ocfg["elem"] if "elem" in ocfg else orc.E2M1, ocfg["scale_fmt"], amax_t)
        oc = orc.Cfg(tensor_scale=orc.TS_GIVEN if sT is not None else orc.TS_NONE, **ocfg)
        r = orc.quantize(oc, band, tensor_scale=sT)
        xh = orc.dequantize(oc, r["packed"], r["scales"], r["tensor_scale"], None, None, r1 - r0, cols)
        st, _ = orc.stats(r["y"], xh)
        t = torch.from_numpy(np.asarray(st, np.float64).copy())
        parallel.reduce_stats(t)
        out.put((rank, r0, r1, r["codes"], r["scales"], r["tensor_scale"], orc.finalize_stats(t.numpy())))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("case,world", [(c, 2) for c in sorted(CASES)] + [("nvfp4_row", 3), ("mxfp4_2d", 3)])
def test_rank_bands_equal_the_whole_tensor(case, world):
    """Two ranks, and three (96 rows: 32 each; 160 rows in 32-row units:
    uneven bands of 64 / 64 / 32)."""
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, case, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = [out.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x, oc, whole = _whole(case)
    rows, cols = x.shape
    unit = parallel.row_align(mx.Config(**CASES[case][0]))
    per_unit = len(whole["scales"]) * unit // rows          # scale bytes per band unit of rows
    xh = orc.dequantize(oc, whole["packed"], whole["scales"], whole["tensor_scale"], None, None, rows, cols)
    want_stats = orc.stats(whole["y"], xh)[0]
    for rank, r0, r1, codes, scales, ts, st in res:
        assert np.array_equal(codes, whole["codes"][r0:r1])
        assert np.array_equal(scales, whole["scales"][r0 // unit * per_unit: r1 // unit * per_unit])
        assert np.float32(ts) == np.float32(whole["tensor_scale"])
        for i in (0, 1, 2, 5, 6, 7, 8):
            assert st[i] == pytest.approx(want_stats[i], rel=1e-12, abs=1e-300)
        for i in (3, 4, 9, 10):
            assert st[i] == want_stats[i]


def _qsnr_rank(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        M, N, K = 384, 128, 256
        a = inputs.laplace_outlier_cols(M, K, seed=6, n_outlier_cols=2)
        w = inputs.normal(N, K, sigma=0.02, seed=7)
        r0, r1 = parallel.row_band(M, world, rank, parallel.row_align(mx.Config(sf_layout=1)))
        st = np.zeros(3)
        if r1 > r0:
            oc = orc.Cfg()
            ra, rw = orc.quantize(oc, a[r0:r1]), orc.quantize(oc, w)
            ah = orc.dequantize(oc, ra["packed"], ra["scales"], None, None, None, r1 - r0, K)
            wh = orc.dequantize(oc, rw["packed"], rw["scales"], None, None, None, N, K)
            st = orc.gemm_qsnr(orc.input_f32(a[r0:r1]), orc.input_f32(w), ah, wh)
        t = torch.from_numpy(np.asarray(st, np.float64).copy())
        parallel.reduce_qsnr_sums(t)
        out.put((rank, t.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_qsnr_ab_row_bands_add_up(world):
    """QSNR(AB) with A split by rows (bands of 128: with four ranks over 384
    rows one band is empty): the two sums of Eq. (2) reduced over the ranks
    are the whole product's."""
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_qsnr_rank, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = [out.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    M, N, K = 384, 128, 256
    a = inputs.laplace_outlier_cols(M, K, seed=6, n_outlier_cols=2)
    w = inputs.normal(N, K, sigma=0.02, seed=7)
    oc = orc.Cfg()
    ra, rw = orc.quantize(oc, a), orc.quantize(oc, w)
    ah = orc.dequantize(oc, ra["packed"], ra["scales"], None, None, None, M, K)
    wh = orc.dequantize(oc, rw["packed"], rw["scales"], None, None, None, N, K)
    whole = orc.gemm_qsnr(orc.input_f32(a), orc.input_f32(w), ah, wh)
    for _, st in res:
        assert st[0] == pytest.approx(whole[0], rel=1e-12)
        assert st[1] == pytest.approx(whole[1], rel=1e-12)
