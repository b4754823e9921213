"""The row-sharded path end to end on the GPU, with two processes.

Two ranks (spawned processes, gloo on CUDA tensors) share the one GPU and
each runs ``parallel.quantize_sharded`` / ``parallel.gemm_qsnr_sharded`` on
its band of rows; their kernels never wait on each other (the collectives are
gloo's, on the host).  Every band's codes and scales, and the tensor scale,
must equal the whole-tensor call's bit for bit; the reduced statistics and
QSNR(AB) sums equal the whole tensor's up to the order of binary64 additions.
Sources: "Unveiling the Potential of Quantization with MXFP4" (Sec.2 one scale
per block; Sec.3 Eq. (1) and (2)); "Is Finer Better?" (the FP32 tensor scale).
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

from microscaling_block_quantization_b200 import inputs

pytestmark = pytest.mark.gpu

CASES = ("nvfp4_row", "mxfp4_2d", "nvfp4_had16_row", "mxfp4_col_mbs")


def _cfg(mx, case):
    return {"nvfp4_row": mx.Config(block=16, scale_fmt=mx.SCALE_UE4M3, rule=mx.RULE_NEAREST,
                                   tensor_scale=mx.TS_COMPUTE),
            "mxfp4_2d": mx.Config(axis=mx.AXIS_2D),
            "nvfp4_had16_row": mx.Config(block=16, scale_fmt=mx.SCALE_UE4M3, rule=mx.RULE_NEAREST,
                                         tensor_scale=mx.TS_COMPUTE, hadamard=16),
            "mxfp4_col_mbs": mx.Config(axis=mx.AXIS_COL, macro_block=128)}[case]


def _input(rows=512, cols=1024):
    x = inputs.laplace_outlier_cols(rows, cols, seed=4, n_outlier_cols=4)
    x[rows // 2:] *= 4                    # the bands' amaxes differ
    return x


def _layer():
    a = inputs.laplace_outlier_cols(512, 768, seed=6, n_outlier_cols=2)
    w = inputs.normal(256, 768, sigma=0.02, seed=7)
    return a, w


def _rank(rank, world, port, out):
    import torch.distributed as dist
    import microscaling_block_quantization_b200 as mx
    from microscaling_block_quantization_b200 import parallel
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    res = {}
    try:
        x = _input().cuda()
        for case in CASES:
            cfg = _cfg(mx, case)
            r0, r1 = parallel.row_band(x.shape[0], world, rank, parallel.row_align(cfg))
            q = parallel.quantize_sharded(x[r0:r1].contiguous(), cfg)
            torch.cuda.synchronize()
            res[case] = (r0, r1, q.codes.cpu().numpy(), q.scales.cpu().numpy(), q.tensor_scale.cpu().numpy(),
                         None if q.macro is None else q.macro.cpu().numpy(), q.stats.cpu().numpy())
        a, w = (t.cuda() for t in _layer())
        g = mx.Config(sf_layout=1)
        r0, r1 = parallel.row_band(a.shape[0], world, rank, parallel.row_align(g))
        qa = mx.quantize(a[r0:r1].contiguous(), g, stats=False)
        qw = mx.quantize(w, g, stats=False)
        st = parallel.gemm_qsnr_sharded(a[r0:r1].contiguous(), w, qa, qw)
        torch.cuda.synchronize()
        res["qsnr_ab"] = st.cpu().numpy()
        res["status"] = mx.mx_device_status()
        out.put((rank, res))
    except Exception as e:                       # reported to the parent, which fails the test
        out.put((rank, repr(e)))
        raise
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture(scope="module")
def mx():
    from microscaling_block_quantization_b200 import build
    build.build()
    import microscaling_block_quantization_b200 as m
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return m


def test_two_ranks_on_one_gpu_equal_the_whole_tensor(mx):
    import torch.multiprocessing as tmp
    world = 2
    ctx = tmp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(out.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=120)
    for r in range(world):
        assert isinstance(got[r], dict), got[r]
        assert got[r]["status"] == 0
    assert all(p.exitcode == 0 for p in procs)

    x = _input().cuda()
    for case in CASES:
        cfg = _cfg(mx, case)
        whole = mx.quantize(x, cfg)
        torch.cuda.synchronize()
        wc = whole.codes.cpu().numpy().reshape(x.shape[0], -1)
        ws = whole.scales.cpu().numpy()
        wst = whole.stats.cpu().numpy()
        parts_codes, parts_scales = [], []
        for r in range(world):
            r0, r1, codes, scales, ts, macro, st = got[r][case]
            parts_codes.append(codes.reshape(r1 - r0, -1))
            parts_scales.append(scales)
            assert np.array_equal(ts, whole.tensor_scale.cpu().numpy()), case
            for i in (0, 1, 2, 5, 6, 7, 8):
                assert st[i] == pytest.approx(wst[i], rel=1e-9, abs=1e-300), (case, i)
            for i in (3, 4, 9, 10):
                assert st[i] == wst[i], (case, i)
        assert np.array_equal(np.concatenate(parts_codes), wc), case
        # scales (row, column and 2D layouts alike) and macro scales are laid
        # out by rows of blocks: the bands' arrays concatenate to the whole's
        assert np.array_equal(np.concatenate(parts_scales), ws), case
        if cfg.macro_block:
            wm = whole.macro.cpu().numpy()
            assert np.array_equal(np.concatenate([got[r][case][5] for r in range(world)]), wm), case

    a, w = (t.cuda() for t in _layer())
    g = mx.Config(sf_layout=1)
    st = mx.gemm_qsnr(a, w, mx.quantize(a, g, stats=False), mx.quantize(w, g, stats=False)).cpu().numpy()
    for r in range(world):
        q = got[r]["qsnr_ab"]
        assert q[0] == pytest.approx(st[0], rel=1e-9) and q[1] == pytest.approx(st[1], rel=1e-9)
        assert q[2] == pytest.approx(st[2], abs=1e-9)
