"""Row bands of one tensor on the GPU, the way the ranks of a row-partitioned
tensor see them, emulated on one device with no collective: the bands'
amax words are combined by a max (what the cross-rank reduction does), each
band is quantized with the combined amax (TS_AMAX), and the bands' sums are
added and re-finalised.  Codes, scales, tensor scale and dequantized values
must be exactly the whole tensor's; the statistics equal up to the order of
the binary64 additions.
"""
import numpy as np
import pytest
import torch

from microscaling_block_quantization_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mx():
    from microscaling_block_quantization_b200 import build
    build.build()
    import microscaling_block_quantization_b200 as m
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return m


def _cases(mx):
    nv = dict(block=16, scale_fmt=mx.SCALE_UE4M3, rule=mx.RULE_NEAREST, tensor_scale=mx.TS_COMPUTE)
    return {
        "nvfp4_row": (mx.Config(**nv), 1024, 2048, 3),
        "nvfp4_row_had16": (mx.Config(hadamard=16, **nv), 512, 1024, 2),
        "nvfp4_gemm_layout": (mx.Config(sf_layout=1, **nv), 1024, 1024, 2),
        "ue5m3_b8_fp32": (mx.Config(block=8, scale_fmt=mx.SCALE_UE5M3, rule=mx.RULE_NEAREST,
                                    tensor_scale=mx.TS_COMPUTE), 512, 512, 2),
        "mxfp4_col": (mx.Config(axis=mx.AXIS_COL), 1024, 512, 3),
        "mxfp4_2d": (mx.Config(axis=mx.AXIS_2D), 1024, 512, 4),
    }


@pytest.mark.parametrize("case", ["nvfp4_row", "nvfp4_row_had16", "nvfp4_gemm_layout", "ue5m3_b8_fp32",
                                  "mxfp4_col", "mxfp4_2d"])
def test_row_bands_equal_the_whole_tensor(mx, case):
    from microscaling_block_quantization_b200 import parallel
    cfg, rows, cols, world = _cases(mx)[case]
    x = inputs.laplace_outlier_cols(rows, cols, seed=4, n_outlier_cols=8)
    x[rows // 2:] *= 4                               # bands with different amax
    if case.endswith("fp32"):
        x = x.float()
    x = x.cuda()
    rotated = bool(cfg.hadamard)
    whole = mx.quantize(x, cfg, rotated=rotated)
    bands = [parallel.row_band(rows, world, r, parallel.row_align(cfg)) for r in range(world)]
    c = cfg
    ws = [mx.new_workspace(cfg, rows, cols, x.device) for _ in bands]
    if cfg.tensor_scale == mx.TS_COMPUTE:
        import dataclasses
        c = dataclasses.replace(cfg, tensor_scale=mx.TS_AMAX)
        for (r0, r1), w in zip(bands, ws):
            mx.tensor_amax(x[r0:r1], c, w)
        words = torch.stack([w[:4].view(torch.int32) for w in ws])
        top = words.max(dim=0).values
        for w in ws:
            w[:4].view(torch.int32).copy_(top)
    qs = [mx.quantize(x[r0:r1], c, workspace=w, rotated=rotated) for (r0, r1), w in zip(bands, ws)]
    torch.cuda.synchronize()
    assert mx.mx_device_status() == 0
    for w in ws:                                     # the quantizer cleared the words
        assert int(w[:256].count_nonzero()) == 0
    codes = torch.cat([q.codes.view(r1 - r0, -1) for q, (r0, r1) in zip(qs, bands)]).flatten()
    assert torch.equal(codes, whole.codes)
    # (chunk layout too: bands of whole 128-row groups hold whole chunks)
    assert torch.equal(torch.cat([q.scales for q in qs]), whole.scales)
    for q in qs:
        assert torch.equal(q.tensor_scale, whole.tensor_scale)
    if rotated:
        assert torch.equal(torch.cat([q.rotated for q in qs]), whole.rotated)
    xh = torch.cat([mx.dequantize(q, torch.float32) for q in qs])
    assert torch.equal(xh.view(torch.int32), mx.dequantize(whole, torch.float32).view(torch.int32))
    st = qs[0].stats.clone()
    idx = torch.tensor(parallel.SUM_ENTRIES, device=st.device)
    st.index_copy_(0, idx, sum(q.stats.index_select(0, idx) for q in qs))
    mx.stats_finalize(st)
    got, want = st.cpu().numpy(), whole.stats.cpu().numpy()
    for i in (0, 1, 2, 5, 6, 8):
        assert got[i] == pytest.approx(want[i], rel=1e-9, abs=1e-300)
    assert abs(got[7] - want[7]) <= 1e-9
    for i in (3, 4, 9, 10):
        assert got[i] == want[i]


def test_tensor_amax_needs_the_amax_mode(mx):
    x = torch.ones(128, 256, dtype=torch.bfloat16, device="cuda")
    w = mx.new_workspace(mx.NVFP4, 128, 256, x.device)
    with pytest.raises(mx.MXError) as e:
        mx.tensor_amax(x, mx.NVFP4, w)
    assert e.value.code == -1
