"""Grouped quantization (``mx_quantize_group``): several tensors of one
configuration in shared launches, each with its own codes, scales, tensor
scale, macro scales and statistics.  Blocks, and tensors, are quantized on
their own ("Unveiling the Potential of Quantization with MXFP4", Sec.2), so
every tensor of a group must match the oracle exactly as a tensor quantized
alone does: codes, scales, macro scales, tensor scale and the dequantized
tensor bit for bit, statistics within 1e-4 ("Is Finer Better?" per-tensor
scale; Sec.3 Eq. (1) of the first page).
"""
import numpy as np
import pytest
import torch

from microscaling_block_quantization_b200 import inputs

from .test_gpu_quantize import run_case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mx():
    from microscaling_block_quantization_b200 import build
    build.build()
    import microscaling_block_quantization_b200 as m
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return m


def _cfgs(mx):
    return {
        "mxfp4": mx.MXFP4,
        "nvfp4": mx.NVFP4,
        "had32": mx.Config(hadamard=32),
        "nvfp4_had16": mx.Config(block=16, scale_fmt=1, rule=3, tensor_scale=1, hadamard=16),
        "mbs_oas": mx.Config(macro_block=128, rule=2, oas_tau=7.0),
        "mbs_b16": mx.Config(block=16, macro_block=128),
        "ue4m3_b64_ts": mx.Config(block=64, scale_fmt=1, rule=3, tensor_scale=1),
        "ue5m3_b256": mx.Config(block=256, scale_fmt=2, rule=3),
        "e8m0_b8": mx.Config(block=8),
        "ceil_sf_gemm": mx.Config(rule=1, sf_layout=1),       # scales in the tcgen05 chunk layout
        "col": mx.Config(axis=1),
        "col_b8": mx.Config(axis=1, block=8),
        "col_nvfp4": mx.Config(axis=1, block=16, scale_fmt=1, rule=3, tensor_scale=1),
        "2d": mx.Config(axis=2),
        # configurations outside the shared launch: one call per tensor
        "col_mbs": mx.Config(axis=1, macro_block=128),
        "int4_asym": mx.Config(elem=mx.INT4, asymmetric=1, rule=1),
        "nvfp4_mse": mx.Config(block=16, scale_fmt=1, rule=4, tensor_scale=1),
    }


def _tensors(name, dtype=torch.bfloat16):
    """Tensors of different shapes and scales (the tensor amaxes differ)."""
    if name == "ceil_sf_gemm":
        shapes = [(128, 512), (256, 256), (128, 1024)]
    elif name.startswith("col") or name == "2d":
        # column blocks need rows in multiples of the block (and of 128 with MBS),
        # 2D tiles multiples of 32
        shapes = [(128, 256), (32, 512), (256, 160), (96, 128)] if name != "col_mbs" else [(128, 256), (256, 512)]
    else:
        shapes = [(40, 768), (264, 512), (1, 256), (96, 1280)]
    out = []
    for i, (r, c) in enumerate(shapes):
        x = inputs.laplace_outlier_cols(r, c, seed=10 + i, n_outlier_cols=min(4, c // 64), dtype=dtype)
        out.append(x * (4.0 ** i))
    return out


@pytest.mark.parametrize("name", ["mxfp4", "nvfp4", "had32", "nvfp4_had16", "mbs_oas", "mbs_b16",
                                  "ue4m3_b64_ts", "ue5m3_b256", "e8m0_b8", "col", "col_b8", "col_nvfp4", "2d",
                                  "col_mbs", "int4_asym", "nvfp4_mse"])
def test_group_matches_oracle(mx, orc, name):
    cfg = _cfgs(mx)[name]
    xs = _tensors(name)
    qs = mx.quantize_group([x.cuda() for x in xs], cfg)
    torch.cuda.synchronize()
    for x, q in zip(xs, qs):
        run_case(mx, orc, x, cfg, want_rotated=False, q=q)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_group_of_six_with_an_empty_tensor(mx, orc, dtype):
    """More tensors than one launch takes (two launches), an empty tensor, and
    a tensor without statistics: every tensor as if quantized alone."""
    cfg = mx.NVFP4
    shapes = [(64, 512), (0, 256), (33, 1024), (128, 256), (7, 2048), (300, 512)]
    xs = [inputs.laplace_outlier_cols(r, c, seed=20 + i, n_outlier_cols=2, dtype=dtype) * (2.0 ** i)
          if r else torch.zeros(0, c, dtype=dtype) for i, (r, c) in enumerate(shapes)]
    outs = [mx.alloc_outputs(cfg, r, c, "cuda", stats=(i != 3)) for i, (r, c) in enumerate(shapes)]
    qs = mx.quantize_group([x.cuda() for x in xs], cfg, outs=outs)
    torch.cuda.synchronize()
    for i, (x, q) in enumerate(zip(xs, qs)):
        if x.shape[0] == 0:
            alone = mx.quantize(x.cuda(), cfg)
            torch.cuda.synchronize()
            assert np.array_equal(q.stats.cpu().numpy(), alone.stats.cpu().numpy(), equal_nan=True)
            continue
        run_case(mx, orc, x, cfg, check_stats=(i != 3), want_rotated=False, q=q)


@pytest.mark.parametrize("name", ["mxfp4", "nvfp4", "had32", "mbs_oas", "ceil_sf_gemm", "col", "col_nvfp4", "2d"])
def test_group_equals_single_calls(mx, name):
    """The same codes, scales (canonical, or the tcgen05 chunk layout the
    oracle does not produce), macro scales and tensor scales as one call per
    tensor, bit for bit; the statistics sums equal up to the order of the
    binary64 additions (the CTAs of a tensor differ), the counts exactly."""
    cfg = _cfgs(mx)[name]
    xs = [x.cuda() for x in _tensors(name)]
    qs = mx.quantize_group(xs, cfg)
    alone = [mx.quantize(x, cfg) for x in xs]
    torch.cuda.synchronize()
    for q, a in zip(qs, alone):
        assert torch.equal(q.codes, a.codes) and torch.equal(q.scales, a.scales)
        assert torch.equal(q.tensor_scale, a.tensor_scale)
        if cfg.macro_block:
            assert torch.equal(q.macro, a.macro)
        gs, ss = q.stats.cpu().numpy(), a.stats.cpu().numpy()
        for k in (0, 1, 2, 5, 6, 7, 8):
            assert gs[k] == pytest.approx(ss[k], rel=1e-9, abs=1e-300), k
        for k in (3, 4, 9, 10):
            assert gs[k] == ss[k], k


def test_group_workspaces_and_repeats(mx):
    """Caller workspaces, and the group run twice in a row: every launch
    leaves the control words zero, so the second run gives the same results."""
    cfg = mx.NVFP4
    xs = [x.cuda() for x in _tensors("nvfp4")]
    wss = [mx.new_workspace(cfg, *x.shape, "cuda") for x in xs]
    q1 = mx.quantize_group(xs, cfg, workspaces=wss)
    q2 = mx.quantize_group(xs, cfg, workspaces=wss)
    torch.cuda.synchronize()
    for a, b in zip(q1, q2):
        assert torch.equal(a.codes, b.codes) and torch.equal(a.scales, b.scales)
        assert torch.equal(a.tensor_scale, b.tensor_scale)
        assert np.array_equal(a.stats.cpu().numpy(), b.stats.cpu().numpy())
    for w in wss:
        assert int(w[:256].count_nonzero()) == 0
    with pytest.raises(mx.MXError):
        mx.quantize_group(xs[:2], cfg, workspaces=[wss[0], wss[0]])
    assert mx.mx_device_status() == 0


def test_group_given_and_reduced_tensor_scales(mx, orc):
    """The two other tensor-scale modes in a group: a given s_T per tensor
    (TS_GIVEN, read from each tensor's own scalar), and an amax word already
    in each tensor's workspace (TS_AMAX, left there by tensor_amax as the
    row-sharded path does): each tensor as if quantized alone."""
    import dataclasses
    xs = _tensors("nvfp4")
    dx = [x.cuda() for x in xs]
    # given: each tensor's own scale, 1/2 and 3 times its computed one
    alone = [mx.quantize(x, mx.NVFP4) for x in dx]
    torch.cuda.synchronize()
    given = dataclasses.replace(mx.NVFP4, tensor_scale=mx.TS_GIVEN)
    outs = []
    for i, (x, a) in enumerate(zip(dx, alone)):
        ts = (a.tensor_scale * (0.5 if i % 2 else 3.0)).clone()
        outs.append(mx.alloc_outputs(given, *x.shape, "cuda", tensor_scale=ts))
    qs = mx.quantize_group(dx, given, outs=outs)
    torch.cuda.synchronize()
    for x, q in zip(xs, qs):
        run_case(mx, orc, x, given, given_ts=float(q.tensor_scale.item()), want_rotated=False, q=q)
    # reduced amax words
    amax_cfg = dataclasses.replace(mx.NVFP4, tensor_scale=mx.TS_AMAX)
    wss = [mx.new_workspace(amax_cfg, *x.shape, "cuda") for x in dx]
    for x, w in zip(dx, wss):
        mx.tensor_amax(x, amax_cfg, w)
    qs = mx.quantize_group(dx, amax_cfg, workspaces=wss)
    torch.cuda.synchronize()
    for q, a in zip(qs, alone):
        assert torch.equal(q.codes, a.codes) and torch.equal(q.scales, a.scales)
        assert torch.equal(q.tensor_scale, a.tensor_scale)
    for w in wss:
        assert int(w[:256].count_nonzero()) == 0
