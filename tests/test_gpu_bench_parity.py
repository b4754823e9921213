"""GPU parity of the launches the benchmark times, element by element.

Every quantizer call of the benchmark's step -- MXFP4, NVFP4 (tensor-amax
pass + UE4M3 nearest scales), 32-point Hadamard + MXFP4 without the rotated
tensor (the TMA-fed quantizer's rotation path) and MBS + OAS(7) MXFP4 -- on
the full Llama-3-8B layer operands, A 8192 x 4096 and W 14336 x 4096, in the
configuration the benchmark launches them with (one grouped launch over A and
W per variant): packed codes, scales, macro scales, tensor scale and the
dequantized tensor of each tensor bit-exact against the oracle, statistics
within 1e-4; the same tensors quantized alone give the same bits.  Then the same kernels on small ragged
shapes for every rotation x scale combination, and the UE4M3 / UE5M3
nearest-scale block-size sweep of "Is Finer Better?" (experimental analysis:
blocks 8 to 256, with and without the FP32 tensor scale).
"""
import numpy as np
import pytest
import torch

import bench
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


_LAYER = {}


def _layer():
    if not _LAYER:
        a, w = inputs.llama_linear(bench.M_TOK, bench.K_DIM, bench.N_OUT)
        _LAYER.update(A=a, W=w)
    return _LAYER


def _step_quantizers(mx):
    return {(name, t): cfg for name, t, cfg, kind in bench.step_plan(mx) if kind == "q"}


@pytest.mark.parametrize("name", ["mxfp4_row", "nvfp4_row", "had32_mxfp4", "mbs_oas_mxfp4"])
def test_step_call_full_size(mx, orc, name):
    """One quantizer call of the benchmark's step, the grouped launch over the
    full-size A and W (no rotated output: the launch configuration the step
    times), and the step's bf16 dequantizer on the MXFP4 codes; then each
    tensor quantized alone, which must give the same bits."""
    calls = {n: (ts, cfg) for n, ts, cfg, kind in bench.step_calls(bench.step_plan(mx)) if kind == "q"}
    ts, cfg = calls[name]
    assert ts == ("A", "W")
    L = _layer()
    xs = [L[t].cuda() for t in ts]
    qs = mx.quantize_group(xs, cfg)
    torch.cuda.synchronize()
    for t, q in zip(ts, qs):
        run_case(mx, orc, L[t], cfg, want_rotated=False, bf16_out=(name == "mxfp4_row"), q=q)
    for x, q in zip(xs, qs):
        a = mx.quantize(x, cfg)
        torch.cuda.synchronize()
        assert torch.equal(a.codes, q.codes) and torch.equal(a.scales, q.scales)
        assert torch.equal(a.tensor_scale, q.tensor_scale)
        if cfg.macro_block:
            assert torch.equal(a.macro, q.macro)


def test_nvfp4_quantizer_launch_alone_full_size(mx):
    """The launch the benchmark times for NVFP4's quantizer alone: the grouped
    NVFP4 launch over the full-size A and W with each tensor's scale given
    (the values the computed call wrote) gives the computed call's bits."""
    import dataclasses
    L = _layer()
    xs = [L[t].cuda() for t in ("A", "W")]
    computed = mx.quantize_group(xs, mx.NVFP4)
    given = dataclasses.replace(mx.NVFP4, tensor_scale=mx.TS_GIVEN)
    outs = [mx.alloc_outputs(given, *x.shape, "cuda", tensor_scale=q.tensor_scale.clone())
            for x, q in zip(xs, computed)]
    qs = mx.quantize_group(xs, given, outs=outs)
    torch.cuda.synchronize()
    for a, q in zip(computed, qs):
        assert torch.equal(a.codes, q.codes) and torch.equal(a.scales, q.scales)
        assert torch.equal(a.tensor_scale, q.tensor_scale)
        st_a, st_q = a.stats.cpu().numpy(), q.stats.cpu().numpy()
        assert np.array_equal(st_a[[3, 4, 9, 10]], st_q[[3, 4, 9, 10]])
        assert np.allclose(st_a, st_q, rtol=1e-9, atol=0, equal_nan=True)


_GRAD = {}


def _grad():
    if not _GRAD:
        _GRAD["G"] = inputs.gradient_like(bench.GRAD_ROWS, bench.GRAD_COLS, seed=bench.GRAD_SEED)
    return _GRAD["G"]


@pytest.mark.parametrize("name", [n for n, _, _ in bench.extra_row_cases(__import__("microscaling_block_quantization_b200"))])
def test_extra_row_full_size(mx, orc, name):
    """Every extra row of the benchmark in the launch it times: column and 2D
    blocks as one grouped call over the full-size A and W, the fp32 gradient
    rows on the 4096 x 14336 tensor; codes, scales (and offsets) against the
    oracle, and the dequantized tensor and statistics (the gradient rows on
    256 sampled rows of x_hat: the statistics of stochastic rounding are
    covered by the smaller tests)."""
    _, ts, cfg = next(c for c in bench.extra_row_cases(mx) if c[0] == name)
    if ts == ("A", "W"):
        L = _layer()
        qs = mx.quantize_group([L[t].cuda() for t in ts], cfg)
        torch.cuda.synchronize()
        for t, q in zip(ts, qs):
            run_case(mx, orc, L[t], cfg, want_rotated=False, q=q)
        return
    from .test_gpu_quantize import assert_same_f32, ocfg
    x = _grad()
    q = mx.quantize(x.cuda(), cfg)
    torch.cuda.synchronize()
    oc = ocfg(orc, cfg)
    full = orc.quantize(oc, x)
    assert np.array_equal(q.codes.cpu().numpy(), full["packed"].ravel()), "packed codes"
    assert np.array_equal(q.scales.cpu().numpy(), full["scales"]), "scales"
    if cfg.asymmetric:
        assert np.array_equal(q.offsets.cpu().numpy().view(np.uint16), full["offsets"]), "offsets"
    rows = np.random.default_rng(1).choice(x.shape[0], 256, replace=False)
    xh = mx.dequantize(q, torch.float32).cpu().numpy()
    oxh = orc.dequantize(oc, full["packed"], full["scales"], None, None, full["offsets"], *x.shape)
    assert_same_f32(xh[rows], oxh[rows], "dequantized sample")


def test_step_plan_is_covered(mx):
    """Every quantizer launch of the benchmark's step is one of the cases
    above, and the step issues each variant as one call over A and W."""
    names = {name for name, _ in _step_quantizers(mx)}
    assert names == {"mxfp4_row", "nvfp4_row", "had32_mxfp4", "mbs_oas_mxfp4"}
    qcalls = [c for c in bench.step_calls(bench.step_plan(mx)) if c[3] == "q"]
    assert sorted(c[0] for c in qcalls) == sorted(names) and all(c[1] == ("A", "W") for c in qcalls)


RAGGED = [(40, 640), (96, 1152), (1, 128), (264, 384)]


@pytest.mark.parametrize("shape", RAGGED)
@pytest.mark.parametrize("n", [16, 32])
@pytest.mark.parametrize("variant", ["e8m0_b32", "e8m0_b16", "nvfp4", "ue4m3_no_ts", "ue5m3",
                                     "mbs_b32", "mbs_oas_b16", "oas_b32"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_fast_rotation_without_rotated_output(mx, orc, shape, n, variant, dtype):
    """The TMA-fed quantizer's rotation (groups of 16 / 32 butterflied in the
    lane, the normaliser folded into power-of-two scales) on ragged shapes:
    the tile count is not a multiple of the consumer lanes."""
    rows, cols = shape
    kw = dict(hadamard=n)
    if variant == "e8m0_b32":
        kw.update(block=32)
    elif variant == "e8m0_b16":
        kw.update(block=16)
    elif variant == "oas_b32":
        kw.update(block=32, rule=2, oas_tau=7.0)
    elif variant == "nvfp4":
        kw.update(block=16, scale_fmt=1, rule=3, tensor_scale=1)
    elif variant == "ue4m3_no_ts":
        kw.update(block=16, scale_fmt=1, rule=3)
    elif variant == "ue5m3":
        kw.update(block=32, scale_fmt=2, rule=3, tensor_scale=1)
    elif variant == "mbs_b32":
        kw.update(block=32, macro_block=128)
    elif variant == "mbs_oas_b16":
        kw.update(block=16, macro_block=128, rule=2, oas_tau=7.0)
    x = inputs.laplace_outlier_cols(rows, cols, seed=4, n_outlier_cols=min(4, cols // 32), dtype=dtype)
    cfg = mx.Config(**kw)
    q, _ = run_case(mx, orc, x, cfg, want_rotated=False)
    # the lane-per-chunk kernel (taken when the rotated tensor is asked for)
    # gives the same codes and scales
    q2, _ = run_case(mx, orc, x, cfg, want_rotated=True)
    assert torch.equal(q.codes, q2.codes) and torch.equal(q.scales, q2.scales)


@pytest.mark.parametrize("block", [64, 128, 256])
@pytest.mark.parametrize("fmt", [1, 2])
@pytest.mark.parametrize("ts", [0, 1])
@pytest.mark.parametrize("sigma", [0.002, 0.02, 0.2])
def test_nearest_scales_large_blocks(mx, orc, block, fmt, ts, sigma):
    """UE4M3 / UE5M3 nearest scales on blocks of 64, 128 and 256 (a block
    spans 2, 4 or 8 lanes), with and without the FP32 tensor scale."""
    x = inputs.normal(72, 1536, sigma=sigma, seed=1)
    run_case(mx, orc, x, mx.Config(block=block, scale_fmt=fmt, rule=3, tensor_scale=ts))


@pytest.mark.parametrize("block", [8, 16, 32, 64, 128, 256])
@pytest.mark.parametrize("fmt", [1, 2])
@pytest.mark.parametrize("ts", [0, 1])
def test_block_size_sweep_full_size(mx, orc, block, fmt, ts):
    """The block-size sweep on a 4096 x 4096 N(0, 0.002) weight-like tensor
    (seed 1): at this sigma UE4M3 without a tensor scale rounds small blocks'
    scales to zero, the error inversion of "Is Finer Better?"."""
    if "x" not in _C2:
        _C2["x"] = inputs.normal(4096, 4096, sigma=0.002, seed=1)
    run_case(mx, orc, _C2["x"], mx.Config(block=block, scale_fmt=fmt, rule=3, tensor_scale=ts))


_C2 = {}
