"""GPU parity: the sm_100a kernels (through the C ABI) against the CPU oracle.

Bit-exact: packed codes, scale codes, macro-scale codes, offsets, the
per-tensor scale, the rotated tensor and the dequantized values.
Tolerance (binary64 sums of binary32 terms in a different order): 1e-4
relative on the squared sums / MSE / R-MSE, 1e-3 dB on QSNR, exact counts.
"""
import dataclasses
import math

import numpy as np
import pytest
import torch

from microscaling_block_quantization_b200 import inputs

pytestmark = pytest.mark.gpu

REL = 1e-4


@pytest.fixture(scope="module")
def mx():
    from microscaling_block_quantization_b200 import build
    build.build()
    import microscaling_block_quantization_b200 as m
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return m


def ocfg(orc, c):
    return orc.Cfg(elem=c.elem, scale_fmt=c.scale_fmt, rule=c.rule, oas_tau=c.oas_tau,
                   block=c.block, axis=c.axis, round_mode=c.round, asymmetric=c.asymmetric,
                   tensor_scale=c.tensor_scale, macro_block=c.macro_block, hadamard=c.hadamard,
                   seed=c.seed)


def assert_same_f32(a, b, what):
    a = np.asarray(a, np.float32).ravel()
    b = np.asarray(b, np.float32).ravel()
    ab, bb = a.view(np.uint32), b.view(np.uint32)
    nan = np.isnan(a) & np.isnan(b)
    bad = (ab != bb) & ~nan
    assert not bad.any(), f"{what}: {bad.sum()} mismatches, first at {np.argmax(bad)}: {a[bad][:4]} vs {b[bad][:4]}"


def assert_stats(g, o, n):
    g = np.asarray(g, np.float64)
    for i in (0, 1, 5, 6):
        if math.isnan(o[i]):
            assert math.isnan(g[i])
        else:
            assert abs(g[i] - o[i]) <= REL * abs(o[i]) + 1e-300, (i, g[i], o[i])
    if math.isfinite(o[7]):
        assert abs(g[7] - o[7]) <= 1e-3, (g[7], o[7])
    else:
        assert (math.isnan(g[7]) and math.isnan(o[7])) or g[7] == o[7]
    if math.isfinite(o[1]):
        assert abs(g[2] - o[2]) <= 1e-6 * math.sqrt(max(n * o[1], 1e-300)) + 1e-300, (g[2], o[2])
    assert g[3] == o[3] and g[4] == o[4] and g[10] == o[10]


def run_case(mx, orc, x_cpu, cfg, check_stats=True, given_ts=None, want_rotated=None, bf16_out=False, q=None):
    """Quantize on the GPU and with the oracle; compare every output.
    want_rotated: ask the library for the rotated tensor y too (default: when
    the config rotates).  Without it, a rotation with blocks of 16 or 32 runs
    on the TMA-fed quantizer, with it on the lane-per-chunk kernel.
    bf16_out: also compare the bf16 dequantized tensor.  q: outputs the GPU
    already produced for x_cpu (a grouped call), checked instead of a new call."""
    rows, cols = x_cpu.shape
    ts_in = None
    if given_ts is not None:
        ts_in = torch.tensor([given_ts], dtype=torch.float32, device="cuda")
    if want_rotated is None:
        want_rotated = bool(cfg.hadamard)
    if q is None:
        q = mx.quantize(x_cpu.cuda(), cfg, stats=check_stats, tensor_scale=ts_in, rotated=want_rotated)
    xh = mx.dequantize(q, torch.float32)
    torch.cuda.synchronize()
    oc = ocfg(orc, cfg)
    r = orc.quantize(oc, x_cpu, tensor_scale=given_ts)
    assert np.array_equal(q.codes.cpu().numpy(), r["packed"].ravel()), "packed codes"
    assert np.array_equal(q.scales.cpu().numpy(), r["scales"]), "scale codes"
    if cfg.tensor_scale:
        assert_same_f32(q.tensor_scale.cpu().numpy(), [r["tensor_scale"]], "tensor scale")
    if cfg.macro_block:
        assert np.array_equal(q.macro.cpu().numpy(), r["macro"]), "macro scale codes"
    if cfg.asymmetric:
        assert np.array_equal(q.offsets.cpu().numpy().view(np.uint16), r["offsets"]), "offsets"
    if cfg.hadamard and want_rotated:
        assert_same_f32(q.rotated.cpu().numpy(), r["y"], "rotated tensor")
    oxh = orc.dequantize(oc, r["packed"], r["scales"], r["tensor_scale"], r["macro"],
                         r["offsets"], rows, cols, unrotate=False)
    if cfg.hadamard:
        # the library rotates back on dequantize; compare against the oracle's
        oxu = orc.dequantize(oc, r["packed"], r["scales"], r["tensor_scale"], r["macro"],
                             r["offsets"], rows, cols, unrotate=True)
        assert_same_f32(xh.cpu().numpy(), oxu, "dequantized (rotated back)")
        want_bf16 = oxu
    else:
        assert_same_f32(xh.cpu().numpy(), oxh, "dequantized")
        want_bf16 = oxh
    if bf16_out:
        xb = mx.dequantize(q, torch.bfloat16)
        wb = torch.from_numpy(np.ascontiguousarray(want_bf16, np.float32)).to(torch.bfloat16)
        assert torch.equal(xb.cpu().view(torch.int16), wb.view(torch.int16)), "bf16 dequantized"
    if check_stats:
        ost, _ = orc.stats(r["y"], oxh)
        assert_stats(q.stats.cpu().numpy(), ost, rows * cols)
    return q, r


SHAPES = [(256, 256), (40, 544), (96, 1024)]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("block", [8, 16, 32, 64, 128, 256])
def test_mxfp4_row_blocks(mx, orc, shape, block):
    rows, cols = shape
    if cols % block:
        pytest.skip("shape not divisible by block")
    x = inputs.laplace_outlier_cols(rows, cols, seed=4, n_outlier_cols=4)
    run_case(mx, orc, x, mx.Config(block=block))


def test_c1_reference_case(mx, orc):
    """256 x 256 N(0,1) seed 0, MXFP4 floor RTNE: codes, scales, x_hat, MSE, QSNR."""
    run_case(mx, orc, inputs.small_normal(256, 256, seed=0), mx.MXFP4)


@pytest.mark.parametrize("rule,tau", [(1, 7.0), (2, 6.0), (2, 6.5), (2, 7.0), (2, 7.5), (2, 8.0)])
def test_scale_rules(mx, orc, rule, tau):
    x = inputs.laplace_outlier_cols(96, 1024, seed=4)
    run_case(mx, orc, x, mx.Config(rule=rule, oas_tau=tau))


@pytest.mark.parametrize("fmt,rule,ts,block", [
    (1, 3, 1, 16),    # NVFP4: UE4M3 + computed FP32 tensor scale
    (1, 3, 0, 16),    # UE4M3 without a tensor scale
    (2, 3, 0, 16),    # UE5M3
    (2, 3, 1, 8),
    (1, 3, 0, 8),
    (1, 0, 0, 16),    # E4M3 as power-of-two scales
    (2, 1, 0, 32),
    (1, 2, 0, 16),
])
@pytest.mark.parametrize("sigma", [0.002, 0.2])
def test_ue_scales(mx, orc, fmt, rule, ts, block, sigma):
    x = inputs.normal(128, 512, sigma=sigma, seed=1)
    run_case(mx, orc, x, mx.Config(block=block, scale_fmt=fmt, rule=rule, tensor_scale=ts))


def _ue_values(fmt):
    """Finite values of the unsigned scale format, ascending (codes 0..max)."""
    bias, top = (7, 0x7E) if fmt == 1 else (15, 0xFE)
    c = np.arange(top + 1)
    e, m = c >> 3, c & 7
    return np.where(e == 0, m * 2.0 ** (1 - bias - 3), (1 + m / 8.0) * 2.0 ** (e - bias))


@pytest.mark.parametrize("fmt", [1, 2])
@pytest.mark.parametrize("ts", [None, 1.0, 0.3712, 1.7e-3, 2.5e4])
def test_nearest_scale_rounding_boundaries(mx, orc, fmt, ts):
    """Nearest block scales s_b = RTNE((alpha / 6) / s_T) with the block amax
    placed within a few ulps of every rounding boundary of the scale format
    (the midpoints between consecutive codes): the two binary32 quotients must
    be correctly rounded for the codes to match."""
    v = _ue_values(fmt)
    mids = (v[:-1] + v[1:]) / 2.0
    sT = 1.0 if ts is None else float(np.float32(ts))
    k = np.arange(-6, 7)
    target = (mids[:, None] * (1.0 + k[None, :] * 2.0 ** -23)).ravel()
    alpha = (target * 6.0 * sT).astype(np.float32)
    j = np.arange(-2, 3, dtype=np.int64)
    alpha = (alpha.view(np.int32)[:, None].astype(np.int64) + j[None, :]).astype(np.int32).view(np.float32).ravel()
    alpha = alpha[np.isfinite(alpha) & (alpha > 0) & (alpha < 3.0e38)]
    nb = (len(alpha) + 15) // 16 * 16
    alpha = np.resize(alpha, nb)
    rng = np.random.default_rng(3)
    blk = (rng.uniform(-1, 1, (nb, 16)) * alpha[:, None] * 0.9).astype(np.float32)
    blk[:, 0] = alpha
    x = torch.from_numpy(blk.reshape(-1, 256))
    cfg = mx.Config(block=16, scale_fmt=fmt, rule=3, tensor_scale=0 if ts is None else 2)
    run_case(mx, orc, x, cfg, given_ts=None if ts is None else sT)


def test_given_tensor_scale(mx, orc):
    x = inputs.normal(64, 256, sigma=0.02, seed=2)
    run_case(mx, orc, x, mx.Config(block=16, scale_fmt=1, rule=3, tensor_scale=2), given_ts=1.5e-5)


@pytest.mark.parametrize("elem,rule,asym,rnd", [
    (1, 1, 0, 0),     # E3M0 with ceil scale
    (2, 0, 0, 0),     # E2M3
    (3, 0, 0, 0),     # E3M2
    (4, 0, 0, 0),     # INT4 symmetric
    (4, 1, 1, 0),     # INT4 asymmetric min/max
    (0, 0, 1, 0),     # E2M1 asymmetric
    (0, 0, 0, 1),     # ceil rounding
    (0, 0, 0, 2),     # stochastic rounding
    (2, 0, 0, 2),
    (4, 1, 1, 2),
    (1, 1, 0, 1),
])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_elements_and_rounding(mx, orc, elem, rule, asym, rnd, dtype):
    x = inputs.gradient_like(64, 512, seed=5, dtype=dtype)
    run_case(mx, orc, x, mx.Config(elem=elem, rule=rule, asymmetric=asym, round=rnd, seed=12345))


@pytest.mark.parametrize("fmt", [1, 2])
def test_measured_mse_follows_the_model(mx, fmt):
    """The quantizer's measured MSE on 4096 x 4096 N(0, sigma^2) tensors
    (nearest UE4M3 / UE5M3 scales, no tensor scale) against the expected-MSE
    model, and the block-size inversion of narrow distributions with UE4M3
    (absent with UE5M3)."""
    from oracle import mse_model
    name = "ue4m3" if fmt == 1 else "ue5m3"
    got = {}
    for sigma in (0.002, 0.02):
        x = inputs.normal(4096, 4096, sigma=sigma, seed=1, dtype=torch.float32).cuda()
        for block in (8, 16, 32):
            st = mx.quantize(x, mx.Config(block=block, scale_fmt=fmt, rule=mx.RULE_NEAREST)).stats.cpu().numpy()
            want = mse_model.expected_mse(sigma, block, name)["mse"]
            assert st[5] == pytest.approx(want, rel=5e-3), (sigma, block, st[5], want)
            got[sigma, block] = st[5]
    if fmt == 1:
        assert got[0.002, 8] > got[0.002, 16] > got[0.002, 32]
    else:
        assert got[0.002, 8] < got[0.002, 16] < got[0.002, 32]
    assert got[0.02, 8] < got[0.02, 16] < got[0.02, 32]


@pytest.mark.parametrize("block", [8, 16, 32])
@pytest.mark.parametrize("fmt", [1, 2])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_mse_nearest_format_group_step(mx, orc, block, fmt, dtype):
    """MSE rule with a UE4M3 / UE5M3 scale and a given (or unit) tensor
    scale: every block's code is the exact argmin of its binary64 squared
    error over all finite codes.  Codes, scales, x_hat and statistics against
    the oracle on a ragged multi-CTA shape with zero / NaN blocks planted."""
    x = inputs.laplace_outlier_cols(72, 544, seed=4, n_outlier_cols=4, dtype=torch.float32)
    x[3, 32:64] = 0.0
    x[7, 100] = float("nan")
    x = x.to(dtype)
    run_case(mx, orc, x, mx.Config(block=block, scale_fmt=fmt, rule=mx.RULE_MSE, tensor_scale=mx.TS_GIVEN),
             given_ts=0.0123)
    if fmt == 1:
        run_case(mx, orc, x, mx.Config(block=block, scale_fmt=fmt, rule=mx.RULE_MSE))


@pytest.mark.parametrize("shape", [(128, 512), (256, 1024)])
@pytest.mark.parametrize("sf_layout", [0, 1])
def test_mse_nearest_format_alternation(mx, orc, shape, sf_layout):
    """NVFP4 with the alternating global / group scale optimisation: the
    tensor scale is a binary32 result of binary64 reductions summed in a
    different order than the oracle's, so it is compared to 1e-5; given that
    scale, the oracle's group step must reproduce the codes and scales
    exactly.  The squared error is below plain NVFP4's; the workspace header
    is left zero; the GEMM takes the operand like an NVFP4 one."""
    rows, cols = shape
    x = inputs.laplace_outlier_cols(rows, cols, seed=4, n_outlier_cols=8)
    cfg = mx.Config(block=16, scale_fmt=mx.SCALE_UE4M3, rule=mx.RULE_MSE, tensor_scale=mx.TS_COMPUTE,
                    sf_layout=sf_layout)
    ws = mx.new_workspace(cfg, rows, cols, "cuda")
    q = mx.quantize(x.cuda(), cfg, workspace=ws)
    torch.cuda.synchronize()
    assert int(ws[:256].count_nonzero()) == 0
    sT = float(q.tensor_scale.item())
    o = orc.quantize(ocfg(orc, dataclasses.replace(cfg, sf_layout=0)), x)
    assert sT == pytest.approx(o["tensor_scale"], rel=1e-5)
    og = ocfg(orc, dataclasses.replace(cfg, tensor_scale=mx.TS_GIVEN, sf_layout=0))
    r = orc.quantize(og, x, tensor_scale=sT)
    S = cols // 16
    if sf_layout:
        from tests.test_gpu_gemm import chunk_layout
        assert np.array_equal(q.scales.cpu().numpy(), chunk_layout(r["scales"], rows, S))
    else:
        assert np.array_equal(q.scales.cpu().numpy(), r["scales"])
    assert np.array_equal(q.codes.cpu().numpy(), r["packed"].ravel())
    oxh = orc.dequantize(og, r["packed"], r["scales"], sT, None, None, rows, cols)
    assert_stats(q.stats.cpu().numpy(), orc.stats(r["y"], oxh)[0], rows * cols)
    if not sf_layout:
        assert_same_f32(mx.dequantize(q, torch.float32).cpu().numpy(), oxh, "dequantized")
    plain = mx.quantize(x.cuda(), mx.Config(block=16, scale_fmt=mx.SCALE_UE4M3, rule=mx.RULE_NEAREST,
                                            tensor_scale=mx.TS_COMPUTE)).stats.cpu().numpy()
    assert q.stats.cpu().numpy()[1] < plain[1]
    if sf_layout and rows % 128 == 0 and rows >= 256:
        w = inputs.normal(256, cols, sigma=0.02, seed=7)
        qw = mx.quantize(w.cuda(), dataclasses.replace(cfg, sf_layout=1))
        c = mx.gemm(q, qw, out_dtype=torch.float32).cpu().numpy().astype(np.float64)
        torch.cuda.synchronize()
        assert mx.mx_device_status() == 0
        rw = orc.quantize(og, w, tensor_scale=float(qw.tensor_scale.item()))
        wh = orc.dequantize(og, rw["packed"], rw["scales"], float(qw.tensor_scale.item()), None, None, 256, cols)
        ref = oxh.astype(np.float64) @ wh.astype(np.float64).T
        assert np.linalg.norm(c - ref) / np.linalg.norm(ref) < 1e-3


@pytest.mark.parametrize("elem", [0, 1, 2, 3, 4])
@pytest.mark.parametrize("rnd", [0, 1, 2])
@pytest.mark.parametrize("asym", [0, 1])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_general_quantizer_matrix(mx, orc, elem, rnd, asym, dtype):
    """Every element type x rounding mode x offset on a ragged row count
    (72 x 544 = 1224 chunks of 32: four full tiles of 256 and a partial one),
    with zero, NaN and Inf blocks and signed zeros planted."""
    x = inputs.gradient_like(72, 544, seed=5, dtype=torch.float32)
    x[3, 32:64] = 0.0
    x[5, 64:96] = -0.0
    x[7, 100] = float("nan")
    x[9, 200] = float("inf")
    x[11, 0:32] = torch.linspace(-1e-3, 1e-3, 32)
    x = x.to(dtype)
    cfg = mx.Config(elem=elem, round=rnd, asymmetric=asym, rule=1 if (elem == 4 and asym) else 0,
                    seed=0x1234_5678_9ABC)
    run_case(mx, orc, x, cfg)


@pytest.mark.parametrize("elem", [0, 1, 2, 3, 4])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_mse_rule(mx, orc, elem, dtype):
    """MSE-optimal E8M0 scales (k_floor or k_floor + 1 per block, the smaller
    nearest-even squared error): codes, scales and statistics against the
    oracle on a ragged shape, with zero / NaN blocks planted."""
    x = inputs.laplace_outlier_cols(72, 544, seed=4, n_outlier_cols=4, dtype=torch.float32)
    x[3, 32:64] = 0.0
    x[7, 100] = float("nan")
    x = x.to(dtype)
    run_case(mx, orc, x, mx.Config(elem=elem, rule=mx.RULE_MSE))


def test_mse_rule_lowers_mse(mx):
    """The MSE rule never leaves a larger tensor MSE than the floor rule."""
    x = inputs.laplace_outlier_cols(512, 1024, seed=4).cuda()
    a = mx.quantize(x, mx.Config(rule=mx.RULE_MSE)).stats.cpu().numpy()
    b = mx.quantize(x, mx.Config(rule=mx.RULE_FLOOR)).stats.cpu().numpy()
    assert a[5] <= b[5]


@pytest.mark.parametrize("elem", [0, 1, 2, 3, 4])
@pytest.mark.parametrize("rnd", [0, 1, 2])
def test_general_grid_sweep(mx, orc, elem, rnd):
    """Scaled values swept densely across each grid (multiples of 2^-7, so every
    grid point and every midpoint is hit exactly) with the block scale pinned to
    one: element 0 of each block is 2^emax and the others stay below
    2^(emax+1)."""
    emax = {0: 2, 1: 4, 2: 2, 3: 4, 4: 2}[elem]
    maxv = {0: 6.0, 1: 16.0, 2: 7.5, 3: 28.0, 4: 7.0}[elem]
    lim = min(maxv * 1.06, 2.0 ** (emax + 1) - 2.0 ** -7)
    v = np.arange(-lim, lim, 2.0 ** -7, dtype=np.float64).astype(np.float32)
    n = (len(v) + 30) // 31 * 31
    v = np.resize(v, n).reshape(-1, 31)
    rows = (v.shape[0] + 7) // 8 * 8
    blk = np.zeros((rows, 32), np.float32)
    blk[:, 0] = 2.0 ** emax
    blk[:v.shape[0], 1:] = v
    x = torch.from_numpy(blk.reshape(-1, 256))
    run_case(mx, orc, x, mx.Config(elem=elem, round=rnd, seed=99))


@pytest.mark.parametrize("axis,block", [(1, 8), (1, 16), (1, 32), (2, 32)])
@pytest.mark.parametrize("variant", ["plain", "oas", "mbs", "fp6", "asym", "sr", "nvfp4"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_column_and_2d(mx, orc, axis, block, variant, dtype):
    rows, cols = 128, 544 if variant != "mbs" else 640
    x = inputs.laplace_outlier_cols(rows, cols, seed=4, n_outlier_cols=4, dtype=dtype)
    kw = dict(axis=axis, block=block)
    if variant == "oas":
        kw.update(rule=2, oas_tau=7.0)
    elif variant == "mbs":
        kw.update(macro_block=128)
    elif variant == "fp6":
        kw.update(elem=2)
    elif variant == "asym":
        kw.update(elem=4, asymmetric=1, rule=1)
    elif variant == "sr":
        kw.update(round=2, seed=7)
    elif variant == "nvfp4":
        kw.update(scale_fmt=1, rule=3, tensor_scale=1)
    run_case(mx, orc, x, mx.Config(**kw))


@pytest.mark.parametrize("axis,block,n", [(0, 32, 32), (0, 16, 16), (0, 32, 16), (0, 16, 32),
                                          (1, 32, 32), (1, 16, 16), (1, 32, 16), (2, 32, 32),
                                          (2, 32, 16)])
@pytest.mark.parametrize("extra", ["plain", "nvfp4", "mbs"])
def test_hadamard(mx, orc, axis, block, n, extra):
    x = inputs.laplace_outlier_cols(128, 640, seed=4, n_outlier_cols=4)
    kw = dict(axis=axis, block=block, hadamard=n)
    if extra == "nvfp4":
        kw.update(scale_fmt=1, rule=3, tensor_scale=1, block=16 if axis != 2 else 32)
        if axis == 1 and n > kw["block"]:
            pytest.skip("column rotation longer than the block")
    elif extra == "mbs":
        kw.update(macro_block=128)
    run_case(mx, orc, x, mx.Config(**kw))


def test_mbs_row(mx, orc):
    x = inputs.laplace_outlier_cols(128, 1024, seed=4)
    for block in (8, 16, 32, 64, 128):
        run_case(mx, orc, x, mx.Config(block=block, macro_block=128))
        run_case(mx, orc, x, mx.Config(block=block, macro_block=128, rule=2))


# ------------------------------------------------------------- edge cases ----
def test_special_values(mx, orc):
    """NaN / Inf blocks, all-zero blocks, signed zeros, bf16 extremes and
    subnormals, every bf16 bit pattern."""
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(2048, 32)
    x = torch.from_numpy(pats.view(np.int16)).view(torch.bfloat16)
    for cfg in (dict(), dict(rule=1), dict(rule=2), dict(elem=2), dict(elem=3), dict(elem=1, rule=1),
                dict(elem=4), dict(round=1), dict(round=2, seed=3)):
        run_case(mx, orc, x, mx.Config(**cfg), check_stats=False)
    x16 = torch.from_numpy(pats.view(np.int16)).view(torch.bfloat16)      # 2048 x 32, 16-blocks
    for cfg in (dict(block=16, scale_fmt=1, rule=3), dict(block=16, scale_fmt=2, rule=3),
                dict(block=16, scale_fmt=1, rule=0), dict(block=16, scale_fmt=1, rule=4),
                dict(block=32, scale_fmt=2, rule=4), dict(rule=4), dict(elem=4, asymmetric=1, rule=1)):
        run_case(mx, orc, x16, mx.Config(**cfg), check_stats=False)


def test_special_values_mbs(mx, orc):
    """Every bf16 bit pattern under the macro-block scale (rows of 128, so
    each 1 x 128 macro block mixes NaN / Inf, huge, subnormal and zero
    values with ordinary ones): macro codes, codes, scales and x_hat."""
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(512, 128)
    x = torch.from_numpy(pats.view(np.int16)).view(torch.bfloat16)
    perm = np.random.default_rng(3).permutation(65536)
    xp = torch.from_numpy(pats.ravel()[perm].reshape(512, 128).view(np.int16)).view(torch.bfloat16)
    for t in (x, xp):
        for cfg in (dict(macro_block=128), dict(macro_block=128, rule=1), dict(macro_block=128, rule=2, oas_tau=7.0),
                    dict(macro_block=128, block=16), dict(macro_block=128, block=16, rule=2, oas_tau=6.5)):
            run_case(mx, orc, t, mx.Config(**cfg), check_stats=False)


@pytest.mark.parametrize("path", ["had32", "had16", "nvfp4_had16", "had32_mbs", "col", "col_nvfp4", "col_mbs", "2d",
                                  "2d_nvfp4"])
def test_special_values_other_paths(mx, orc, path):
    """Every bf16 bit pattern through the rotation (TMA-fed and lane-per-chunk
    kernels), column-block and 2D-tile quantizers: NaN / Inf spreading through
    the butterflies, huge, subnormal and zero values."""
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    perm = np.random.default_rng(5).permutation(65536)
    shape = (512, 128) if path in ("had32_mbs", "col_mbs") else (2048, 32)
    x = torch.from_numpy(pats[perm].reshape(shape).view(np.int16)).view(torch.bfloat16)
    nv = dict(block=16, scale_fmt=1, rule=3, tensor_scale=1)
    cfg = {"had32": dict(hadamard=32), "had16": dict(hadamard=16, block=16),
           "nvfp4_had16": dict(hadamard=16, **nv), "had32_mbs": dict(hadamard=32, macro_block=128),
           "col": dict(axis=1), "col_nvfp4": dict(axis=1, **nv), "col_mbs": dict(axis=1, macro_block=128),
           "2d": dict(axis=2), "2d_nvfp4": dict(axis=2, block=32, scale_fmt=1, rule=3, tensor_scale=1)}[path]
    c = mx.Config(**cfg)
    if c.hadamard:
        run_case(mx, orc, x, c, check_stats=False, want_rotated=False)
        run_case(mx, orc, x, c, check_stats=False, want_rotated=True)
    else:
        run_case(mx, orc, x, c, check_stats=False)


def test_wide_dynamic_range(mx, orc):
    """Finite values from 2^-133 to 2^126 (bf16 subnormals included), the
    magnitudes of a row spread over the whole range or over a narrow band at
    either end, through MBS, MXFP4, NVFP4 (blocks far below the tensor's
    maximum flush to a zero scale), rotation, column and 2D blocks: codes,
    scales, macro codes, x_hat and the statistics (the squares of values
    above 2^64 overflow binary32, so the sums must be taken on scaled values).  The largest values
    stay below 2^126: within a factor 2 of the binary32 maximum a dequantized
    value can itself overflow, where the oracle's error sum is infinite and
    the fused sums (formed exactly as X (s - q) in binary64) are not."""
    rng = np.random.default_rng(11)
    rows = []
    for lo, hi in ((-133, 126), (-133, -100), (100, 126), (-20, 20)):
        e = rng.uniform(lo, hi, size=(64, 256))
        m = rng.uniform(1.0, 2.0, size=(64, 256))
        rows.append(np.where(rng.random((64, 256)) < 0.5, -1.0, 1.0) * m * np.exp2(e))
    x = torch.from_numpy(np.concatenate(rows).astype(np.float32)).to(torch.bfloat16)
    # scales that span the range: E8M0, or UE4M3 with the FP32 tensor scale
    # (UE scales without one saturate for blocks far above their range, and
    # a rotation of values near the binary32 maximum overflows)
    for cfg in (dict(macro_block=128), dict(macro_block=128, rule=2, oas_tau=7.0), dict(macro_block=128, block=16),
                dict(), dict(rule=1), dict(block=16, scale_fmt=1, rule=3, tensor_scale=1),
                dict(axis=1), dict(axis=2), dict(axis=1, block=16, scale_fmt=1, rule=3, tensor_scale=1),
                dict(axis=2, scale_fmt=1, rule=3, tensor_scale=1)):
        c = mx.Config(**cfg)
        run_case(mx, orc, x, c, want_rotated=False if c.hadamard else None)
    # the same values as fp32 input (the lane-per-chunk path of the fast quantizer)
    run_case(mx, orc, x.float(), mx.Config(macro_block=128))
    run_case(mx, orc, x.float(), mx.Config(block=16, scale_fmt=1, rule=3, tensor_scale=1))


def test_zeros_and_empty(mx, orc):
    z = torch.zeros(64, 256, dtype=torch.bfloat16)
    q, _ = run_case(mx, orc, z, mx.MXFP4)
    st = q.stats.cpu().numpy()
    assert math.isnan(st[7]) and st[5] == 0
    e = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    q = mx.quantize(e, mx.MXFP4)
    st = q.stats.cpu().numpy()
    assert st[10] == 0 and math.isnan(st[7])


def test_workspace_control_words_left_zero(mx):
    """The quantizer's last CTA sums the statistics and clears the workspace's
    control words (tensor-amax accumulator, launch ticket): after calls with a
    computed tensor scale and statistics the first 256 bytes are zero again,
    and repeated calls give identical statistics."""
    x = inputs.normal(512, 1024, sigma=0.02, seed=2).cuda()
    runs = []
    for cfg in (mx.NVFP4, mx.MXFP4, mx.NVFP4, mx.Config(elem=mx.E2M3), mx.Config(axis=1)):
        q = mx.quantize(x, cfg, stats=True)
        torch.cuda.synchronize()
        ws = mx._default_ws[str(x.device)].buf
        assert int(ws[:256].count_nonzero()) == 0
        runs.append(q.stats.cpu().numpy().copy())
    assert np.array_equal(runs[0], runs[2])


def test_fast_path_conversion_rounding(mx):
    """The E2M1 conversion instruction used by the fast path, swept over
    [-7.5, 7.5] with the block scale pinned to 1: every code is the nearest
    grid point (ties to the even code), saturating at 6, sign kept."""
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    v = np.linspace(-7.5, 7.5, 32 * 2048, dtype=np.float32).reshape(2048, 32)
    v[:, 0] = 6.0                                   # fixes every block scale to 1
    q = mx.quantize(torch.from_numpy(v).cuda(), mx.MXFP4, stats=False)
    codes = q.codes.cpu().numpy()
    lo, hi = codes & 0xF, codes >> 4
    c = np.stack([lo, hi], axis=-1).reshape(2048, 32)
    mag = np.abs(v.astype(np.float64))
    d = np.abs(mag[..., None] - grid)
    best = np.argmin(d, axis=-1)
    ties = (np.sort(d, axis=-1)[..., 0] == np.sort(d, axis=-1)[..., 1])
    best = np.where(ties & (best % 2 == 1), best + 1, best)
    best = np.minimum(best, 7)
    want = best | ((np.signbit(v)).astype(np.int64) << 3)
    assert np.array_equal(c, want)


# ------------------------------------------------------- standalone qsnr ----
@pytest.mark.parametrize("axis,block", [(0, 32), (0, 8), (0, 256), (1, 16), (1, 32), (2, 32)])
def test_qsnr_and_per_block_mse(mx, orc, axis, block):
    x = inputs.laplace_outlier_cols(128, 512, seed=4)
    q = mx.quantize(x.cuda(), mx.Config(axis=axis, block=block), stats=False)
    xh = mx.dequantize(q, torch.float32)
    st, pb = mx.qsnr(x.cuda(), xh, block=block, axis=axis, per_block=True)
    ost, opb = orc.stats(orc.input_f32(x), xh.cpu().numpy(), block=block, axis=axis)
    assert_stats(st.cpu().numpy(), ost, x.numel())
    assert np.allclose(pb.cpu().numpy(), opb, rtol=1e-5, atol=1e-30)
    xb = mx.dequantize(q, torch.bfloat16)
    assert torch.equal(xb.cpu(), xh.cpu().to(torch.bfloat16))
    st2, _ = mx.qsnr(x.cuda(), xb)
    ost2, _ = orc.stats(orc.input_f32(x), orc.input_f32(xb.cpu()))
    assert_stats(st2.cpu().numpy(), ost2, x.numel())


def test_concurrent_streams_with_own_workspaces(mx):
    """Quantizer calls running at the same time on two streams, each with its
    own workspace (control words and statistics records), give exactly the
    results of the same calls one after the other."""
    a = inputs.laplace_outlier_cols(2048, 4096, seed=4).cuda()
    w = inputs.normal(4096, 4096, sigma=0.02, seed=7).cuda()
    cfgs = [mx.MXFP4, mx.NVFP4, mx.Config(hadamard=32)]
    ref = [(mx.quantize(x, c), c) for c in cfgs for x in (a, w)]
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    w1, w2 = mx.new_workspace(mx.MXFP4, 1, 32, "cuda"), mx.new_workspace(mx.MXFP4, 1, 32, "cuda")
    outs = []
    for _ in range(3):
        for c in cfgs:
            with torch.cuda.stream(s1):
                q1 = mx.quantize(a, c, stream=s1, workspace=w1)
            with torch.cuda.stream(s2):
                q2 = mx.quantize(w, c, stream=s2, workspace=w2)
            outs += [q1, q2]
    torch.cuda.synchronize()
    assert mx.mx_device_status() == 0
    for k, q in enumerate(outs):
        r, _ = ref[k % len(ref)]
        assert torch.equal(q.codes, r.codes) and torch.equal(q.scales, r.scales)
        assert torch.equal(q.tensor_scale, r.tensor_scale)
        assert np.array_equal(q.stats.cpu().numpy(), r.stats.cpu().numpy())
    for ws in (w1, w2):
        assert int(ws[:256].count_nonzero()) == 0


def test_stats_reproducible(mx):
    x = inputs.laplace_outlier_cols(512, 1024, seed=4).cuda()
    a = mx.quantize(x, mx.MXFP4).stats.cpu().numpy()
    b = mx.quantize(x, mx.MXFP4).stats.cpu().numpy()
    assert np.array_equal(a, b)


# ------------------------------------------------------ full-size configs ----
@pytest.mark.parametrize("name", ["c3_row", "c3_col", "c3_2d", "c3_mbs", "c3_had", "c3_oas"])
def test_activation_config_full_size(mx, orc, name):
    """8192 x 4096 Laplace activations with 16 outlier columns: every output
    against the oracle at full size, in the launch configuration of the
    benchmark."""
    x = _c3()
    cfg = {"c3_row": mx.MXFP4, "c3_col": mx.Config(axis=1), "c3_2d": mx.Config(axis=2),
           "c3_mbs": mx.Config(macro_block=128), "c3_had": mx.Config(hadamard=32),
           "c3_oas": mx.Config(rule=2, oas_tau=7.0)}[name]
    run_case(mx, orc, x, cfg)


_C3 = {}


def _c3():
    if "x" not in _C3:
        _C3["x"] = inputs.laplace_outlier_cols(8192, 4096, seed=4)
    return _C3["x"]


def test_gradient_config_full_size(mx, orc):
    """4096 x 14336 fp32 gradients with 1% large entries, stochastic rounding
    (Philox keyed on the seed and the element index): codes and scales against
    the oracle at full size; the sampled 256 rows also through dequantize."""
    x = inputs.gradient_like(4096, 14336, seed=5)
    cfg = mx.Config(round=2, seed=5)
    q = mx.quantize(x.cuda(), cfg)
    full = orc.quantize(ocfg(orc, cfg), x)
    assert np.array_equal(q.codes.cpu().numpy(), full["packed"].ravel())
    assert np.array_equal(q.scales.cpu().numpy(), full["scales"])
    rows = np.random.default_rng(0).choice(4096, 256, replace=False)
    xh = mx.dequantize(q, torch.float32).cpu().numpy()
    oxh = orc.dequantize(ocfg(orc, cfg), full["packed"], full["scales"], None, None, None,
                         4096, 14336)
    assert_same_f32(xh[rows], oxh[rows], "dequantized sample")
