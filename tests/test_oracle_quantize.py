"""CPU pins of the oracle quantizer, dequantizer and fidelity reductions.

Pins used here: closed forms (single-value blocks under the floor rule, QSNR
of a uniformly shrunk tensor), exhaustive sweeps over all 65536 bf16 bit
patterns, invariants of the scale rules (ceil never saturates, OAS(6) ==
ceil, OAS(8) == floor), library routines for special cases (scipy's
Hadamard matrix, numpy's binary64 matmul), statistical properties
(stochastic-rounding unbiasedness) and the trends the pages report.
"""
import math

import numpy as np
import pytest
import scipy.linalg
import torch

from microscaling_block_quantization_b200 import inputs
from tests.test_oracle_formats import page_facts, _nearest_even

E2M1_GRID = [float(v) for v in page_facts()["e2m1_magnitudes"].split()]


def all_bf16_patterns():
    return np.arange(65536, dtype=np.uint32).astype(np.uint16)


def bf16_value(bits):
    return float(np.array([int(bits) << 16], np.uint32).view(np.float32)[0])


# ------------------------------------------------ floor rule, exhaustive ----
def test_floor_rule_single_value_blocks_exhaustive(orc):
    """Every finite bf16 value v alone in a 32-block (rest zeros): its scale is
    2^(floor(log2|v|) - 2) clamped to E8M0, and it decodes to 4*2^(e-2) when
    the mantissa m <= 1.25 (5 is a tie that goes to the even code, 4), else
    6*2^(e-2)."""
    pats = all_bf16_patterns()
    vals = (pats.astype(np.uint32) << 16).view(np.float32)
    keep = np.isfinite(vals) & (vals != 0)
    pats = pats[keep]
    vals = vals[keep]
    x = np.zeros((len(pats), 32), np.uint16)
    x[:, 0] = pats
    cfg = orc.Cfg(block=32)
    q = orc.quantize(cfg, x)
    xh = orc.dequantize(cfg, q["packed"], q["scales"], None, None, None, *x.shape)
    assert np.all(xh[:, 1:] == 0)
    for i, v in enumerate(vals.tolist()):
        m, e2 = math.frexp(abs(v))          # |v| = m 2^e2, m in [0.5, 1)
        e = e2 - 1
        mant = m * 2
        k = max(e - 2, -127)
        assert q["scales"][i] == k + 127
        if e - 2 >= -127:
            want = (4.0 if mant <= 1.25 else 6.0) * 2.0 ** (e - 2)
        else:
            r = abs(v) * 2.0 ** 127       # exact in binary64
            want = E2M1_GRID[_nearest_even(E2M1_GRID, r)] * 2.0 ** -127
        assert xh[i, 0] == math.copysign(want, v), (v, xh[i, 0], want)


@pytest.mark.parametrize("elem", ["E2M1", "E3M0", "E2M3", "E3M2", "INT4"])
def test_all_bf16_patterns_as_blocks(orc, elem):
    """All 65536 bf16 patterns laid out as 2048 x 32: blocks holding a
    non-finite value get the NaN scale code and zero codes; every other block
    has a power-of-two scale X with alpha/X in [2^emax, 2^(emax+1)) (the floor
    rule's defining property) unless clamped, and each code is the grid point
    nearest to x/X (ties to even), saturating."""
    E = getattr(orc, elem)
    x = all_bf16_patterns().reshape(2048, 32)
    cfg = orc.Cfg(elem=E, block=32)
    q = orc.quantize(cfg, x)
    xf = orc.bf16_bits_to_f32(x)
    emax = {"E2M1": 2, "E3M0": 4, "E2M3": 2, "E3M2": 4, "INT4": 2}[elem]
    nb = 6 if elem in ("E2M3", "E3M2") else 4
    ncode = 1 << (nb - 1)
    grid = [orc.decode_elem(E, c) for c in range(ncode)]
    for b in range(2048):
        row = xf[b]
        if not np.all(np.isfinite(row)):
            assert q["scales"][b] == 0xff
            assert np.all(q["codes"][b] == 0)
            continue
        alpha = float(np.max(np.abs(row)))
        if alpha == 0:
            assert q["scales"][b] == 0 and np.all(q["codes"][b] == 0)
            continue
        X = 2.0 ** (int(q["scales"][b]) - 127)
        if int(q["scales"][b]) > 0:
            assert 2 ** emax <= alpha / X < 2 ** (emax + 1)
        for t in range(32):
            v = float(row[t]) / X
            code = int(q["codes"][b, t])
            if elem == "INT4":
                mag = abs(orc.decode_elem(E, code))
            else:
                mag = grid[code & (ncode - 1)]
            want = grid[_nearest_even(grid, min(abs(v), grid[-1]))]
            assert mag == want, (b, t, v, mag, want)


# ------------------------------------------------ ceil / OAS invariants ----
def _laplace(rows=256, cols=256, seed=4):
    return inputs.laplace_outlier_cols(rows, cols, seed=seed, n_outlier_cols=4)


def test_ceil_never_saturates_and_oas_bounds(orc):
    x = _laplace()
    xf = orc.input_f32(x)
    fl = orc.quantize(orc.Cfg(rule=orc.FLOOR), x)
    ce = orc.quantize(orc.Cfg(rule=orc.CEIL), x)
    alpha = np.abs(xf).reshape(-1, 32).max(axis=1)
    Xc = 2.0 ** (ce["scales"].astype(np.float64) - 127)
    assert np.all(alpha <= 6.0 * Xc)                      # no overflow under ceil
    assert np.all(alpha > 6.0 * Xc / 2)                   # and it is the smallest such
    for tau in (6.5, 7.0, 7.5):
        oa = orc.quantize(orc.Cfg(rule=orc.OAS, oas_tau=tau), x)
        d = oa["scales"].astype(int) - fl["scales"].astype(int)
        assert set(np.unique(d)) <= {0, 1}                 # OAS in {X_floor, 2 X_floor}
    o6 = orc.quantize(orc.Cfg(rule=orc.OAS, oas_tau=6.0), x)
    o8 = orc.quantize(orc.Cfg(rule=orc.OAS, oas_tau=8.0), x)
    assert np.array_equal(o6["scales"], ce["scales"]) and np.array_equal(o6["codes"], ce["codes"])
    assert np.array_equal(o8["scales"], fl["scales"]) and np.array_equal(o8["codes"], fl["codes"])


def test_e3m0_ceil_scale_gradients(orc):
    x = inputs.gradient_like(64, 256, seed=5)
    q = orc.quantize(orc.Cfg(elem=orc.E3M0, rule=orc.CEIL), x)
    xf = orc.input_f32(x)
    alpha = np.abs(xf).reshape(-1, 32).max(axis=1)
    X = 2.0 ** (q["scales"].astype(np.float64) - 127)
    assert np.all(alpha <= 16 * X) and np.all(alpha > 8 * X)


# ------------------------------------------------------ scale formats ----
def test_nvfp4_tensor_scale_puts_top_block_at_448(orc):
    x = inputs.laplace_outlier_cols(128, 256, seed=6, n_outlier_cols=2)
    cfg = orc.Cfg(block=16, scale_fmt=orc.UE4M3, rule=orc.NEAREST, tensor_scale=orc.TS_COMPUTE)
    q = orc.quantize(cfg, x)
    xf = orc.input_f32(x)
    assert q["tensor_scale"] == np.float32(np.abs(xf).max()) / np.float32(6 * 448)
    assert q["scales"].max() == 0x7e
    assert q["scales"].max() == orc.scale_encode_nearest(orc.UE4M3, 448.0)


def test_ue4m3_zero_rounding_block(orc):
    """A block whose alpha/6 is below half the UE4M3 minimum (2^-9) rounds its
    scale to zero and flushes every element (the zero-rounding error term)."""
    x = np.zeros((1, 16), np.float32)
    x[0, :] = np.linspace(-1, 1, 16, dtype=np.float32) * np.float32(6 * 2 ** -11)
    cfg = orc.Cfg(block=16, scale_fmt=orc.UE4M3, rule=orc.NEAREST)
    q = orc.quantize(cfg, x)
    assert q["scales"][0] == 0 and np.all(q["codes"] & 7 == 0)
    q5 = orc.quantize(orc.Cfg(block=16, scale_fmt=orc.UE5M3, rule=orc.NEAREST), x)
    assert q5["scales"][0] != 0 and np.any(q5["codes"] & 7 != 0)


def test_storage_bits_per_element(orc):
    f = page_facts()
    x = inputs.small_normal(64, 256, seed=0)
    mx = orc.quantize(orc.Cfg(block=32), x)
    nv = orc.quantize(orc.Cfg(block=16, scale_fmt=orc.UE4M3, rule=orc.NEAREST,
                              tensor_scale=orc.TS_COMPUTE), x)
    n = x.numel()
    assert (mx["packed"].nbytes + mx["scales"].nbytes) * 8 / n == float(f["mxfp4_bits_per_element"])
    assert (nv["packed"].nbytes + nv["scales"].nbytes) * 8 / n == float(f["nvfp4_bits_per_element"])


def test_power_of_two_ue4m3_equals_e8m0_in_range(orc):
    """E4M3 restricted to powers of two ("E4M0"): identical codes to E8M0 when
    every block exponent is inside the E4M3 range."""
    x = inputs.small_normal(64, 256, seed=3)
    a = orc.quantize(orc.Cfg(block=16), x)
    b = orc.quantize(orc.Cfg(block=16, scale_fmt=orc.UE4M3, rule=orc.FLOOR), x)
    assert np.array_equal(a["codes"], b["codes"])
    for sa, sb in zip(a["scales"], b["scales"]):
        assert orc.scale_decode(orc.E8M0, int(sa)) == orc.scale_decode(orc.UE4M3, int(sb))


# ------------------------------------------------- stochastic rounding ----
def test_sr_unbiased_and_seeded(orc):
    rows, cols = 4096, 32
    x = np.zeros((rows, cols), np.float32)
    x[:, 0] = 6.0                                   # fixes X = 1 in every block
    v = np.float32(2.3)
    x[:, 1:] = v
    means = []
    for seed in (1, 2):
        q = orc.quantize(orc.Cfg(round_mode=orc.SR, seed=seed), x)
        xh = orc.dequantize(orc.Cfg(), q["packed"], q["scales"], None, None, None, rows, cols)
        s = xh[:, 1:].astype(np.float64)
        assert set(np.unique(s)) == {2.0, 3.0}
        p = 0.3
        sigma = math.sqrt(p * (1 - p)) / math.sqrt(s.size)
        assert abs(s.mean() - float(v)) < 4 * sigma
        means.append(q["codes"])
    assert not np.array_equal(means[0], means[1])          # seed changes codes
    again = orc.quantize(orc.Cfg(round_mode=orc.SR, seed=1), x)
    assert np.array_equal(again["codes"], means[0])        # same seed, same codes


def test_sr_word_is_philox_of_element_index(orc):
    """Single block, SR: element i rounds up iff (word_i >> 8) < p * 2^24 with
    word_i = Philox4x32-10(counter (i/4, 0, 0, 0), key seed)[i % 4]."""
    seed = 0x1234_5678_9ABC
    x = np.full((1, 32), 2.3, np.float32)
    x[0, 0] = 6.0
    q = orc.quantize(orc.Cfg(round_mode=orc.SR, seed=seed), x)
    p = (np.float32(2.3) - np.float32(2.0)) / np.float32(1.0)
    for i in range(1, 32):
        words = orc.philox([i // 4, 0, 0, 0], [seed & 0xffffffff, seed >> 32])
        up = float(words[i % 4] >> 8) < float(p) * 2 ** 24
        assert orc.decode_elem(orc.E2M1, int(q["codes"][0, i])) == (3.0 if up else 2.0)


# ------------------------------------------------------------ INT4 asym ----
def test_int4_asymmetric_properties(orc):
    x = inputs.gradient_like(32, 128, seed=5)
    cfg = orc.Cfg(elem=orc.INT4, asymmetric=1, rule=orc.CEIL)
    q = orc.quantize(cfg, x)
    xh = orc.dequantize(cfg, q["packed"], q["scales"], None, None, q["offsets"], 32, 128)
    xf = orc.input_f32(x).reshape(-1, 32).astype(np.float64)
    X = 2.0 ** (q["scales"].astype(np.float64) - 127)
    o = orc.bf16_bits_to_f32(q["offsets"]).astype(np.float64)
    mn = xf.min(axis=1)
    mx = xf.max(axis=1)
    assert np.all(o == orc.bf16_bits_to_f32(torch.from_numpy(mn.astype(np.float32)).to(
        torch.bfloat16).view(torch.int16).numpy().view(np.uint16)))           # o = bf16(min)
    assert np.all(mx - o <= 15 * X) and np.all(mx - o > 15 * X / 2)          # smallest k
    qv = (xh.reshape(-1, 32) - o[:, None]) / X[:, None]
    assert np.all(np.abs(qv - np.round(qv)) < 1e-6) and qv.min() >= 0 and qv.max() <= 15
    err = np.abs(xh.reshape(-1, 32) - xf)
    assert np.all(err <= X[:, None] / 2 + np.abs(o)[:, None] * 2 ** -23 + 1e-30)


def test_asymmetric_int4_beats_symmetric(orc):
    """Asymmetric scaling greatly improves INT4 (fmread summary of Yang et al.,
    design-choice results) on one-sided blocks."""
    x = np.abs(inputs.gradient_like(64, 256, seed=5).numpy()) + np.float32(1e-3)
    sy = orc.quantize(orc.Cfg(elem=orc.INT4, rule=orc.CEIL), x)
    asy_cfg = orc.Cfg(elem=orc.INT4, asymmetric=1, rule=orc.CEIL)
    asy = orc.quantize(asy_cfg, x)
    xs = orc.dequantize(orc.Cfg(elem=orc.INT4), sy["packed"], sy["scales"], None, None, None, 64, 256)
    xa = orc.dequantize(asy_cfg, asy["packed"], asy["scales"], None, None, asy["offsets"], 64, 256)
    assert orc.stats(x, xa)[0][5] < 0.5 * orc.stats(x, xs)[0][5]


# --------------------------------------------------------------- Hadamard ----
@pytest.mark.parametrize("n", [16, 32])
def test_fwht_matches_sylvester_matrix(orc, n):
    H = scipy.linalg.hadamard(n)
    assert np.array_equal(H @ H.T, n * np.eye(n))
    rng = np.random.default_rng(n)
    for _ in range(20):
        v = rng.integers(-1000, 1000, n).astype(np.float32)
        assert np.array_equal(orc.fwht(v, normalise=False), (H @ v.astype(np.int64)).astype(np.float32))
    cols = np.stack([orc.fwht(np.eye(n, dtype=np.float32)[i], normalise=False) for i in range(n)])
    assert np.array_equal(cols, H)


def test_fwht16_normalised_exact_for_dyadic(orc):
    H = scipy.linalg.hadamard(16)
    rng = np.random.default_rng(2)
    v = (rng.integers(-64, 64, 16) / 8).astype(np.float32)
    assert np.array_equal(orc.fwht(v), (H @ v.astype(np.float64) / 4).astype(np.float32))


def test_hadamard_quantize_reference_is_rotation(orc):
    x = _laplace(64, 128)
    for axis in (orc.ROW, orc.COL, orc.TWO_D):
        q = orc.quantize(orc.Cfg(hadamard=32, axis=axis), x)
        xf = orc.input_f32(x).astype(np.float64)
        H = scipy.linalg.hadamard(32) / math.sqrt(32)
        if axis == orc.COL:
            want = np.concatenate([H @ xf[i:i + 32] for i in range(0, 64, 32)])
        else:
            want = np.concatenate([xf[:, j:j + 32] @ H for j in range(0, 128, 32)], axis=1)
        assert np.allclose(q["y"], want, rtol=0, atol=1e-5 * np.abs(xf).max())


# -------------------------------------------------------------------- MBS ----
def test_mbs_identity_when_macro_mantissa_is_1p5(orc):
    rng = np.random.default_rng(0)
    x = (rng.standard_normal((8, 256)) * 0.3).astype(np.float32)
    x = np.clip(x, -0.7, 0.7)
    x[:, 5] = 1.5 * 2.0                # every macro block's absmax = 3 = 1.5 * 2
    x[:, 130] = -3.0
    plain = orc.quantize(orc.Cfg(), x)
    mbs = orc.quantize(orc.Cfg(macro_block=128), x)
    assert np.all(mbs["macro"] == orc.scale_encode_nearest(orc.UE4M3, 1.0))
    assert np.array_equal(plain["codes"], mbs["codes"])
    assert np.array_equal(plain["scales"], mbs["scales"])


def test_mbs_macro_max_exact(orc):
    """With S_M exactly representable in E4M3, the macro-block maximum is
    reproduced exactly (MBS keeps outliers)."""
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((16, 256)) * 0.05).astype(np.float32)
    amax = np.float32(1.3125 * 2.0 ** -1)           # 1.3125 / 1.5 = 0.875 in E4M3
    x[:, 7] = amax
    x[:, 200] = -amax
    cfg = orc.Cfg(macro_block=128)
    q = orc.quantize(cfg, x)
    xh = orc.dequantize(cfg, q["packed"], q["scales"], None, q["macro"], None, 16, 256)
    assert np.all(xh[:, 7] == amax) and np.all(xh[:, 200] == -amax)
    plain = orc.quantize(orc.Cfg(), x)
    xp = orc.dequantize(orc.Cfg(), plain["packed"], plain["scales"], None, None, None, 16, 256)
    assert np.all(xp[:, 7] != amax)                 # plain MXFP4 cannot represent it


# ------------------------------------------------------------- reductions ----
def test_qsnr_closed_form(orc):
    x = orc.input_f32(inputs.small_normal(64, 64, seed=9))
    for j in (2, 4, 6):
        eps = 2.0 ** -j
        xh = (x * np.float32(1 - eps)).astype(np.float32)      # exact: bf16 x, 1 - 2^-j
        st, _ = orc.stats(x, xh)
        assert abs(st[7] - (-20 * math.log10(eps))) < 1e-9
        assert abs(st[5] - eps ** 2 * np.mean(x.astype(np.float64) ** 2)) < 1e-12
        assert abs(st[6] - math.sqrt(st[5])) < 1e-15
        assert abs(st[8] + eps * np.mean(x.astype(np.float64))) < 1e-12
    st, _ = orc.stats(x, x)
    assert st[7] == math.inf
    st, _ = orc.stats(np.zeros_like(x), x)
    assert math.isnan(st[7])


def test_ftz_fraction_and_per_block_mse(orc):
    x = _laplace(64, 128)
    q = orc.quantize(orc.Cfg(), x)
    xh = orc.dequantize(orc.Cfg(), q["packed"], q["scales"], None, None, None, 64, 128)
    xf = orc.input_f32(x)
    st, pb = orc.stats(xf, xh, block=32, axis=orc.ROW)
    nz = xf != 0
    assert st[9] == np.sum(nz & (xh == 0)) / np.sum(nz)
    assert abs(np.mean(pb.astype(np.float64)) - st[5]) < 1e-6 * st[5]


def test_gemm_oracle_against_blas_and_closed_form(orc):
    rng = np.random.default_rng(0)
    # bf16-representable operands, so that A * (1 - 2^-5) is exact in binary32
    A = orc.input_f32(inputs.to_bf16(rng.standard_normal((24, 64)).astype(np.float32)))
    B = orc.input_f32(inputs.to_bf16(rng.standard_normal((40, 64)).astype(np.float32)))
    C = orc.gemm(A, B)
    assert np.allclose(C, A.astype(np.float64) @ B.T.astype(np.float64), rtol=1e-12, atol=1e-12)
    eps = 2.0 ** -5
    out = orc.gemm_qsnr(A, B, (A * np.float32(1 - eps)).astype(np.float32), B)
    assert abs(out[2] - (-20 * math.log10(eps))) < 1e-9
    Ah = rng.standard_normal((24, 64)).astype(np.float32)
    assert np.allclose(orc.gemm_qsnr(A, B, Ah, B), orc.gemm_qsnr_blas(A, B, Ah, B), rtol=1e-10)


# -------------------------------------------------------- trends of pages ----
def _qsnr(orc, cfg, x, **kw):
    q = orc.quantize(cfg, x)
    xh = orc.dequantize(cfg, q["packed"], q["scales"], q["tensor_scale"], q["macro"],
                        q["offsets"], *q["y"].shape)
    return orc.stats(q["y"], xh)[0]


def test_trend_block16_and_oas_raise_qsnr(orc):
    x = inputs.laplace_outlier_cols(512, 512, seed=4, n_outlier_cols=2)
    b32 = _qsnr(orc, orc.Cfg(block=32), x)[7]
    b16 = _qsnr(orc, orc.Cfg(block=16), x)[7]
    oas = _qsnr(orc, orc.Cfg(block=32, rule=orc.OAS, oas_tau=7.0), x)[7]
    had = _qsnr(orc, orc.Cfg(block=32, hadamard=32), x)[7]
    assert 0.3 < b16 - b32 < 2.5          # pages: about +1 dB from 32 to 16
    assert 0.1 < oas - b32 < 1.5          # pages: OAS about +0.5 dB
    assert had > b32                      # rotation helps MXFP4 on Laplace data


def test_trend_small_block_inversion_ue4m3(orc):
    """Narrow weights (sigma = 0.002) with UE4M3 scales and no tensor scale:
    the per-tensor MSE at block 8 exceeds that at block 16; with UE5M3, or a
    per-tensor FP32 scale, it does not (Is Finer Better?)."""
    x = inputs.normal(512, 512, sigma=0.002, seed=1)

    def mse(fmt, B, ts):
        return _qsnr(orc, orc.Cfg(block=B, scale_fmt=fmt, rule=orc.NEAREST, tensor_scale=ts), x)[5]

    assert mse(orc.UE4M3, 8, orc.TS_NONE) > mse(orc.UE4M3, 16, orc.TS_NONE)
    assert mse(orc.UE5M3, 8, orc.TS_NONE) < mse(orc.UE5M3, 16, orc.TS_NONE)
    assert mse(orc.UE4M3, 8, orc.TS_COMPUTE) < mse(orc.UE4M3, 16, orc.TS_COMPUTE)


def _grid(elem):
    """Magnitude grids, built here from their definitions (independent of the
    oracle's tables): E2M1 as printed on the page, the others from their
    exponent / mantissa fields."""
    if elem == 0:
        return np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    if elem == 1:
        return np.array([0] + [2.0 ** (f - 3) for f in range(1, 8)], np.float64)
    if elem in (2, 3):
        mb, bias = (3, 1) if elem == 2 else (2, 3)
        out = []
        for c in range(32):
            e, m = c >> mb, c & ((1 << mb) - 1)
            out.append(m / 2.0 ** mb * 2.0 ** (1 - bias) if e == 0 else (1 + m / 2.0 ** mb) * 2.0 ** (e - bias))
        return np.array(out, np.float64)
    return np.arange(8, dtype=np.float64)


def _sse_nearest(v, grid):
    """Sum of (v - q)^2, q the nearest grid magnitude (ties to the even index,
    saturating), by brute force over the grid, accumulated in element order."""
    acc = 0.0
    for x in v:
        a = abs(float(x))
        d = np.abs(grid - a)
        best = np.flatnonzero(d == d.min())
        i = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
        if a >= grid[-1]:
            i = len(grid) - 1
        acc += (a - grid[i]) ** 2
    return acc


@pytest.mark.parametrize("elem", [0, 1, 2, 3, 4])
def test_mse_rule_brute_force(orc, elem):
    """MSE-optimal scale: the chosen E8M0 exponent is the one of k_floor,
    k_floor + 1 whose block squared error (in x units: 4^k sum) is smaller,
    ties to k_floor, checked against a brute-force grid rounding."""
    rng = np.random.default_rng(11 + elem)
    grid = _grid(elem)
    emax = {0: 2, 1: 4, 2: 2, 3: 4, 4: 2}[elem]
    x = (rng.standard_normal((64, 32)) * np.exp(rng.uniform(-3, 3, (64, 1)))).astype(np.float32)
    x[::7] *= 1.9                       # push some block maxima towards saturation
    r = orc.quantize(orc.Cfg(elem=elem, rule=orc.MSE), torch.from_numpy(x))
    for b in range(64):
        v = x[b]
        alpha = float(np.max(np.abs(v)))
        kf = math.frexp(alpha)[1] - 1 - emax
        sse = [_sse_nearest((v.astype(np.float32) * np.float32(2.0 ** -k)).astype(np.float32), grid)
               for k in (kf, kf + 1)]
        want = kf if sse[0] <= 4.0 * sse[1] else kf + 1
        assert int(r["scales"][b]) == want + 127, (b, sse)


def test_mse_rule_constant_blocks(orc):
    """Closed forms for E2M1 constant blocks: 7.0 and 5.0 tie (error 1 either
    way) and keep k_floor; 7.5 has error 1.5 at k_floor against 0.5 at
    k_floor + 1 (3.75 rounds to 4, i.e. 8)."""
    for val, k in ((7.0, 0), (5.0, 0), (7.5, 1), (6.0, 0)):
        x = torch.full((1, 32), val, dtype=torch.float32)
        r = orc.quantize(orc.Cfg(rule=orc.MSE), x)
        assert int(r["scales"][0]) == 127 + k, (val, r["scales"][0])


def _ue4m3_values():
    """UE4M3 values of codes 0..126 from the format's fields (bias 7, three
    mantissa bits, subnormals for exponent field 0)."""
    out = []
    for c in range(127):
        e, m = c >> 3, c & 7
        out.append(m / 8.0 * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7))
    return np.array(out, np.float64)


def _nearest_even_e2m1(v):
    grid = _grid(0)
    a = abs(float(v))
    if a >= 6.0:
        return math.copysign(6.0, v)
    d = np.abs(grid - a)
    best = np.flatnonzero(d == d.min())
    i = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
    return math.copysign(grid[i], v)


def _brute_force_ue_code(v, sT):
    """Argmin over every finite UE4M3 code of the block's squared error, with
    the element rule of the nearest formats, evaluated from the definitions
    (binary32 steps via numpy float32, binary64 sum in element order); ties
    keep the lower code."""
    f32 = np.float32
    best, bc = math.inf, 0
    for c, s in enumerate(_ue4m3_values()):
        s = f32(s)
        d = f32(s * f32(sT))
        with np.errstate(divide="ignore", over="ignore"):
            inv = f32(f32(1.0) / d)
        zero = s == 0 or not np.isfinite(inv)
        acc = 0.0
        for x in v:
            xh = f32(0.0)
            if not zero:
                q = f32(_nearest_even_e2m1(f32(f32(x) * inv)))
                xh = f32(f32(q * s) * f32(sT))
            e = float(x) - float(xh)
            acc += e * e
        if acc < best:
            best, bc = acc, c
    return bc


@pytest.mark.parametrize("sT", [1.0, 0.0123, 3.7e-4])
def test_mse_ue_group_step_brute_force(orc, sT):
    """MSE rule with UE4M3 scales and a given tensor scale: every block's code
    is the brute-force argmin over all 127 finite codes (checked here from
    the format's and the grid's definitions)."""
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((12, 32)) * np.exp(rng.uniform(-2, 2, (12, 1)))).astype(np.float32)
    x *= np.float32(sT * 200)
    x[3, :16] = 0.0                              # an all-zero block
    x[5, 3] *= 30                                # an outlier
    cfg = orc.Cfg(block=16, scale_fmt=orc.UE4M3, rule=orc.MSE, tensor_scale=orc.TS_GIVEN)
    r = orc.quantize(cfg, torch.from_numpy(x), tensor_scale=sT)
    for b in range(24):
        v = x.reshape(-1, 16)[b]
        assert int(r["scales"][b]) == _brute_force_ue_code(v, sT), b


def test_mse_ue_reproduces_single_values(orc):
    """Closed form: a block holding one value v = q s (q on the E2M1 grid, s a
    UE4M3 value) and zeros has a zero-error scale, so the MSE rule returns v
    exactly; the nearest rule, which maps the block max to 6, misses many."""
    vals = _ue4m3_values()[8::5]                 # normal scales across the range
    misses = 0
    for s in vals:
        for q in (0.5, 1.0, 1.5, 3.0, 4.0, 6.0):
            v = np.float32(q * s)
            x = np.zeros((1, 32), np.float32)
            x[0, 5] = v
            x[0, 20] = -v
            for rule in (orc.MSE, orc.NEAREST):
                cfg = orc.Cfg(block=16, scale_fmt=orc.UE4M3, rule=rule)
                r = orc.quantize(cfg, torch.from_numpy(x))
                xh = orc.dequantize(cfg, r["packed"], r["scales"], 1.0, None, None, 1, 32)
                if rule == orc.MSE:
                    assert np.array_equal(xh, x), (q, s)
                else:
                    misses += int(not np.array_equal(xh, x))
    assert misses > 0


def _block_sse(x, xh, B):
    d = x.astype(np.float64).reshape(-1, B) - xh.astype(np.float64).reshape(-1, B)
    return (d * d).sum(axis=1)


@pytest.mark.parametrize("B", [8, 16, 32])
def test_mse_ue_never_worse_than_nearest(orc, B):
    """Invariant: for the same tensor scale the MSE rule's block error is
    never above the nearest rule's, block by block."""
    from microscaling_block_quantization_b200 import inputs
    for x in (inputs.laplace_outlier_cols(64, 256, seed=4, n_outlier_cols=4),
              inputs.normal(64, 256, sigma=0.02, seed=7)):
        near = orc.Cfg(block=B, scale_fmt=orc.UE4M3, rule=orc.NEAREST, tensor_scale=orc.TS_COMPUTE)
        rn = orc.quantize(near, x)
        sT = rn["tensor_scale"]
        mse = orc.Cfg(block=B, scale_fmt=orc.UE4M3, rule=orc.MSE, tensor_scale=orc.TS_GIVEN)
        rm = orc.quantize(mse, x, tensor_scale=sT)
        xn = orc.dequantize(near, rn["packed"], rn["scales"], sT, None, None, 64, 256)
        xm = orc.dequantize(mse, rm["packed"], rm["scales"], sT, None, None, 64, 256)
        y = orc.input_f32(x)
        sn, sm = _block_sse(y, xn, B), _block_sse(y, xm, B)
        assert np.all(sm <= sn * (1 + 1e-12) + 1e-300)
        assert sm.sum() < sn.sum()


def test_mse_ue_alternation(orc):
    """Alternating optimisation of the global and group scales: the squared
    error after each group step does not rise (up to binary32 rounding of
    x_hat and s_T); every global step is the least-squares factor of the
    fixed element values u = q s_c (checked against numpy's sums, and as a
    minimum: moving s_T either way raises the fixed-u error); the quantizer
    with a computed tensor scale ends on the trace's last s_T."""
    from microscaling_block_quantization_b200 import inputs
    for x in (inputs.laplace_outlier_cols(128, 256, seed=4, n_outlier_cols=4),
              inputs.normal(128, 256, sigma=0.02, seed=7)):
        sfin, st, se = orc.mse_grid_trace(orc.UE4M3, 16, x, rounds=4)
        assert np.all(se[1:] <= se[:-1] * (1 + 1e-6))
        y = orc.input_f32(x).astype(np.float64)
        for i in range(4):
            cfg = orc.Cfg(block=16, scale_fmt=orc.UE4M3, rule=orc.MSE, tensor_scale=orc.TS_GIVEN)
            r = orc.quantize(cfg, x, tensor_scale=float(st[i]))
            # u = q s_c: the dequantized values with a unit tensor scale
            u = orc.dequantize(cfg, r["packed"], r["scales"], 1.0, None, None, 128, 256).astype(np.float64)
            s_ls = float((y * u).sum() / (u * u).sum())
            assert st[i + 1] == pytest.approx(s_ls, rel=1e-6)
            f = lambda s: float(((y - u * s) ** 2).sum())
            assert f(s_ls) <= min(f(s_ls * (1 + 1e-3)), f(s_ls * (1 - 1e-3)))
        cfg = orc.Cfg(block=16, scale_fmt=orc.UE4M3, rule=orc.MSE, tensor_scale=orc.TS_COMPUTE)
        r = orc.quantize(cfg, x)
        assert np.float32(r["tensor_scale"]) == np.float32(sfin) == st[-1]
        near = orc.Cfg(block=16, scale_fmt=orc.UE4M3, rule=orc.NEAREST, tensor_scale=orc.TS_COMPUTE)
        rn = orc.quantize(near, x)
        xn = orc.dequantize(near, rn["packed"], rn["scales"], rn["tensor_scale"], None, None, 128, 256)
        assert se[-1] < float(((y - xn) ** 2).sum())
