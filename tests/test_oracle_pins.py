"""Pins of the oracle's block walks, offsets, nearest scales and inverse
rotation against definitions written out here independently (numpy, the
formats' field definitions, scipy's Hadamard matrix), so that a transposed
walk, a wrong offset formula, a truncation in place of a rounding or a
misordered rotation fails a test.

Sources: "Unveiling the Potential of Quantization with MXFP4" (Sec.2 the
E2M1 grid and E8M0 floor scale, Sec.3 the flush-to-zero share and its drop
from block 32 to 16, Sec.4 NVFP4's UE4M3 block scales); "Is Finer Better?"
(UE4M3 / UE5M3 scales with an FP32 tensor scale); the fmread summary of
Yang et al. (row-wise, column-wise and 2D blocks; asymmetric scaling);
"Bridging the Gap ... Microscaling FP4" (sec. 2.1: block Hadamard rotation).
"""
import math

import numpy as np
import pytest
import scipy.linalg
import torch

from microscaling_block_quantization_b200 import inputs

E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


def _rne_e2m1_codes(v):
    """Sign-magnitude E2M1 codes of binary32 values: nearest grid point, ties
    to the even magnitude code, saturating at 6, the sign bit kept."""
    v = np.asarray(v, np.float32)
    a = np.abs(v.astype(np.float64))
    d = np.abs(a[..., None] - E2M1)
    best = np.argmin(d, axis=-1)
    srt = np.sort(d, axis=-1)
    tie = srt[..., 0] == srt[..., 1]
    best = np.where(tie & (best % 2 == 1), best + 1, best)
    best = np.where(a >= 6.0, 7, best)
    return (best | (np.signbit(v).astype(np.int64) << 3)).astype(np.uint8)


def _f32(x):
    return np.asarray(x, np.float32)


def _bf16_rne(v32):
    return torch.from_numpy(np.ascontiguousarray(_f32(v32))).to(torch.bfloat16).float().numpy()


def _bf16_trunc(v32):
    b = np.ascontiguousarray(_f32(v32)).view(np.uint32) & np.uint32(0xFFFF0000)
    return b.view(np.float32)


# ---------------------------------------------------------------- axes -----
@pytest.mark.parametrize("variant", ["b8", "b16", "b32", "ceil", "oas", "mbs", "asym_e2m1",
                                     "asym_int4", "e3m2", "nvfp4", "ue5m3", "had16", "had32"])
def test_column_blocks_are_row_blocks_of_the_transpose(orc, variant):
    """A column-wise B x 1 block of x is the row-wise 1 x B block of x^T:
    codes, scales, macro scales, offsets, tensor scale and the rotated tensor
    of (COL, x) are those of (ROW, x^T), transposed back."""
    kw = dict(block=32)
    kw.update({"b8": dict(block=8), "b16": dict(block=16), "b32": {}, "ceil": dict(rule=orc.CEIL),
               "oas": dict(rule=orc.OAS, oas_tau=7.0), "mbs": dict(macro_block=128),
               "asym_e2m1": dict(asymmetric=1), "asym_int4": dict(elem=orc.INT4, asymmetric=1, rule=orc.CEIL),
               "e3m2": dict(elem=orc.E3M2),
               "nvfp4": dict(block=16, scale_fmt=orc.UE4M3, rule=orc.NEAREST, tensor_scale=orc.TS_COMPUTE),
               "ue5m3": dict(block=8, scale_fmt=orc.UE5M3, rule=orc.NEAREST),
               "had16": dict(hadamard=16), "had32": dict(hadamard=32)}[variant])
    x = inputs.laplace_outlier_cols(256, 384, seed=4, n_outlier_cols=6, dtype=torch.float32).numpy()
    x[:, 5] -= 3.0                                   # one-sided columns for the offsets
    rows, cols = x.shape
    col = orc.quantize(orc.Cfg(axis=orc.COL, **kw), torch.from_numpy(x))
    row = orc.quantize(orc.Cfg(axis=orc.ROW, **kw), torch.from_numpy(np.ascontiguousarray(x.T)))
    B = kw["block"]
    assert np.array_equal(col["codes"], row["codes"].T)
    assert np.array_equal(col["scales"].reshape(rows // B, cols), row["scales"].reshape(cols, rows // B).T)
    assert np.array_equal(col["offsets"].reshape(rows // B, cols), row["offsets"].reshape(cols, rows // B).T)
    if kw.get("macro_block"):
        assert np.array_equal(col["macro"].reshape(rows // 128, cols), row["macro"].reshape(cols, rows // 128).T)
    assert col["tensor_scale"] == row["tensor_scale"]
    assert np.array_equal(col["y"], row["y"].T)
    if variant in ("asym_e2m1", "b32"):
        assert len(set(col["scales"].tolist())) > 3       # the blocks really differ


def test_2d_blocks_follow_the_floor_rule_on_tile_amax(orc):
    """2D 32 x 32 tiles: the E8M0 scale of tile (i, j) is 2^(floor(log2 amax) - 2)
    of numpy's absmax over rows 32i.. and columns 32j.., scales laid out
    [rows/32][cols/32]; every code is the nearest-even E2M1 code of x / 2^k."""
    x = inputs.laplace_outlier_cols(96, 160, seed=4, n_outlier_cols=3).float().numpy()
    x[32:64, 64:96] = 0.0                          # an all-zero tile
    x[0:32, 128:160] *= 1e-30                      # exponents far below the others
    r = orc.quantize(orc.Cfg(axis=orc.TWO_D), torch.from_numpy(x))
    tiles = np.abs(x).reshape(3, 32, 5, 32).max(axis=(1, 3))
    m, e = np.frexp(tiles.astype(np.float64))
    k = np.clip(e - 1 - 2, -127, 127)
    want = np.where(tiles == 0, 0, k + 127).astype(np.uint8)
    assert np.array_equal(r["scales"].reshape(3, 5), want)
    kk = np.repeat(np.repeat(k, 32, axis=0), 32, axis=1)
    v = _f32(x * np.exp2(-kk.astype(np.float64)))
    zero = np.repeat(np.repeat(tiles == 0, 32, axis=0), 32, axis=1)
    codes = np.where(zero, 0, _rne_e2m1_codes(v))
    assert np.array_equal(r["codes"], codes)


# ---------------------------------------------------------- E2M1 offset ----
def test_e2m1_asymmetric_offset_closed_form(orc):
    """E2M1 asymmetric blocks: the offset is bf16_rne((max + min) / 2) with the
    sum and the halving in binary32.  Two-valued blocks whose midpoint is not
    a bf16 value separate round-to-nearest-even from truncation and from
    (max - min) / 2; constant blocks have offset = the value and zero codes."""
    rng = np.random.default_rng(11)
    hi = _bf16_rne(rng.uniform(0.5, 4.0, 64))
    lo = _bf16_rne(hi - rng.uniform(0.01, 3.0, 64))
    x = np.zeros((64, 32), np.float32)
    x[:, ::2] = hi[:, None]
    x[:, 1::2] = lo[:, None]
    x[60:] = hi[60:, None]                                  # constant blocks
    xb = torch.from_numpy(x).to(torch.bfloat16)
    xf = xb.float().numpy()
    r = orc.quantize(orc.Cfg(asymmetric=1), xb)
    mx, mn = xf.max(axis=1), xf.min(axis=1)
    mid = _f32(_f32(mx + mn) * np.float32(0.5))
    want = _bf16_rne(mid)
    got = orc.bf16_bits_to_f32(r["offsets"])
    assert np.array_equal(got, want)
    assert (_bf16_trunc(mid) != want).sum() >= 8            # truncation would fail here
    assert not np.array_equal(got, _bf16_rne(_f32(mx - mn) * np.float32(0.5)))
    # the symmetric rule on the residuals r = x - o
    res = _f32(xf - got[:, None])
    amax = np.abs(res).max(axis=1)
    for b in range(64):
        if amax[b] == 0:
            assert int(r["scales"][b]) == 0 and not r["codes"][b].any()
            continue
        k = int(np.frexp(np.float64(amax[b]))[1]) - 1 - 2
        assert int(r["scales"][b]) == k + 127
        assert np.array_equal(r["codes"][b], _rne_e2m1_codes(_f32(res[b] * np.float32(2.0 ** -k))))
    xh = orc.dequantize(orc.Cfg(asymmetric=1), r["packed"], r["scales"], None, None, r["offsets"], 64, 32)
    assert np.array_equal(xh[60:], xf[60:])                 # constant blocks come back exactly


# --------------------------------------------------- nearest UE scales ----
def _ue_values(fmt):
    """Values of the finite codes of UE4M3 (bias 7) or UE5M3 (bias 15) from
    the fields: three mantissa bits, subnormals for exponent field 0, the
    all-ones code NaN."""
    bias, top = (7, 0x7E) if fmt == 1 else (15, 0xFE)
    vals = []
    for c in range(top + 1):
        e, m = c >> 3, c & 7
        vals.append(m / 8.0 * 2.0 ** (1 - bias) if e == 0 else (1 + m / 8.0) * 2.0 ** (e - bias))
    return np.array(vals, np.float64)


def _nearest_even_code(vals, s):
    """Code of the nearest value to s >= 0, ties to the even code, saturating."""
    if s >= vals[-1]:
        return len(vals) - 1
    d = np.abs(vals - float(s))
    best = np.flatnonzero(d == d.min())
    return int(best[0]) if len(best) == 1 else int([b for b in best if b % 2 == 0][0])


@pytest.mark.parametrize("fmt,ts,B", [(1, 1, 16), (1, 0, 16), (2, 0, 16), (2, 1, 32), (1, 1, 8)])
def test_nearest_block_scale_per_block_brute_force(orc, fmt, ts, B):
    """Every block's UE scale is the nearest-even format value of
    RN(RN(amax / 6) / s_T) (two binary32 quotients), saturating at the top
    code; the codes are the nearest-even E2M1 codes of x * RN(1 / RN(s_b s_T)),
    a block whose scale is zero stays all zero."""
    rng = np.random.default_rng(3)
    rows, cols = 48, 256
    mag = np.exp(rng.uniform(-14, 6, (rows, cols // B, 1)))
    x = _f32((rng.laplace(size=(rows, cols // B, B)) * mag).reshape(rows, cols))
    x[7, :B] = 0.0
    xb = torch.from_numpy(x).to(torch.bfloat16)
    xf = xb.float().numpy()
    cfg = orc.Cfg(block=B, scale_fmt=fmt, rule=orc.NEAREST, tensor_scale=orc.TS_COMPUTE if ts else orc.TS_NONE)
    r = orc.quantize(cfg, xb)
    vals = _ue_values(fmt)
    sT = np.float32(r["tensor_scale"]) if ts else np.float32(1.0)
    if ts:
        top = 448.0 if fmt == 1 else 1.75 * 2.0 ** 16
        assert sT == _f32(_f32(np.abs(xf).max()) / _f32(6.0 * top))
    blocks = xf.reshape(-1, B)
    codes = r["codes"].reshape(-1, B)
    n_zero = 0
    for b in range(blocks.shape[0]):
        amax = np.float32(np.abs(blocks[b]).max())
        s_real = _f32(_f32(amax / np.float32(6.0)) / sT)
        c = _nearest_even_code(vals, s_real)
        assert int(r["scales"][b]) == c, (b, amax, s_real)
        sb = np.float32(vals[c])
        if sb == 0:
            n_zero += 1
            assert not codes[b].any()
            continue
        inv = _f32(np.float32(1.0) / _f32(sb * sT))
        assert np.array_equal(codes[b], _rne_e2m1_codes(_f32(blocks[b] * inv))), b
    if fmt == 1 and not ts:
        assert n_zero > 0            # the small blocks' scales round to zero without s_T


# ------------------------------------------------------ inverse rotation ----
@pytest.mark.parametrize("axis,n", [(0, 16), (0, 32), (1, 16), (1, 32), (2, 32), (2, 16)])
def test_unrotate_is_the_normalised_hadamard(orc, axis, n):
    """x_hat in the input space is the rotated-domain x_hat times H_n / sqrt(n)
    (scipy's Sylvester matrix) over each group of n along the block axis (the
    row direction for 2D): within binary32 butterfly rounding."""
    x = inputs.laplace_outlier_cols(64, 128, seed=4, n_outlier_cols=2).float()
    cfg = orc.Cfg(axis=axis, block=32, hadamard=n)
    r = orc.quantize(cfg, x)
    rot = orc.dequantize(cfg, r["packed"], r["scales"], None, None, None, 64, 128, unrotate=False)
    back = orc.dequantize(cfg, r["packed"], r["scales"], None, None, None, 64, 128, unrotate=True)
    H = scipy.linalg.hadamard(n).astype(np.float64) / math.sqrt(n)
    z = rot.astype(np.float64)
    if axis == 1:
        z = z.T
    want = (z.reshape(z.shape[0], -1, n) @ H).reshape(z.shape)
    if axis == 1:
        want = want.T
    assert np.abs(back - want).max() <= 1e-6 * np.abs(want).max()
    # and it inverts the forward rotation on an exact round trip
    yy = r["y"].astype(np.float64)
    if axis == 1:
        yy = yy.T
    fwd = (yy.reshape(yy.shape[0], -1, n) @ H).reshape(yy.shape)
    xin = x.numpy().astype(np.float64)
    assert np.abs((fwd.T if axis == 1 else fwd) - xin).max() <= 1e-5 * np.abs(xin).max()


# ------------------------------------------------------- flush to zero -----
def test_flush_to_zero_share_falls_from_block_32_to_16(orc):
    """Activation-like tensors (Laplace with outlier channels): the share of
    nonzero elements flushed to zero by MXFP4 falls when the block shrinks
    from 32 to 16 ("Unveiling ...", Sec.3: about 20% to 13% on real
    activations); here about 23% to 17%, counted by brute force."""
    x = inputs.laplace_outlier_cols(1024, 4096, seed=4)
    xf = x.float().numpy()
    share = {}
    for B in (32, 16):
        r = orc.quantize(orc.Cfg(block=B), x)
        xh = orc.dequantize(orc.Cfg(block=B), r["packed"], r["scales"], None, None, None, 1024, 4096)
        st, _ = orc.stats(r["y"], xh)
        nz = xf != 0
        share[B] = float(((xh == 0) & nz).sum() / nz.sum())
        assert st[9] == pytest.approx(share[B], abs=1e-12)
    assert 0.12 < share[32] < 0.35
    assert share[16] < 0.85 * share[32]
