"""CPU pins of the oracle's number formats, rounding and scale rules.

Every check compares the oracle against something other than itself: values
printed on the pages (tests/golden/page_facts.txt), brute-force searches over
grids enumerated here from their plain description, closed forms, or
invariants of the rules.
"""
import math
import os
import struct
from fractions import Fraction

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def page_facts():
    facts = {}
    with open(os.path.join(GOLDEN, "page_facts.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            k, v = (s.strip() for s in line.split("=", 1))
            facts[k] = v
    return facts


def _num(s):
    if s.startswith("2^"):
        return 2.0 ** int(s[2:])
    return float(s)


def f32(x):
    return struct.unpack("<f", struct.pack("<f", x))[0]


# ---------------------------------------------------------------- E2M1 ----
def test_e2m1_grid_matches_page(orc):
    mags = [float(v) for v in page_facts()["e2m1_magnitudes"].split()]
    got = [orc.decode_elem(orc.E2M1, c) for c in range(8)]
    assert got == mags
    neg = [orc.decode_elem(orc.E2M1, 8 + c) for c in range(8)]
    assert neg == [-m for m in mags]
    assert math.copysign(1.0, neg[0]) == -1.0          # sign kept on zero
    nz = [m for m in mags if m > 0]
    assert max(nz) / min(nz) == float(page_facts()["e2m1_dynamic_range"])


def _nearest_even(grid, v):
    """Brute force: argmin |v - g| over the grid; ties -> even index."""
    best, bd = None, None
    for i, g in enumerate(grid):
        d = abs(Fraction(v) - Fraction(g))
        if bd is None or d < bd or (d == bd and i % 2 == 0):
            best, bd = i, d
    return best


def test_e2m1_rtne_ties_and_saturation(orc):
    ties = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for v, want in ties.items():
        assert orc.decode_elem(orc.E2M1, orc.encode_elem(orc.E2M1, v)) == want
        assert orc.decode_elem(orc.E2M1, orc.encode_elem(orc.E2M1, -v)) == -want
    for v in (6.0, 6.5, 7.9, 1e30, float("inf")):
        assert orc.decode_elem(orc.E2M1, orc.encode_elem(orc.E2M1, v)) == 6.0


def test_e2m1_rtne_brute_force_dense(orc):
    grid = [float(v) for v in page_facts()["e2m1_magnitudes"].split()]
    vals = [i / 256.0 for i in range(0, 6 * 256 + 1)]
    rng = np.random.default_rng(11)
    vals += [f32(v) for v in rng.uniform(0, 6, 2000)]
    for v in vals:
        code = orc.encode_elem(orc.E2M1, v)
        assert code == _nearest_even(grid, v), v


def test_e2m1_max_error_between_4_and_6(orc):
    want = float(page_facts()["e2m1_max_rel_error_4_6"])
    vs = np.linspace(4.0, 6.0, 4001)[1:-1].astype(np.float32)
    errs = [abs(orc.decode_elem(orc.E2M1, orc.encode_elem(orc.E2M1, float(v))) - v) / v for v in vs]
    assert max(errs) <= want + 1e-6
    assert max(errs) >= want - 1e-3
    assert abs(errs[int(np.argmin(abs(vs - 5.0)))] - want) < 1e-6     # at 5: |5-4|/5


# ------------------------------------------------------ other elements ----
def _fp_grid_from_description(steps_per_binade, lowest_binade, top):
    """Positive grid of a minifloat described as: `steps_per_binade` evenly
    spaced values in every binade [2^j, 2^(j+1)) from 2^lowest_binade up,
    the same spacing continuing down to 0 below it, capped at `top`."""
    g = set()
    step0 = Fraction(2) ** lowest_binade / steps_per_binade
    v = Fraction(0)
    while v < Fraction(2) ** lowest_binade:
        g.add(v)
        v += step0
    j = lowest_binade
    while True:
        step = Fraction(2) ** j / steps_per_binade
        v = Fraction(2) ** j
        while v < Fraction(2) ** (j + 1) and v <= top:
            g.add(v)
            v += step
        if Fraction(2) ** (j + 1) > top:
            break
        j += 1
    return sorted(float(x) for x in g)


@pytest.mark.parametrize("elem,grid", [
    ("E2M3", _fp_grid_from_description(8, 0, Fraction(15, 2))),   # 3 mantissa bits, max 7.5
    ("E3M2", _fp_grid_from_description(4, -2, Fraction(28))),      # 2 mantissa bits, max 28
    ("E3M0", [0.0] + [2.0 ** j for j in range(-2, 5)]),            # powers of two 1/4 .. 16
    ("INT4", [float(i) for i in range(8)]),
])
def test_other_grids_and_rtne(orc, elem, grid):
    e = getattr(orc, elem)
    nbits = 6 if elem in ("E2M3", "E3M2") else 4
    if elem == "INT4":
        got = [orc.decode_elem(e, c) for c in range(16)]
        assert sorted(set(got)) == [float(i) for i in range(-8, 8)]
        assert [orc.decode_elem(e, c) for c in range(8)] == grid
    else:
        got = [orc.decode_elem(e, c) for c in range(1 << (nbits - 1))]
        assert got == grid
    rng = np.random.default_rng(5)
    vals = [f32(v) for v in rng.uniform(0, grid[-1] * 1.1, 3000)]
    vals += [(a + b) / 2 for a, b in zip(grid[:-1], grid[1:])]      # every tie
    for v in vals:
        code = orc.encode_elem(e, v)
        want = _nearest_even(grid, v)
        if elem == "INT4":
            assert code == want, v
        else:
            assert code == want, (v, code, want)


@pytest.mark.parametrize("elem", ["E2M1", "E3M0", "E2M3", "E3M2"])
def test_ceil_rounding_is_next_grid_point(orc, elem):
    e = getattr(orc, elem)
    nb = 6 if elem in ("E2M3", "E3M2") else 4
    grid = [orc.decode_elem(e, c) for c in range(1 << (nb - 1))]
    rng = np.random.default_rng(3)
    for v in [f32(x) for x in rng.uniform(0, grid[-1], 2000)] + grid:
        got = orc.decode_elem(e, orc.encode_elem(e, v, mode=orc.RCEIL))
        want = min(g for g in grid if g >= v)
        assert got == want


# ------------------------------------------------------------ scales ----
def test_scale_format_extremes(orc):
    f = page_facts()
    assert orc.scale_decode(orc.UE4M3, 1) == _num(f["ue4m3_min_nonzero"])
    assert orc.scale_decode(orc.UE5M3, 1) == _num(f["ue5m3_min_nonzero"])
    assert min(orc.scale_decode(orc.UE4M3, c) for c in range(1, 0x7f)) == _num(f["ue4m3_min_nonzero"])
    assert min(orc.scale_decode(orc.UE5M3, c) for c in range(1, 0xff)) == _num(f["ue5m3_min_nonzero"])
    assert orc.scale_decode(orc.UE4M3, 0x7e) == 448.0
    assert math.isnan(orc.scale_decode(orc.UE4M3, 0x7f))
    assert math.isnan(orc.scale_decode(orc.UE5M3, 0xff))
    for c in range(255):
        assert orc.scale_decode(orc.E8M0, c) == 2.0 ** (c - 127)     # powers of two only
    assert math.isnan(orc.scale_decode(orc.E8M0, 0xff))


@pytest.mark.parametrize("fmt,top", [("UE4M3", 0x7e), ("UE5M3", 0xfe)])
def test_scale_codes_round_trip_and_nearest(orc, fmt, top):
    F = getattr(orc, fmt)
    vals = [orc.scale_decode(F, c) for c in range(top + 1)]
    assert all(b > a for a, b in zip(vals[:-1], vals[1:]))          # monotone
    for c in range(top + 1):
        assert orc.scale_encode_nearest(F, vals[c]) == c
    rng = np.random.default_rng(1)
    xs = [f32(v) for v in np.exp(rng.uniform(np.log(vals[1] / 4), np.log(vals[-1] * 2), 3000))]
    xs += [(a + b) / 2 for a, b in zip(vals[:-1], vals[1:])]
    arr = np.array(vals)
    for x in xs:
        code = orc.scale_encode_nearest(F, x)
        if x >= vals[-1]:
            assert code == top
            continue
        i = int(np.searchsorted(arr, x, side="right")) - 1
        lo, hi = i, min(i + 1, top)
        dlo, dhi = abs(x - vals[lo]), abs(vals[hi] - x)
        want = lo if dlo < dhi else hi if dhi < dlo else (lo if lo % 2 == 0 else hi)
        assert code == want, (x, code, want)


# ---------------------------------------------------------- philox ----
def test_philox_known_answers(orc):
    with open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")) as f:
        rows = [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]
    assert rows
    for r in rows:
        v = [int(t, 16) for t in r]
        assert orc.philox(v[0:4], v[4:6]) == v[6:10]


def test_fp6_tensor_core_layout(orc):
    """FP6 codes in the dense tensor-core operand form: 16 codes per 12
    bytes, code i at bits [6i, 6i + 6) of the little-endian 96-bit group,
    groups back to back (6 bits per element); checked against an integer
    construction, and the round trip."""
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 64, size=(4, 64), dtype=np.uint8)
    got = orc.pack_tc(2, codes)
    assert got.size == codes.size * 6 // 8
    got = got.reshape(-1, 12)
    flat = codes.reshape(-1, 16)
    for g in range(flat.shape[0]):
        v = 0
        for i in range(16):
            v |= int(flat[g, i]) << (6 * i)
        assert list(got[g]) == list(v.to_bytes(12, "little"))
    assert np.array_equal(orc.unpack_tc(3, orc.pack_tc(3, codes), 4, 64), codes)
    assert np.array_equal(orc.pack_tc(0, codes & 15), orc.pack(0, codes & 15))   # FP4 unchanged
