"""Expected quantization MSE of N(0, sigma^2) blocks: the theoretical model
of "Is Finer Better? The Limits of Microscaling Formats in LLMs" (Theoretical
framework), written out here from first principles.

TEST INFRASTRUCTURE: imported only by the tests (a trend validator for the
quantizers' measured MSE); nothing in the library uses it.

The page splits the MSE of a block-scaled FP4 tensor into three parts (the
non-maximum elements, the block maximum itself once the scale is quantized,
and the zero-rounding error of blocks whose maximum falls below the smallest
scale) and fits measured MSE-vs-sigma curves with it, but prints no formula.
PARITY UNPINNED against the page for that reason; what pins this code is the
oracle's own measured MSE on seeded samples (tests), within sampling error.

Model, for one block of B i.i.d. N(0, sigma^2) values with no rounding of the
inputs: M = max |x_i| has density f_M(m) = B g(m) G(m)^(B-1), g and G the
half-normal density and distribution.  The scale is the nearest value s(m) of
the scale format to m / (max_elem s_T) (saturating at the format's largest
value; 0 below half its smallest one), d = s(m) s_T, and an element x
becomes d Q(x / d) with Q the nearest E2M1 value (saturating at 6); with
d = 0 the block is zero.  Given M = m the other B - 1 magnitudes are i.i.d.
half-normal conditioned on |x| < m, so with e(x; d) = x - d Q(x / d)

  E[SSE] = int f_M(m) e(m; d(m))^2 dm                            (maximum)
         + int B (B - 1) g(m) G(m)^(B-2) int_0^m e(x; d(m))^2 g(x) dx dm
                                                                 (the others)

and the zero-rounding part is the piece of both integrals where d(m) = 0.
The MSE per element is E[SSE] / B.  Integrals: trapezoid rule on a fine grid.
"""
from __future__ import annotations

import numpy as np
from scipy.stats import norm

E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def scale_values(fmt: str) -> np.ndarray:
    """Finite non-negative values of an 8-bit unsigned scale format with three
    mantissa bits: UE4M3 (bias 7) or UE5M3 (bias 15); the all-ones code is
    NaN."""
    ebits, bias = {"ue4m3": (4, 7), "ue5m3": (5, 15)}[fmt]
    out = []
    for c in range((1 << (ebits + 3)) - 1):
        e, m = c >> 3, c & 7
        out.append(m / 8 * 2.0 ** (1 - bias) if e == 0 else (1 + m / 8) * 2.0 ** (e - bias))
    return np.array(out)


def _nearest(values: np.ndarray, t: np.ndarray) -> np.ndarray:
    """Nearest entry of the ascending array `values` to each t (saturating)."""
    i = np.clip(np.searchsorted(values, t), 1, len(values) - 1)
    lo, hi = values[i - 1], values[i]
    return np.where(t - lo <= hi - t, lo, hi)


def _elem_error2(x: np.ndarray, d: float) -> np.ndarray:
    if d == 0.0:
        return x * x
    q = _nearest(E2M1, np.minimum(x / d, 6.0))
    e = x - d * q
    return e * e


def expected_mse(sigma: float, block: int, fmt: str = "ue4m3", tensor_scale: float = 1.0,
                 n_grid: int = 20000) -> dict:
    """Expected per-element MSE of nearest-scale E2M1 block quantization of
    N(0, sigma^2) data, and its three parts."""
    sv = scale_values(fmt)
    hi = sigma * (np.sqrt(2 * np.log(max(block, 2))) + 8.0)
    m = np.linspace(0.0, hi, n_grid)
    g = 2.0 * norm.pdf(m, scale=sigma)
    G = 2.0 * norm.cdf(m, scale=sigma) - 1.0
    s = _nearest(sv, m / (6.0 * tensor_scale))
    d = s * tensor_scale
    # e(m; d(m))^2 of the maximum and int_0^m e(x; d(m))^2 g(x) dx, grouped
    # by the (piecewise constant) scale
    emax2 = np.zeros_like(m)
    inner = np.zeros_like(m)
    for dv in np.unique(d):
        sel = d == dv
        emax2[sel] = _elem_error2(m[sel], dv)
        cum = np.concatenate([[0.0], np.cumsum(0.5 * (_elem_error2(m[1:], dv) * g[1:] +
                                                      _elem_error2(m[:-1], dv) * g[:-1]) * np.diff(m))])
        inner[sel] = cum[sel]
    f_max = block * g * G ** (block - 1)
    f_rest = block * (block - 1) * g * G ** (block - 2) if block > 1 else np.zeros_like(m)
    zero = d == 0.0
    part_max = np.trapezoid(f_max * emax2, m)
    part_rest = np.trapezoid(f_rest * inner, m)
    part_zero = np.trapezoid(np.where(zero, f_max * emax2 + f_rest * inner, 0.0), m)
    return {"mse": (part_max + part_rest) / block, "max": np.trapezoid(np.where(zero, 0, f_max * emax2), m) / block,
            "others": np.trapezoid(np.where(zero, 0, f_rest * inner), m) / block, "zero": part_zero / block}
