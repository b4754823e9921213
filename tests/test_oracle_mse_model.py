"""The expected-MSE model of N(0, sigma^2) blocks ("Is Finer Better? The
Limits of Microscaling Formats in LLMs", theoretical framework; the page
prints no formula, so the model is derived in oracle/mse_model.py and pinned
here to the oracle's measured MSE on seeded samples, within sampling error,
and to its closed forms)."""
import numpy as np
import pytest
import torch

from microscaling_block_quantization_b200 import inputs
from oracle import mse_model


@pytest.mark.parametrize("sigma,block,fmt", [(0.002, 8, "ue4m3"), (0.002, 16, "ue4m3"), (0.02, 16, "ue4m3"),
                                             (1.0, 32, "ue4m3"), (0.002, 8, "ue5m3"), (0.3, 64, "ue5m3")])
def test_model_matches_measured_mse(orc, sigma, block, fmt):
    r = mse_model.expected_mse(sigma, block, fmt)
    x = inputs.normal(256, 4096, sigma=sigma, seed=2, dtype=torch.float32)
    c = orc.Cfg(block=block, scale_fmt=orc.UE4M3 if fmt == "ue4m3" else orc.UE5M3, rule=orc.NEAREST)
    q = orc.quantize(c, x)
    xh = orc.dequantize(c, q["packed"], q["scales"], 1.0, None, None, 256, 4096)
    e2 = (x.numpy().astype(np.float64) - xh) ** 2
    se = e2.std() / np.sqrt(e2.size)
    assert abs(e2.mean() - r["mse"]) <= 4 * se + 1e-3 * r["mse"], (e2.mean(), r["mse"], se)


def test_model_closed_forms():
    # every block below half the smallest UE4M3 scale: all zero, MSE = sigma^2
    r = mse_model.expected_mse(1e-4, 16, "ue4m3")
    assert r["mse"] == pytest.approx(1e-8, rel=1e-6)
    assert r["zero"] == pytest.approx(r["mse"], rel=1e-9)
    # UE5M3 in its normal range: the error scales with sigma^2 (power-of-two
    # sigma steps move every scale by an exact power of two)
    a, b = mse_model.expected_mse(0.25, 16, "ue5m3"), mse_model.expected_mse(1.0, 16, "ue5m3")
    assert b["mse"] == pytest.approx(16 * a["mse"], rel=1e-6)
    assert a["zero"] < 1e-12 * a["mse"]
    # the three parts add up
    r = mse_model.expected_mse(0.002, 8, "ue4m3")
    assert r["max"] + r["others"] + r["zero"] == pytest.approx(r["mse"], rel=1e-9)


def test_model_inversion_trend():
    """The page's finding: with UE4M3 scales and no tensor scale, narrow
    distributions get a larger MSE from smaller blocks (zero-rounding of
    blocks below the smallest scale, 2^-9); wider ones do not, and UE5M3
    (smallest scale 2^-17) removes the inversion."""
    m = lambda s, b, f: mse_model.expected_mse(s, b, f)["mse"]
    assert m(0.002, 8, "ue4m3") > m(0.002, 16, "ue4m3") > m(0.002, 32, "ue4m3")
    assert m(0.02, 8, "ue4m3") < m(0.02, 16, "ue4m3") < m(0.02, 32, "ue4m3")
    assert m(0.002, 8, "ue5m3") < m(0.002, 16, "ue5m3") < m(0.002, 32, "ue5m3")
