"""Seeded synthetic input tensors for the quantizer workloads.

This module holds no arithmetic of the quantization method: it only draws
random numbers with numpy's ``default_rng`` and casts them to the storage
dtype (float32 -> bfloat16 with round-to-nearest-even, done by torch's CPU
cast).  Both the CUDA path and the CPU oracle are fed the very same bytes
produced here.

The workloads stand in for the tensors the pages measure on (dumped
Llama-3.1-8B / Qwen3-8B activations and weights, LLaMA training gradients),
which are not available; their shapes and value distributions follow the
pages' descriptions:

* weight-like: i.i.d. normal with a small sigma (``Is Finer Better?``,
  research method: weights are close to N(0, sigma));
* activation-like: heavy-tailed Laplace with a few outlier channels
  (``Bridging the Gap ... Microscaling FP4``, section 2.1: raw activations
  are Laplace-like; ``Unveiling the Potential of Quantization with MXFP4``,
  Sec.3: systematic tensor outliers dominate the block maxima);
* gradient-like: tiny-sigma normal with 1% large entries (the fmread summary
  of Yang et al., design-choice study on gradient quantization).
"""
from __future__ import annotations

import numpy as np
import torch

__all__ = [
    "normal",
    "laplace_outlier_cols",
    "gradient_like",
    "to_bf16",
    "small_normal",
    "llama_linear",
]


def to_bf16(x32: np.ndarray) -> torch.Tensor:
    """float32 numpy array -> bfloat16 CPU tensor (RNE cast by torch)."""
    return torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32)).to(torch.bfloat16)


def small_normal(rows: int, cols: int, seed: int = 0, sigma: float = 1.0,
                 dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    """i.i.d. N(0, sigma) of the given shape (the 256x256 seed-0 case)."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols), dtype=np.float32) * np.float32(sigma)
    t = torch.from_numpy(x)
    return t.to(dtype) if dtype != torch.float32 else t


def normal(rows: int, cols: int, sigma: float, seed: int,
           dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    """Weight-like tensor: i.i.d. N(0, sigma)."""
    return small_normal(rows, cols, seed=seed, sigma=sigma, dtype=dtype)


def laplace_outlier_cols(rows: int, cols: int, seed: int, n_outlier_cols: int = 16,
                         outlier_gain: float = 50.0,
                         dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    """Activation-like tensor: i.i.d. Laplace(0, 1); ``n_outlier_cols`` columns
    drawn without replacement are multiplied by ``outlier_gain``."""
    rng = np.random.default_rng(seed)
    x = rng.laplace(0.0, 1.0, size=(rows, cols)).astype(np.float32)
    if n_outlier_cols > 0:
        cols_idx = rng.choice(cols, n_outlier_cols, replace=False)
        x[:, cols_idx] *= np.float32(outlier_gain)
    t = torch.from_numpy(x)
    return t.to(dtype) if dtype != torch.float32 else t


def gradient_like(rows: int, cols: int, seed: int, sigma: float = 1e-3,
                  frac_large: float = 0.01, gain: float = 20.0,
                  dtype: torch.dtype = torch.float32) -> torch.Tensor:
    """Gradient-like tensor: i.i.d. N(0, sigma) with a fraction of entries
    (chosen by ``rng.random() < frac_large``) multiplied by ``gain``."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols), dtype=np.float32) * np.float32(sigma)
    mask = rng.random((rows, cols)) < frac_large
    x[mask] *= np.float32(gain)
    t = torch.from_numpy(x)
    return t.to(dtype) if dtype != torch.float32 else t


def llama_linear(m: int = 8192, k: int = 4096, n: int = 14336,
                 seed_a: int = 6, seed_w: int = 7):
    """Llama-3-8B-shaped linear layer operands.

    A: [m, k] bf16 activations, Laplace(0, 1).
    W: [n, k] bf16 weights, N(0, 0.02), stored out-features x in-features so
    that both operands are contiguous along the reduction dimension k; the
    product is A @ W^T.
    """
    rng = np.random.default_rng(seed_a)
    a = rng.laplace(0.0, 1.0, size=(m, k)).astype(np.float32)
    rng = np.random.default_rng(seed_w)
    w = rng.standard_normal((n, k), dtype=np.float32) * np.float32(0.02)
    return to_bf16(a), to_bf16(w)
