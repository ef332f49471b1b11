"""Seeded synthetic inputs (weights and activations) for tests, smoke check and benchmark.

This module only draws random numbers; it holds none of the quantization or
GEMV arithmetic and imports neither the CUDA library nor the oracle, so both
sides of every parity check consume the same inputs from here.

Distributions (stand-ins for the trained Llama / Gemma weights the pages
evaluate on, which are not available):
  * ``outlier_normal``: W ~ N(0, 0.02^2) with a Bernoulli(0.01) mask of entries
    multiplied by 10 (tiny INT4 parity case).
  * ``llama_like``: W = 0.02 * t5 * exp(0.5 * Z_row): Student-t with 5 degrees
    of freedom (t5 = Z / sqrt(chi2_5 / 5)) times a per-row lognormal(0, 0.5)
    scale.
  * activations: x ~ N(0, 1), rounded to fp16 or bf16 by the consumer.
Host generators use numpy's Philox bit generator; device generators (used for
matrices too large to draw on the host in seconds) use torch's CUDA generator.
"""
from __future__ import annotations

import numpy as np


def _rng(seed: int, stream: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(key=[seed, stream]))


def outlier_normal(N: int, K: int, seed: int = 0, stream: int = 0) -> np.ndarray:
    rng = _rng(seed, stream)
    W = rng.normal(0.0, 0.02, size=(N, K))
    mask = rng.random(size=(N, K)) < 0.01
    W[mask] *= 10.0
    return W.astype(np.float32)


def llama_like(N: int, K: int, seed: int = 1, stream: int = 0) -> np.ndarray:
    rng = _rng(seed, stream)
    z = rng.normal(size=(N, K))
    chi2 = rng.chisquare(5.0, size=(N, K))
    t5 = z / np.sqrt(chi2 / 5.0)
    row = np.exp(0.5 * rng.normal(size=(N, 1)))
    return (0.02 * t5 * row).astype(np.float32)


def activations(M: int, K: int, seed: int = 0, stream: int = 1) -> np.ndarray:
    """x ~ N(0, 1) as binary32 [M, K]; the caller rounds to fp16 / bf16."""
    return _rng(seed, stream).normal(size=(M, K)).astype(np.float32)


def llama_like_device(N: int, K: int, seed: int, device="cuda"):
    """Same distribution as ``llama_like`` drawn on the GPU with torch (fp32)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    W = torch.empty((N, K), dtype=torch.float32, device=device)
    W.normal_(generator=g)
    chi2 = torch.zeros_like(W)
    tmp = torch.empty_like(W)
    for _ in range(5):
        tmp.normal_(generator=g)
        chi2.addcmul_(tmp, tmp)
    del tmp
    W.div_(torch.sqrt(chi2.div_(5.0)))
    del chi2
    row = torch.empty((N, 1), dtype=torch.float32, device=device).normal_(generator=g).mul_(0.5).exp_()
    W.mul_(row).mul_(0.02)
    return W


def activations_device(M: int, K: int, seed: int, dtype, device="cuda"):
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return torch.empty((M, K), dtype=torch.float32, device=device).normal_(generator=g).to(dtype)
