"""Seeded synthetic inputs for the W4A16 group-128 linear layer.

This module only draws random inputs.  It holds none of the layer's arithmetic
(no dequantisation, no product, no packing), so both the CPU oracle's tests and
the CUDA path can take their inputs from here without sharing any code.

Canonical (unpacked) arrays, the form every caller starts from:

* ``q``      uint8  [M, K]        integer weight codes, uniform in 0..15
* ``zeros``  uint8  [M, K/G]      one unsigned 4-bit zero point per group
* ``scales`` uint16 [M, K/G]      fp16 bit patterns, one scale per group
* ``x``      uint16 [N, K]        fp16 bit patterns, activations, token-major

Value distributions follow the workloads of the AWQ int4 / group-128 setting
described in "PerfXLLM on Snapdragon 8 Gen2" (section 3.1, low-precision
quantisation): codes and zeros uniform over the 16 values of a uint4, scales
uniform in [0.001, 0.02] rounded once to fp16, activations N(0, 1) rounded once
to fp16.  The optional activation-outlier channels (a fixed 1 % of the K
channels, shared by every token, scaled by 20 in fp32 before the single fp16
rounding) model the prefill inputs.

Draw order from one ``numpy.random.default_rng(seed)`` stream:
q, zeros, scales, x, outlier channel indices.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

GROUP = 128
SCALE_LO = 0.001
SCALE_HI = 0.02
OUTLIER_GAIN = 20.0


@dataclass
class Problem:
    """One synthetic W4A16 problem in canonical form."""

    q: np.ndarray        # uint8  [M, K]
    zeros: np.ndarray    # uint8  [M, K/G]
    scales: np.ndarray   # uint16 [M, K/G]  (fp16 bits)
    x: np.ndarray        # uint16 [N, K]    (fp16 bits)
    group: int
    outliers: np.ndarray  # int64 indices of the scaled activation channels

    @property
    def M(self) -> int:
        return int(self.q.shape[0])

    @property
    def K(self) -> int:
        return int(self.q.shape[1])

    @property
    def N(self) -> int:
        return int(self.x.shape[0])


def _fp16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32/float64 values once to fp16 and return the bit patterns."""
    return np.ascontiguousarray(a.astype(np.float16)).view(np.uint16)


def draw_weights(rng: np.random.Generator, M: int, K: int, group: int = GROUP):
    """Draw (q, zeros, scales) for an M x K weight, in that order."""
    if K % group:
        raise ValueError(f"K={K} is not a multiple of group={group}")
    kg = K // group
    q = rng.integers(0, 16, size=(M, K), dtype=np.uint8)
    zeros = rng.integers(0, 16, size=(M, kg), dtype=np.uint8)
    scales = _fp16_bits(rng.uniform(SCALE_LO, SCALE_HI, size=(M, kg)))
    return q, zeros, scales


def draw_activations(rng: np.random.Generator, N: int, K: int,
                     outlier_frac: float = 0.0):
    """Draw fp16 activations [N, K]; optionally scale a fixed set of channels."""
    x = rng.standard_normal(size=(N, K), dtype=np.float32)
    n_out = int(round(outlier_frac * K))
    idx = np.sort(rng.choice(K, size=n_out, replace=False)) if n_out else \
        np.zeros(0, dtype=np.int64)
    if n_out:
        x[:, idx] *= np.float32(OUTLIER_GAIN)
    return _fp16_bits(x), idx.astype(np.int64)


def make_problem(M: int, K: int, N: int, group: int = GROUP, seed: int = 0,
                 outlier_frac: float = 0.0) -> Problem:
    """The seeded problem used by tests and the benchmark."""
    rng = np.random.default_rng(seed)
    q, zeros, scales = draw_weights(rng, M, K, group)
    x, idx = draw_activations(rng, N, K, outlier_frac)
    return Problem(q=q, zeros=zeros, scales=scales, x=x, group=group,
                   outliers=idx)


def make_weights_torch(M: int, K: int, group: int, generator, device):
    """Fast on-device draw of canonical weights with the same distributions.

    Used where many large distinct weight sets are needed (a multi-layer
    decode step).  Returns torch tensors (q uint8, zeros uint8, scales fp16).
    """
    import torch

    kg = K // group
    q = torch.randint(0, 16, (M, K), dtype=torch.uint8, device=device,
                      generator=generator)
    zeros = torch.randint(0, 16, (M, kg), dtype=torch.uint8, device=device,
                          generator=generator)
    scales = (torch.rand((M, kg), dtype=torch.float64, device=device,
                         generator=generator) * (SCALE_HI - SCALE_LO)
              + SCALE_LO).to(torch.float16)
    return q, zeros, scales


def make_activations_torch(N: int, K: int, generator, device):
    """Fast on-device draw of fp16 N(0,1) activations [N, K]."""
    import torch

    return torch.randn((N, K), dtype=torch.float32, device=device,
                       generator=generator).to(torch.float16)
