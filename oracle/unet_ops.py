"""fp64 CPU oracles for the two specialised UNet kernels beside attention.

TEST INFRASTRUCTURE ONLY: the tests and the benchmark's checks call these;
the CUDA product path never imports them.  They share no code with the CUDA
library.

"Speed Is All You Need: On-Device Acceleration of Large Diffusion Models via
GPU-Aware Optimizations" (news summary, section on the three optimisations,
the specialised-kernels paragraphs) names two kernels besides attention:

* group normalisation, used throughout the UNet: the channels of a feature
  map are divided into groups and each group is normalised on its own; the
  paper runs it as one GPU command with no intermediate tensor;
* the GELU activation (the Gaussian error function and the arithmetic around
  it) fused with the split and multiplication that accompany it in the UNet's
  feed-forward layers (the gated form: the projection's output is split in two
  halves h and g, and the result is h * GELU(g)).

Readings of what the page leaves open:

* GroupNorm statistics are the mean and the biased (population) variance of
  each group's C/G channels x H x W values; y = (x - mean) / sqrt(var + eps)
  * gamma_c + beta_c with per-channel gamma, beta; eps is the caller's
  (1e-6 in SD's UNet).
* GELU is the exact form GELU(x) = x/2 (1 + erf(x / sqrt(2))) (the page names
  the Gaussian error function); the split takes the first half of the last
  dimension as h and the second as the gate g.
"""
from __future__ import annotations

import numpy as np
from scipy.special import erf


def group_norm(x, gamma, beta, groups: int, eps: float):
    """GroupNorm in fp64.  x [B, C, H, W] (or [B, C, HW]); gamma, beta [C]."""
    x = np.asarray(x, dtype=np.float64)
    B, C = x.shape[:2]
    if C % groups:
        raise ValueError("C must be a multiple of the group count")
    xg = x.reshape(B, groups, -1)                       # a group: C/G channels x spatial, contiguous
    mean = xg.mean(axis=2, keepdims=True)
    var = ((xg - mean) ** 2).mean(axis=2, keepdims=True)
    xhat = ((xg - mean) / np.sqrt(var + eps)).reshape(x.shape)
    shape = (1, C) + (1,) * (x.ndim - 2)
    return (xhat * np.asarray(gamma, np.float64).reshape(shape) + np.asarray(beta, np.float64).reshape(shape))


def gelu(x):
    """Exact GELU in fp64: x/2 (1 + erf(x / sqrt(2)))."""
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + erf(x / np.sqrt(2.0)))


def geglu(x):
    """The gated feed-forward activation: x [..., 2F] -> h * GELU(g), h = x[..., :F], g = x[..., F:]."""
    x = np.asarray(x, dtype=np.float64)
    F = x.shape[-1] // 2
    if x.shape[-1] != 2 * F:
        raise ValueError("the last dimension must be even")
    return x[..., :F] * gelu(x[..., F:])
