"""fp64 CPU oracle for the 3x3 convolution that the Winograd kernels compute.

TEST INFRASTRUCTURE ONLY: the tests and the benchmark's checks call this; the
CUDA product path never imports it.  It shares no code with the CUDA library.

"Speed Is All You Need: On-Device Acceleration of Large Diffusion Models via
GPU-Aware Optimizations" (news summary, section on the three optimisations,
Winograd paragraphs): the UNet's 3x3 convolutions are computed with the
Winograd algorithm, which turns a convolution into fewer multiplications on
transformed tiles, and a 4x4 tile is named as the best balance of compute
efficiency and memory.  Winograd's minimal filtering reaches exactly the
convolution (it is an exact rearrangement of the same sums, up to rounding),
so the oracle is the convolution written out by its definition.

Readings of what the page leaves open:

* the convolution is the UNet's: 3x3 kernel, stride 1, zero padding 1 (the
  output has the input's H x W), NCHW layout, weights [K][C][3][3] applied as
  cross-correlation (no kernel flip), an optional per-output-channel bias;
* "4x4 tile" is the output tile: F(4x4, 3x3), whose input tile is 6x6.
"""
from __future__ import annotations

import numpy as np


def conv3x3(x, w, bias=None):
    """y[n,k,h,w] = bias[k] + sum_{c,r,s} w[k,c,r,s] x[n,c,h+r-1,w+s-1] in fp64,
    x zero outside its H x W.  x [N, C, H, W]; w [K, C, 3, 3]; bias [K] or None."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    N, C, H, W = x.shape
    K = w.shape[0]
    if w.shape != (K, C, 3, 3):
        raise ValueError("w must be [K, C, 3, 3] with the input's C")
    xp = np.zeros((N, C, H + 2, W + 2), dtype=np.float64)
    xp[:, :, 1:H + 1, 1:W + 1] = x
    y = np.zeros((N, K, H, W), dtype=np.float64)
    for r in range(3):
        for s in range(3):
            # one tap of every filter against the shifted input: a matrix product over c
            y += np.einsum("kc,nchw->nkhw", w[:, :, r, s], xp[:, :, r:r + H, s:s + W], optimize=True)
    if bias is not None:
        y += np.asarray(bias, dtype=np.float64)[None, :, None, None]
    return y


def conv3x3_points(x, w, bias, points):
    """The same convolution at a list of (n, k, h, w) output positions only."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    N, C, H, W = x.shape
    out = np.empty(len(points), dtype=np.float64)
    for i, (n, k, h, ww) in enumerate(points):
        acc = 0.0 if bias is None else float(bias[k])
        for r in range(3):
            hh = h + r - 1
            if hh < 0 or hh >= H:
                continue
            for s in range(3):
                wc = ww + s - 1
                if wc < 0 or wc >= W:
                    continue
                acc += float(np.dot(w[k, :, r, s], x[n, :, hh, wc]))
        out[i] = acc
    return out
