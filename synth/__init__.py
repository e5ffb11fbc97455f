"""Seeded synthetic inputs for the Stable Diffusion 1.4 UNet attention shapes.

This module is shared by the tests, the benchmark and the CPU oracle's callers.
It holds no attention arithmetic: it only draws numbers and names shapes.

Random numbers: SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014) gives 64-bit words; the top 53 bits make a
uniform double in [0, 1); Box-Muller (1958) turns pairs of uniforms into
N(0, 1) doubles; numpy's float64 -> float16 cast rounds to nearest even.

Workload: SD 1.4 at 512x512 has a 64x64 latent; the UNet's transformer blocks
run self-attention over the h*w latent positions and cross-attention over the
77 text-context tokens, with 8 heads of width 320*k/8 for channel widths
320/640/1280 (k = 1, 2, 4).  The paper under study ("Speed Is All You Need:
On-Device Acceleration of Large Diffusion Models via GPU-Aware Optimizations",
Chen et al., CVPR Workshops 2023) benchmarks SD 1.4, 512x512, 20 iterations;
the N(0, 1) tensors drawn here stand in for the activations of that run,
since no trained weights or prompts are used.
"""
from __future__ import annotations

import hashlib
from dataclasses import dataclass

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_MIX1 = np.uint64(0xBF58476D1CE4E5B9)
_MIX2 = np.uint64(0x94D049BB133111EB)


def splitmix64(seed: int, count: int) -> np.ndarray:
    """`count` consecutive SplitMix64 outputs for state `seed` (uint64 array)."""
    with np.errstate(over="ignore"):
        idx = np.arange(1, count + 1, dtype=np.uint64)
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + idx * _GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _MIX1
        z = (z ^ (z >> np.uint64(27))) * _MIX2
        z = z ^ (z >> np.uint64(31))
    return z


def uniform01(seed: int, count: int) -> np.ndarray:
    """Uniform doubles in [0, 1) from the top 53 bits of each SplitMix64 word."""
    return (splitmix64(seed, count) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def normal_f64(seed: int, shape) -> np.ndarray:
    """N(0, 1) doubles by Box-Muller: u1 feeds the radius, u2 the angle."""
    n = int(np.prod(shape))
    pairs = (n + 1) // 2
    u = uniform01(seed, 2 * pairs)
    u1, u2 = u[0::2], u[1::2]
    r = np.sqrt(-2.0 * np.log1p(-u1))          # 1 - u1 lies in (0, 1]
    theta = 2.0 * np.pi * u2
    z = np.empty(2 * pairs, dtype=np.float64)
    z[0::2] = r * np.cos(theta)
    z[1::2] = r * np.sin(theta)
    return z[:n].reshape(shape)


def normal(seed: int, shape, dtype=np.float16) -> np.ndarray:
    """N(0, 1) values rounded (nearest even) to `dtype` (float16 or float32)."""
    return normal_f64(seed, shape).astype(dtype)


def sha256(a: np.ndarray) -> str:
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()


@dataclass(frozen=True)
class Shape:
    """One attention call: batch B, heads H, N queries, M keys, head width d."""
    name: str
    B: int
    H: int
    N: int
    M: int
    d: int

    @property
    def flops(self) -> int:
        """Algorithmic FLOPs of Q K^T plus P V: 2*N*M*d each, per (b, h)."""
        return 4 * self.B * self.H * self.N * self.M * self.d

    def a_bytes(self) -> int:
        """Bytes of the fp32 score matrix A (unpadded)."""
        return 4 * self.B * self.H * self.N * self.M


# The single-call workloads of the study, by name, and the seed stream each
# draws its inputs from.  Seeds follow 1000 * stream + {Q: 0, K: 1, V: 2} + 10 * call_id.
WORKLOADS = {
    "tiny": Shape("tiny self-attention", 1, 1, 256, 256, 40),
    "self64": Shape("64x64-latent self-attention", 2, 8, 4096, 4096, 40),
    "cross64": Shape("64x64-latent cross-attention", 2, 8, 4096, 77, 40),
    "self32": Shape("32x32-latent self-attention", 2, 8, 1024, 1024, 80),
    "self16": Shape("16x16-latent self-attention", 2, 8, 256, 256, 160),
    "self8": Shape("8x8 mid-block self-attention", 2, 8, 64, 64, 160),
}
STREAM = {"tiny": 1, "self64": 2, "cross64": 3, "self32": 4, "self16": 5, "self8": 6}
STEP_SET_ID = 7
TEXT_TOKENS = 77


def unet_step_set(B: int = 2, H: int = 8):
    """The 32 attention calls of one 512x512 SD 1.4 UNet step.

    16 transformer blocks: 64^2 x2 and 32^2 x2 and 16^2 x2 (down), 8^2 x1 (mid),
    16^2 x3, 32^2 x3, 64^2 x3 (up); each runs self-attention (M = N = h*w)
    and cross-attention (M = 77).  Head width d = 40 / 80 / 160 at 64^2 / 32^2 /
    16^2 and 8^2 (channels 320 / 640 / 1280 over 8 heads).
    """
    blocks = ([64] * 2 + [32] * 2 + [16] * 2 + [8] + [16] * 3 + [32] * 3 + [64] * 3)
    width = {64: 40, 32: 80, 16: 160, 8: 160}
    calls = []
    for bi, hw in enumerate(blocks):
        n = hw * hw
        d = width[hw]
        calls.append(Shape(f"block{bi:02d} self {hw}x{hw}", B, H, n, n, d))
        calls.append(Shape(f"block{bi:02d} cross {hw}x{hw}", B, H, n, TEXT_TOKENS, d))
    return calls


def seeds(stream: int, call_id: int = 0):
    """(seed_Q, seed_K, seed_V) for one call drawn from one seed stream."""
    base = 1000 * stream + 10 * call_id
    return base + 0, base + 1, base + 2


def make_qkv(shape: Shape, stream: int, call_id: int = 0, dtype=np.float16):
    """Seeded Q [B,H,N,d], K and V [B,H,M,d], N(0,1) rounded to `dtype`."""
    sq, sk, sv = seeds(stream, call_id)
    q = normal(sq, (shape.B, shape.H, shape.N, shape.d), dtype)
    k = normal(sk, (shape.B, shape.H, shape.M, shape.d), dtype)
    v = normal(sv, (shape.B, shape.H, shape.M, shape.d), dtype)
    return q, k, v
