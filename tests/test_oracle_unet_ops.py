"""Pins for the fp64 GroupNorm and gated-GELU oracles (no GPU).

Each oracle is checked against things other than itself: closed forms of the
normalisation (zero mean, variance var / (var + eps), a constant group maps to
beta), invariance to a per-group affine change of the input when eps = 0, a
pure-Python brute force with math.fsum and math.erf, and torch's CPU
group_norm and gelu in float64 as textbook routines.  A last test plants
plausible mistakes in copies of the oracles and checks that the pins catch
every one of them.
"""
import math

import numpy as np
import pytest

from oracle import unet_ops

torch = pytest.importorskip("torch")


def _x(seed, shape, loc=0.0, scale=1.0):
    return np.random.default_rng(seed).normal(loc, scale, shape)


# --------------------------------------------------------------------------
# GroupNorm pins: each takes a group_norm implementation and asserts.
# --------------------------------------------------------------------------

def pin_gn_moments(gn):
    x = _x(1, (2, 8, 5, 7), loc=3.0, scale=2.0)
    eps = 1e-3
    y = gn(x, np.ones(8), np.zeros(8), 4, eps).reshape(2, 4, -1)
    xg = x.reshape(2, 4, -1)
    var = xg.var(axis=2)
    np.testing.assert_allclose(y.mean(axis=2), 0.0, atol=1e-12)
    np.testing.assert_allclose(y.var(axis=2), var / (var + eps), rtol=1e-12)


def pin_gn_constant_group(gn):
    x = np.ones((1, 4, 3, 3)) * np.array([5.0, 5.0, -2.0, -2.0]).reshape(1, 4, 1, 1)
    beta = np.array([0.25, -1.0, 3.0, 0.5])
    y = gn(x, np.full(4, 7.0), beta, 2, 1e-5)
    np.testing.assert_allclose(y, np.broadcast_to(beta.reshape(1, 4, 1, 1), y.shape), atol=1e-12)


def pin_gn_affine_invariance(gn):
    x = _x(2, (2, 6, 4, 4))
    a = np.array([2.0, 0.5, 3.0]).reshape(1, 3, 1, 1, 1)
    b = np.array([-1.0, 4.0, 0.25]).reshape(1, 3, 1, 1, 1)
    x2 = (x.reshape(2, 3, 2, 4, 4) * a + b).reshape(x.shape)
    g, be = _x(3, 6), _x(4, 6)
    np.testing.assert_allclose(gn(x2, g, be, 3, 0.0), gn(x, g, be, 3, 0.0), atol=1e-12)


def _gn_brute(x, gamma, beta, G, eps):
    B, C, H, W = x.shape
    cpg = C // G
    y = np.zeros_like(x)
    for b in range(B):
        for g in range(G):
            vals = [float(x[b, c, i, j]) for c in range(g * cpg, (g + 1) * cpg) for i in range(H) for j in range(W)]
            mu = math.fsum(vals) / len(vals)
            var = math.fsum((v - mu) ** 2 for v in vals) / len(vals)
            for c in range(g * cpg, (g + 1) * cpg):
                for i in range(H):
                    for j in range(W):
                        y[b, c, i, j] = (float(x[b, c, i, j]) - mu) / math.sqrt(var + eps) * gamma[c] + beta[c]
    return y


def pin_gn_brute(gn):
    x = _x(5, (2, 6, 3, 2))
    g, be = _x(6, 6), _x(7, 6)
    np.testing.assert_allclose(gn(x, g, be, 3, 1e-6), _gn_brute(x, g, be, 3, 1e-6), atol=1e-12)


def pin_gn_torch(gn):
    x = _x(8, (2, 64, 8, 8), loc=0.5)
    g, be = _x(9, 64), _x(10, 64)
    ref = torch.nn.functional.group_norm(torch.from_numpy(x), 32, torch.from_numpy(g), torch.from_numpy(be),
                                         1e-6).numpy()
    np.testing.assert_allclose(gn(x, g, be, 32, 1e-6), ref, atol=1e-12)


GN_PINS = [pin_gn_moments, pin_gn_constant_group, pin_gn_affine_invariance, pin_gn_brute, pin_gn_torch]


@pytest.mark.parametrize("pin", GN_PINS, ids=lambda f: f.__name__)
def test_group_norm_pins(pin):
    pin(unet_ops.group_norm)


# --------------------------------------------------------------------------
# gated GELU pins
# --------------------------------------------------------------------------

def pin_gelu_identities(gelu):
    x = np.linspace(-6, 6, 241)
    np.testing.assert_allclose(gelu(np.zeros(3)), 0.0, atol=0)
    np.testing.assert_allclose(gelu(x) - gelu(-x), x, atol=1e-14)      # erf is odd
    np.testing.assert_allclose(gelu(np.array([40.0])), [40.0], rtol=1e-15)
    np.testing.assert_allclose(gelu(np.array([-40.0])), [0.0], atol=1e-300)


def pin_gelu_brute(gelu):
    x = _x(11, 64) * 3
    want = [0.5 * v * (1 + math.erf(v / math.sqrt(2))) for v in x]
    np.testing.assert_allclose(gelu(x), want, rtol=1e-14, atol=1e-300)


def pin_gelu_torch(gelu):
    x = _x(12, 4096) * 4
    ref = torch.nn.functional.gelu(torch.from_numpy(x), approximate="none").numpy()
    np.testing.assert_allclose(gelu(x), ref, rtol=1e-12, atol=1e-15)


def pin_geglu_split(geglu):
    # h = 1 everywhere: the result is GELU of the second half
    g = _x(13, (3, 16)) * 2
    x = np.concatenate([np.ones((3, 16)), g], axis=-1)
    want = np.array([[0.5 * v * (1 + math.erf(v / math.sqrt(2))) for v in row] for row in g])
    np.testing.assert_allclose(geglu(x), want, rtol=1e-14, atol=1e-300)
    # a gate of 40 passes h through times 40
    h = _x(14, (2, 8))
    np.testing.assert_allclose(geglu(np.concatenate([h, np.full((2, 8), 40.0)], axis=-1)), 40 * h, rtol=1e-15)


GELU_PINS = [pin_gelu_identities, pin_gelu_brute, pin_gelu_torch]


@pytest.mark.parametrize("pin", GELU_PINS, ids=lambda f: f.__name__)
def test_gelu_pins(pin):
    pin(unet_ops.gelu)


def test_geglu_split_pin():
    pin_geglu_split(unet_ops.geglu)


# --------------------------------------------------------------------------
# planted mistakes: every one must fail at least one pin
# --------------------------------------------------------------------------

def _gn_unbiased(x, gamma, beta, groups, eps):
    x = np.asarray(x, np.float64)
    B, C = x.shape[:2]
    xg = x.reshape(B, groups, -1)
    mean = xg.mean(axis=2, keepdims=True)
    var = xg.var(axis=2, ddof=1, keepdims=True)
    return ((xg - mean) / np.sqrt(var + eps)).reshape(x.shape) * gamma.reshape(1, C, 1, 1) + beta.reshape(1, C, 1, 1)


def _gn_strided_groups(x, gamma, beta, groups, eps):
    # groups taken as channels c, c + G, c + 2G, ... instead of contiguous runs
    x = np.asarray(x, np.float64)
    B, C = x.shape[:2]
    xt = x.reshape(B, C // groups, groups, -1).transpose(0, 2, 1, 3).reshape(B, groups, -1)
    mean = xt.mean(axis=2, keepdims=True)
    var = ((xt - mean) ** 2).mean(axis=2, keepdims=True)
    y = ((xt - mean) / np.sqrt(var + eps)).reshape(B, groups, C // groups, -1).transpose(0, 2, 1, 3)
    return y.reshape(x.shape) * gamma.reshape(1, C, 1, 1) + beta.reshape(1, C, 1, 1)


def _gn_eps_outside(x, gamma, beta, groups, eps):
    x = np.asarray(x, np.float64)
    B, C = x.shape[:2]
    xg = x.reshape(B, groups, -1)
    mean = xg.mean(axis=2, keepdims=True)
    var = ((xg - mean) ** 2).mean(axis=2, keepdims=True)
    return ((xg - mean) / (np.sqrt(var) + eps)).reshape(x.shape) * gamma.reshape(1, C, 1, 1) + \
        beta.reshape(1, C, 1, 1)


def _gn_gamma_per_group(x, gamma, beta, groups, eps):
    x = np.asarray(x, np.float64)
    B, C = x.shape[:2]
    y = unet_ops.group_norm(x, np.ones(C), np.zeros(C), groups, eps)
    gi = np.arange(C) // (C // groups)
    return y * gamma[gi].reshape(1, C, 1, 1) + beta.reshape(1, C, 1, 1)


def _gelu_tanh(x):
    x = np.asarray(x, np.float64)
    return 0.5 * x * (1 + np.tanh(math.sqrt(2 / math.pi) * (x + 0.044715 * x ** 3)))


def _gelu_no_sqrt2(x):
    from scipy.special import erf
    x = np.asarray(x, np.float64)
    return 0.5 * x * (1 + erf(x))


def _geglu_swapped(x):
    x = np.asarray(x, np.float64)
    F = x.shape[-1] // 2
    return x[..., F:] * unet_ops.gelu(x[..., :F])


def _fails(pins, impl):
    for pin in pins:
        try:
            pin(impl)
        except AssertionError:
            return True
    return False


@pytest.mark.parametrize("mutant", [_gn_unbiased, _gn_strided_groups, _gn_eps_outside, _gn_gamma_per_group],
                         ids=lambda f: f.__name__)
def test_group_norm_pins_catch_planted_mistakes(mutant):
    assert _fails(GN_PINS, mutant), mutant.__name__


@pytest.mark.parametrize("mutant", [_gelu_tanh, _gelu_no_sqrt2], ids=lambda f: f.__name__)
def test_gelu_pins_catch_planted_mistakes(mutant):
    assert _fails(GELU_PINS, mutant), mutant.__name__


def test_geglu_pin_catches_swapped_halves():
    with pytest.raises(AssertionError):
        pin_geglu_split(_geglu_swapped)

