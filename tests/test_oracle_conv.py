"""Pins for the fp64 3x3 convolution oracle (no GPU).

The oracle is checked against things other than itself: a pure-Python brute
force with math.fsum, scipy's 2-D cross-correlation summed over channels and
torch's CPU conv2d in float64 (textbook routines), closed forms (the identity
filter returns the input, a corner tap shifts it with a zero border, a bias
adds a constant), and linearity.  A last test plants plausible mistakes in
copies of the oracle (a flipped kernel, a padding off by one, K and C swapped,
a dropped bias) and checks that the pins catch every one of them.
"""
import math

import numpy as np
import pytest
from scipy.signal import correlate2d

from oracle import conv

torch = pytest.importorskip("torch")


def _r(seed, shape):
    return np.random.default_rng(seed).normal(0.0, 1.0, shape)


def brute(x, w, bias):
    N, C, H, W = x.shape
    K = w.shape[0]
    y = np.zeros((N, K, H, W))
    for n in range(N):
        for k in range(K):
            for h in range(H):
                for ww in range(W):
                    terms = [0.0 if bias is None else float(bias[k])]
                    for c in range(C):
                        for r in range(3):
                            for s in range(3):
                                hh, wc = h + r - 1, ww + s - 1
                                if 0 <= hh < H and 0 <= wc < W:
                                    terms.append(float(w[k, c, r, s]) * float(x[n, c, hh, wc]))
                    y[n, k, h, ww] = math.fsum(terms)
    return y


# --------------------------------------------------------------------------
# pins, each taking a conv3x3 implementation
# --------------------------------------------------------------------------

def pin_brute_force(f):
    for (N, C, K, H, W) in [(1, 1, 1, 1, 1), (1, 2, 3, 2, 3), (2, 3, 2, 5, 4), (1, 2, 2, 3, 1)]:
        x, w, b = _r(1 + H, (N, C, H, W)), _r(2 + W, (K, C, 3, 3)), _r(3, (K,))
        assert np.allclose(f(x, w, b), brute(x, w, b), rtol=1e-12, atol=1e-12)


def pin_scipy(f):
    x, w = _r(4, (2, 3, 9, 7)), _r(5, (4, 3, 3, 3))
    y = f(x, w, None)
    for n in range(2):
        for k in range(4):
            ref = sum(correlate2d(x[n, c], w[k, c], mode="same", boundary="fill") for c in range(3))
            assert np.allclose(y[n, k], ref, rtol=1e-12, atol=1e-12)


def pin_torch(f):
    x, w, b = _r(6, (2, 5, 8, 6)), _r(7, (3, 5, 3, 3)), _r(8, (3,))
    ref = torch.nn.functional.conv2d(torch.from_numpy(x), torch.from_numpy(w), torch.from_numpy(b), padding=1)
    assert np.allclose(f(x, w, b), ref.numpy(), rtol=1e-12, atol=1e-12)


def pin_identity_and_shift(f):
    x = _r(9, (2, 4, 6, 5))
    w = np.zeros((4, 4, 3, 3))
    for c in range(4):
        w[c, c, 1, 1] = 1.0
    assert np.array_equal(f(x, w, None), x)
    # tap (0, 0): y[h, w] = x[h - 1, w - 1], zero on the top row and left column
    w = np.zeros((4, 4, 3, 3))
    for c in range(4):
        w[c, c, 0, 0] = 1.0
    y = f(x, w, None)
    assert np.array_equal(y[:, :, 1:, 1:], x[:, :, :-1, :-1])
    assert np.all(y[:, :, 0, :] == 0) and np.all(y[:, :, :, 0] == 0)


def pin_bias_and_linearity(f):
    x1, x2, w, b = _r(10, (1, 3, 5, 5)), _r(11, (1, 3, 5, 5)), _r(12, (2, 3, 3, 3)), _r(13, (2,))
    assert np.allclose(f(x1, w, b) - f(x1, w, None), b[None, :, None, None] * np.ones((1, 2, 5, 5)), atol=1e-12)
    assert np.allclose(f(2.0 * x1 - 3.0 * x2, w, None), 2.0 * f(x1, w, None) - 3.0 * f(x2, w, None), atol=1e-12)


PINS = [pin_brute_force, pin_scipy, pin_torch, pin_identity_and_shift, pin_bias_and_linearity]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_pins(pin):
    pin(conv.conv3x3)


def test_points_match_full():
    x, w, b = _r(14, (2, 6, 9, 11)), _r(15, (5, 6, 3, 3)), _r(16, (5,))
    y = conv.conv3x3(x, w, b)
    pts = [(0, 0, 0, 0), (1, 4, 8, 10), (0, 2, 4, 0), (1, 1, 0, 10), (1, 3, 5, 6)]
    assert np.allclose(conv.conv3x3_points(x, w, b, pts), [y[p] for p in pts], rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# planted mistakes: each must fail at least one pin
# --------------------------------------------------------------------------

def _flipped(x, w, bias=None):
    return conv.conv3x3(x, np.asarray(w)[:, :, ::-1, ::-1], bias)


def _pad_off_by_one(x, w, bias=None):
    x = np.asarray(x, dtype=np.float64)
    y = conv.conv3x3(x, w, bias)
    return np.roll(y, 1, axis=3)


def _k_c_swapped(x, w, bias=None):
    w = np.asarray(w)
    if w.shape[0] != w.shape[1]:
        return conv.conv3x3(x, w, bias)[:, ::-1]
    return conv.conv3x3(x, np.transpose(w, (1, 0, 2, 3)), bias)


def _bias_dropped(x, w, bias=None):
    return conv.conv3x3(x, w, None)


@pytest.mark.parametrize("wrong", [_flipped, _pad_off_by_one, _k_c_swapped, _bias_dropped],
                         ids=["flipped", "pad_off_by_one", "k_c_swapped", "bias_dropped"])
def test_pins_catch_planted_mistakes(wrong):
    caught = 0
    for pin in PINS:
        try:
            pin(wrong)
        except AssertionError:
            caught += 1
    assert caught >= 1, f"no pin catches {wrong.__name__}"
