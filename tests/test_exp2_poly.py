"""The FMA-pipe 2^x routine of the flash kernel, emulated bit-for-bit in fp32
on the CPU (no GPU): finite everywhere, within its stated error bound where
fp16 P can hold the result, and rounding to zero in fp16 below that."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "diffusion_unet_attention_b200", "csrc", "sm100.cuh")


def _constants():
    text = open(HDR).read()
    c = [np.float32(float(re.search(rf"kExp2C{i} = ([0-9.eE+-]+)f;", text).group(1))) for i in range(4)]
    clamp = np.float32(float(re.search(r"x0 = fmaxf\(x0, (-[0-9.]+)f\);", text).group(1)))
    return c, clamp


def exp2_poly(x):
    """fp32 emulation of exp2_poly2 (round-to-nearest-even at every step)."""
    c, clamp = _constants()
    x = np.maximum(np.asarray(x, np.float32), clamp)
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    j = (t - magic).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = (f * c[3] + c[2]).astype(np.float32)      # fma: products of fp32 are exact in fp64
    p = (f.astype(np.float64) * c[3] + c[2]).astype(np.float32)
    p = (p.astype(np.float64) * f + c[1]).astype(np.float32)
    p = (p.astype(np.float64) * f + c[0]).astype(np.float32)
    bits = p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_accuracy_where_fp16_can_hold_it():
    x = np.linspace(-24.0, 8.0, 400001, dtype=np.float32)
    y = exp2_poly(x).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1)
    assert rel.max() < 8e-5


def test_finite_and_zero_in_fp16_far_below():
    x = np.concatenate([np.linspace(-300.0, -24.0, 100001, dtype=np.float32),
                        np.array([-np.inf, -1e30, -126.0, -125.5, -125.0, -124.9], np.float32)])
    y = exp2_poly(x)
    assert np.all(np.isfinite(y)) and np.all(y >= 0)
    assert np.all(y[x < -25] .astype(np.float16) == 0)


def test_matches_exact_powers_of_two_closely():
    x = np.arange(-120, 9, dtype=np.float32)
    y = exp2_poly(x).astype(np.float64)
    assert np.abs(y / np.exp2(x.astype(np.float64)) - 1).max() < 8e-5


def test_committed_fit_reproduces_the_kernel_constants():
    """The coefficients in sm100.cuh are the degree-3 fit of csrc/exp2_poly_fit.py."""
    import importlib.util
    path = os.path.join(os.path.dirname(HDR), "exp2_poly_fit.py")
    spec = importlib.util.spec_from_file_location("exp2_poly_fit", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    c32, lp = mod.fit(3)
    want, _ = _constants()
    np.testing.assert_allclose(c32, np.array(want, np.float32), rtol=2e-6, atol=0)
    assert lp < 7.6e-5 and mod.horner_max_rel(c32) < 8e-5
