"""The gated-GELU kernel's GELU (no GPU): erf by Abramowitz and Stegun,
Handbook of Mathematical Functions (1964), formula 7.1.26, emulated in fp32
and held to the formula's stated bound (1.5e-7 absolute on erf) plus fp32
rounding, against the oracle's exact GELU (scipy's erf in fp64)."""
import numpy as np

from oracle import unet_ops


def _gelu_as7126_fp32(g):
    """fp32 emulation of the kernel's GELU (rcp and exp2 taken exact here)."""
    g = np.asarray(g, np.float32)
    p, a = np.float32(0.3275911), [np.float32(c) for c in (0.254829592, -0.284496736, 1.421413741,
                                                             -1.453152027, 1.061405429)]
    x = (np.abs(g) * np.float32(0.7071067811865476)).astype(np.float32)
    t = (np.float32(1) / (p * x + np.float32(1))).astype(np.float32)
    poly = t * (a[0] + t * (a[1] + t * (a[2] + t * (a[3] + t * a[4]))))
    e = np.exp2((-x * x * np.float32(1.4426950408889634)).astype(np.float64)).astype(np.float32)
    erfc = (poly * e).astype(np.float32)
    return (np.float32(0.5) * g * np.where(g >= 0, np.float32(2) - erfc, erfc)).astype(np.float64)


def test_kernel_gelu_approximation_within_its_bound():
    g = np.linspace(-12, 12, 480001)
    got = _gelu_as7126_fp32(g)
    ref = unet_ops.gelu(g)
    # erf to 1.5e-7 absolute (the formula) plus fp32 rounding: |GELU error| <= |g|/2 * 4e-7 + 2 ulp(GELU)
    bound = 0.5 * np.abs(g) * 4e-7 + 2 * np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(got - ref) <= bound)
