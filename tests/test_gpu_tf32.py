"""GPU parity of the fp32-input FlashAttention form (sdattn_flash_tf32) against
the fp64 oracle on the raw fp32 inputs, including the small fp32
configuration (B = H = 1, N = M = 256, d = 40) without rounding to fp16.

Gate for O: the standard one, max |O - O_ref| <= 2e-3 and relative Frobenius
<= 1e-3.  L is no longer exact: the kernel rounds each fp32 operand to tf32
(10-bit mantissa, nearest: relative error at most 2^-11, bounded here by
2^-10 to leave room), so |L_gpu - L| <= scale * (2 * 2^-10 + 2^-20) *
max_j sum_i |q_i k_ji| + fp32 rounding; S within expm1(2 x that bound) + 2^-10 relative (every
score, and the max, move by at most the bound; P is rounded to tf32).
"""
import math

import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import diffusion_unet_attention_b200 as sd  # noqa: E402

DEV = torch.device("cuda:0")


def run(B, H, N, M, d, seed, q_scale=1.0, max_abs=2e-3):
    shape = synth.Shape("tf32", B, H, N, M, d)
    q, k, v = synth.make_qkv(shape, seed, dtype=np.float32)
    q = (q * q_scale).astype(np.float32)
    scale = float(np.float32(1 / math.sqrt(d)))
    ref = oracle.attention(q.astype(np.float64), k.astype(np.float64), v.astype(np.float64), scale)
    tq, tk, tv = (torch.from_numpy(np.ascontiguousarray(x)).to(DEV) for x in (q, k, v))
    o, ls = sd.flash_tf32(tq, tk, tv, scale, return_ls=True)
    torch.cuda.synchronize()
    got = o.double().cpu().numpy()
    err = np.abs(got - ref["O"])
    rel = float(np.linalg.norm(got - ref["O"]) / np.linalg.norm(ref["O"]))
    print(f"tf32 {B}x{H}x{N}x{M} d{d}: max_abs {err.max():.2e} rel_frob {rel:.2e}")
    assert np.all(np.isfinite(got))
    assert err.max() <= max_abs and rel <= 1e-3
    ls_h = ls.double().cpu().numpy()
    absdot = np.einsum("bhnd,bhmd->bhnm", np.abs(q.astype(np.float64)), np.abs(k.astype(np.float64))).max(-1)
    l_bound = scale * (2 * 2.0 ** -10 + 2.0 ** -20) * absdot + 1e-6 * (1 + np.abs(ref["L"]))
    assert np.all(np.abs(ls_h[..., 0] - ref["L"]) <= l_bound)
    # every score moves by at most the row's L bound, so S by at most expm1 of
    # twice it (score and max), plus the tf32 rounding of P and the exponential's error
    assert np.all(np.abs(ls_h[..., 1] / ref["S"] - 1) <= np.expm1(2 * l_bound) + 2.0 ** -10)
    return rel


def test_tiny_config_native_fp32():
    """The small fp32 configuration, read as fp32 (no fp16 rounding of the inputs)."""
    run(1, 1, 256, 256, 40, synth.STREAM["tiny"])


@pytest.mark.parametrize("B,H,N,M,d", [
    (2, 2, 300, 200, 40),    # ragged rows and keys
    (1, 3, 130, 77, 80),     # cross-attention width
    (1, 2, 64, 300, 160),    # 32-key tiles, ragged
    (1, 1, 1, 1, 40),        # one row, one key
    (2, 1, 129, 1000, 80),   # many key tiles, two query tiles per head
])
def test_shapes(B, H, N, M, d):
    run(B, H, N, M, d, seed=B * 100 + N % 97 + d)


def test_peaked_scores_rescale():
    """Q x3 (scores with sigma ~ 3): the running max grows across key tiles.
    The scores' tf32 rounding error is proportional to sum |q_i k_i|, three
    times that of unscaled inputs, so the max-abs bound scales with it (the
    relative Frobenius gate stays 1e-3); the 16-bit paths' scores are exact
    products and need no such allowance."""
    run(1, 2, 200, 900, 40, seed=7, q_scale=3.0, max_abs=3 * 2e-3)


def test_rejects_16bit_descriptor():
    q = torch.zeros(1, 1, 8, 40, device=DEV, dtype=torch.float16)
    with pytest.raises(TypeError):
        sd.flash_tf32(q, q, q)


def test_no_device_error_after_tf32():
    assert sd.device_error()[0] == "SDATTN_OK"
