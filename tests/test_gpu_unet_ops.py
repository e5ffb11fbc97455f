"""GPU parity of the GroupNorm and gated-GELU kernels against their fp64 oracles.

Shapes are those of SD 1.4's UNet at 512x512 (B = 2; GroupNorm with 32
groups over 320/640/1280 channels at 64x64 .. 8x8; the gated GELU over
2 x h x w tokens with F = 4 x channels) plus ragged and extreme ones.  Both
kernels compute in fp32 and round the output once to 16 bits, so the bar is
relative: max |y - y_ref| / max(|y_ref|, 1) <= 1e-3 (an fp16 rounding is at
most 2^-11 ~ 4.9e-4 of the value) and ||y - y_ref||_F / ||y_ref||_F <= 1e-3.
"""
import numpy as np
import pytest

import synth
from oracle import unet_ops

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import diffusion_unet_attention_b200 as sd  # noqa: E402

DEV = torch.device("cuda:0")


def check(got, ref, what, tol=1e-3):
    got = np.asarray(got, np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    rel = float((np.abs(got - ref) / np.maximum(np.abs(ref), 1.0)).max())
    frob = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    assert rel <= tol and frob <= tol, f"{what}: max rel {rel:.3e}, rel_frob {frob:.3e}"
    return rel, frob


GN_SHAPES = [(2, 320, 64, 64, 32), (2, 640, 32, 32, 32), (2, 1280, 16, 16, 32), (2, 1280, 8, 8, 32),
             (2, 640, 64, 64, 32), (1, 96, 8, 8, 32), (1, 32, 2, 4, 32), (1, 64, 64, 64, 1), (1, 32, 64, 64, 1), (3, 64, 4, 6, 8)]


@pytest.mark.parametrize("B,C,H,W,G", GN_SHAPES)
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_group_norm(B, C, H, W, G, dtype):
    x64 = synth.normal_f64(500 + C + H, (B, C, H, W)) * 2.0 + 0.5
    x = torch.from_numpy(x64).to(dtype)
    xr = x.double().numpy()                     # the values the GPU receives
    gamma = 1.0 + 0.1 * synth.normal_f64(501, (C,))
    beta = 0.1 * synth.normal_f64(502, (C,))
    ref = unet_ops.group_norm(xr, gamma.astype(np.float32), beta.astype(np.float32), G, 1e-6)
    y = sd.group_norm(x.to(DEV), torch.from_numpy(gamma).float(), torch.from_numpy(beta).float(), G, 1e-6)
    torch.cuda.synchronize()
    # bf16 output rounds to 2^-9 of the value
    check(y.double().cpu().numpy(), ref, f"group_norm {B, C, H, W, G}", tol=1e-3 if dtype == torch.float16 else 4e-3)


def test_group_norm_constant_group_gives_beta():
    x = torch.full((1, 64, 8, 8), 3.0, dtype=torch.float16)
    beta = torch.linspace(-1, 1, 64)
    y = sd.group_norm(x.to(DEV), torch.ones(64), beta, 32, 1e-6)
    np.testing.assert_allclose(y.float().cpu().numpy(), beta.half().float().numpy().reshape(1, 64, 1, 1)
                               .repeat(8, 2).repeat(8, 3), rtol=0, atol=0)


GEGLU_SHAPES = [(2 * 64 * 64, 1280), (2 * 32 * 32, 2560), (2 * 16 * 16, 5120), (2 * 8 * 8, 5120), (1, 8), (3, 24),
                (777, 1000)]


@pytest.mark.parametrize("T,F", GEGLU_SHAPES)
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_geglu(T, F, dtype):
    x = torch.from_numpy(synth.normal_f64(600 + F % 97, (T, 2 * F)) * 1.5).to(dtype)
    ref = unet_ops.geglu(x.double().numpy())
    y = sd.geglu(x.to(DEV))
    torch.cuda.synchronize()
    check(y.double().cpu().numpy(), ref, f"geglu {T, F}", tol=1e-3 if dtype == torch.float16 else 4e-3)


def test_no_device_error_after_unet_ops():
    status, detail = sd.device_error()
    assert status == "SDATTN_OK", (status, hex(detail))
