"""The flash kernel's FMA-pipe 2^x routine, run on the device (the CPU test
emulates it in fp32; this one runs the routine itself, compiled from the
library's header into a small test kernel).

* Bit for bit the fp32 emulation of the CPU test, so the emulation's error
  analysis applies to the device code.
* Within 8e-5 of exact 2^x (relative) over [-24, 8], where an fp16 P can hold
  the value, and within 8e-5 of the MUFU ex2 instruction beside it.
* Finite and zero in fp16 far below (including -inf, the masked scores).
"""
import ctypes
import os
import subprocess
import tempfile

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from test_exp2_poly import exp2_poly  # noqa: E402

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "diffusion_unet_attention_b200", "csrc")


@pytest.fixture(scope="module")
def probe():
    out = os.path.join(tempfile.mkdtemp(), "exp2_probe.so")
    nvcc = "/usr/local/cuda/bin/nvcc" if os.path.exists("/usr/local/cuda/bin/nvcc") else "nvcc"
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-Xcompiler", "-fPIC",
                    "-shared", "-I", CSRC, "-o", out, os.path.join(HERE, "cuda", "exp2_poly_device.cu")], check=True)
    lib = ctypes.CDLL(out)
    lib.exp2_poly_probe_run.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int]
    lib.exp2_poly_probe_run.restype = ctypes.c_int
    return lib


def run(lib, x):
    x = np.ascontiguousarray(x, np.float32)
    tx = torch.from_numpy(x).cuda()
    yp, ym = torch.empty_like(tx), torch.empty_like(tx)
    assert lib.exp2_poly_probe_run(tx.data_ptr(), yp.data_ptr(), ym.data_ptr(), x.size) == 0
    return yp.cpu().numpy(), ym.cpu().numpy()


def test_device_routine_within_its_bound(probe):
    x = np.linspace(-24.0, 8.0, 400002, dtype=np.float32)
    yp, ym = run(probe, x)
    assert np.array_equal(yp.view(np.uint32), exp2_poly(x).view(np.uint32)), "device and emulation differ"
    exact = np.exp2(x.astype(np.float64))
    assert np.abs(yp / exact - 1).max() < 8e-5
    assert np.abs(yp.astype(np.float64) / ym.astype(np.float64) - 1).max() < 8e-5


def test_device_routine_far_below(probe):
    x = np.concatenate([np.linspace(-300.0, -24.0, 100000, dtype=np.float32),
                        np.array([-np.inf, -1e30, -126.0, -125.5, -125.0, -124.9], np.float32)])
    yp, _ = run(probe, x)
    assert np.array_equal(yp.view(np.uint32), exp2_poly(x).view(np.uint32))
    assert np.all(np.isfinite(yp)) and np.all(yp >= 0)
    assert np.all(yp[x < -25].astype(np.float16) == 0)
