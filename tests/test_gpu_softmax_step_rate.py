"""Rate of the flash kernel's softmax step on its own (tests/cuda/softmax_step_rate.cu):
tensor-memory load of 128 scores, the library's exponential block, store of
the packed weights, per warp, with nothing else running.  This is the ceiling
the d = 40 flash kernel works under (one exponential per score), measured
rather than assumed:

* with every exponential on MUFU the SM cannot pass the MUFU rate of 16 per
  clock (from the instruction throughput of the exponential unit), so the
  measurement is sane;
* moving 3 of 8 pairs to the FMA-pipe polynomial (the kernel's mix) raises
  the rate above the MUFU-only rate with two or more warps per scheduler.

Printed with -s: exponentials per clock per SM at 1, 2 and 3 warps per
scheduler; the design notes quote these numbers.
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

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "diffusion_unet_attention_b200", "csrc")
ITERS = 400


@pytest.fixture(scope="module")
def probe():
    out = os.path.join(tempfile.mkdtemp(), "softmax_step_rate.so")
    nvcc = "/usr/local/cuda/bin/nvcc" if os.path.exists("/usr/local/cuda/bin/nvcc") else "nvcc"
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-Xcompiler", "-fPIC",
                    "-shared", "-I", CSRC, "-o", out, os.path.join(HERE, "cuda", "softmax_step_rate.cu")], check=True)
    lib = ctypes.CDLL(out)
    lib.softmax_step_rate_run.argtypes = [ctypes.c_int] * 4 + [ctypes.c_void_p] * 2
    lib.softmax_step_rate_run.restype = ctypes.c_int
    return lib


def rate(lib, npoly, warps):
    """Exponentials per clock per SM, averaged over the warps of every SM."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    scores = torch.from_numpy((-0.1 * ((np.arange(4096) * 13) % 97)).astype(np.float32)).cuda()
    cycles = torch.zeros(sms * 12, dtype=torch.int64, device="cuda")
    assert lib.softmax_step_rate_run(npoly, sms, warps, ITERS, cycles.data_ptr(), scores.data_ptr()) == 0
    torch.cuda.synchronize()
    c = cycles.view(sms, 12)[:, :warps].double().mean().item() / ITERS   # cycles per iteration per warp
    return 32 * 128 * warps / c


def test_softmax_step_rate(probe):
    table = {(npoly, w): rate(probe, npoly, w) for npoly in (0, 3, 4) for w in (4, 8, 12)}
    for (npoly, w), r in sorted(table.items()):
        print(f"NPOLY {npoly}/8 on the FMA pipe, {w:2d} warps/SM ({w // 4} per scheduler): {r:6.2f} exp/clk/SM")
    for w in (4, 8, 12):
        assert 4.0 < table[(0, w)] <= 16.5, "MUFU-only rate outside (4, 16.5]"
    for w in (8, 12):
        assert table[(3, w)] > table[(0, w)], "the polynomial share should add throughput"
