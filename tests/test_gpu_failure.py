"""Failure detection without a GPU fault: a wait inside the flash kernel is
made to run out (it waits on a barrier that nothing completes, selected by a
test-only environment switch).  The kernel must give up after its time limit,
every role must leave, the host must read SDATTN_ERR_TIMEOUT from the device
error word, and the context must stay usable: the next call is correct."""
import math
import os

import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import diffusion_unet_attention_b200 as sd  # noqa: E402


def test_bounded_wait_reports_timeout_and_context_survives():
    dev = torch.device("cuda:0")
    shape = synth.Shape("t", 2, 8, 512, 512, 40)
    q, k, v = synth.make_qkv(shape, 81)
    tq, tk, tv = (torch.from_numpy(x).to(dev) for x in (q, k, v))
    assert sd.device_error()[0] == "SDATTN_OK"
    os.environ["SDATTN_TEST_INJECT_STALL"] = "1"
    try:
        sd.flash(tq, tk, tv, use_workspace=False)
        status, detail = sd.device_error()          # synchronises; about one second
    finally:
        del os.environ["SDATTN_TEST_INJECT_STALL"]
    assert status == "SDATTN_ERR_TIMEOUT"
    # the first role to give up records its wait site (0x100 + site): the
    # injected wait, or a role that was waiting on it, whichever ran out first
    assert 0x101 <= detail <= 0x100 + 17
    assert sd.device_error()[0] == "SDATTN_OK"      # reading cleared it
    o = sd.flash(tq, tk, tv).float().cpu().numpy()
    ref = oracle.attention(q, k, v, float(np.float32(1 / math.sqrt(40))))
    err = np.linalg.norm(o - ref["O"]) / np.linalg.norm(ref["O"])
    assert err <= 1e-3
    assert sd.device_error()[0] == "SDATTN_OK"
