"""GPU parity over the whole UNet-step attention set the benchmark times.

The 32 calls of one 512x512 SD 1.4 UNet step (16 transformer blocks, each a
self-attention and a cross-attention), on the benchmark's own seeded inputs
(its first input set) and in its launch configuration (one shared workspace
and scratch, as `bench.Scratch` issues them), in both forms and so under the
paper's policy too.  Each call is compared with the fp64 oracle on a sample of
query rows that covers every 128-row tile and the first and last row of each,
at the gate: max |O - O_ref| <= 2e-3 and ||O - O_ref||_F / ||O_ref||_F <= 1e-3.
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

import bench  # noqa: E402
import diffusion_unet_attention_b200 as sd  # noqa: E402

DEV = torch.device("cuda:0")
MAX_ABS, REL_FROB = 2e-3, 1e-3


def sample_rows(N):
    if N <= 256:
        return np.arange(N)
    step = 7 if N <= 1024 else 29
    return np.unique(np.concatenate([np.arange(0, N, step), np.arange(127, N, 128), np.arange(128, N, 128),
                                     [N - 1]]))


@pytest.fixture(scope="module")
def step_set():
    sets = bench.StepSet(sd, torch, DEV, 0)
    scratch = bench.Scratch(sd, torch, DEV, bench.CALLS)
    return sets, scratch


@pytest.mark.parametrize("form", ["flash", "partial"])
def test_step_set_against_oracle(step_set, form):
    sets, scratch = step_set
    worst = (0.0, 0.0, "")
    for ci, (call, q, k, v, o) in enumerate(sets.inputs):
        o.fill_(float("nan"))
        scratch.run(call, q, k, v, o, form)
        torch.cuda.synchronize()
        rows = sample_rows(call.N)
        qh, kh, vh = synth.make_qkv(call, synth.STEP_SET_ID, call_id=ci)
        assert np.array_equal(qh, q.cpu().numpy())     # the benchmark's inputs, unchanged
        ref = oracle.attention(qh[:, :, rows], kh, vh, float(np.float32(1.0 / math.sqrt(call.d))))
        got = o[:, :, torch.from_numpy(rows).to(DEV)].float().cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(got)), f"{call.name} {form}: non-finite output"
        diff = got - ref["O"]
        ea = float(np.abs(diff).max())
        er = float(np.linalg.norm(diff) / np.linalg.norm(ref["O"]))
        assert ea <= MAX_ABS and er <= REL_FROB, f"{call.name} {form}: max_abs {ea:.3e} rel_frob {er:.3e}"
        if er > worst[1]:
            worst = (ea, er, call.name)
    print(f"{form}: worst call {worst[2]}: max_abs {worst[0]:.3e} rel_frob {worst[1]:.3e}")


def test_step_set_policy_matches_its_forms(step_set):
    """The policy issues exactly the per-call forms checked above: flash for
    d = 40, the partially fused pair otherwise, bitwise reproducible."""
    sets, scratch = step_set
    for call, q, k, v, o in sets.inputs:
        form = bench.policy_form(call)
        scratch.run(call, q, k, v, o, form)
        ref = torch.empty_like(o)
        scratch.run(call, q, k, v, ref, form)
        torch.cuda.synchronize()
        assert torch.equal(o, ref), call.name
    status, detail = sd.device_error()
    assert status == "SDATTN_OK", (status, hex(detail))
