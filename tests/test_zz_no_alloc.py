"""sdattn_qk_stats_noalloc: the allocation-free variant of sdattn_qk_stats.

It serves callers that may not allocate device memory (no workspace of their
own): its split-reduction scratch is a fixed array inside the library.  These
checks call it through the C ABI and compare it with sdattn_qk_stats (given a
caller-owned workspace) on the same inputs, twice in a row, since every call
reuses the one array that the previous call left behind.  Both entry points
run the same kernel with the same work split, and the split merge has a fixed
order, so A and LS must be bitwise identical.  The cases run from the most
column splits to none, so a call always finds the array as a call with a
different layout left it.

This file is named to be collected last, so that a run stopping at the first
failure has already run every other test; it also passes on its own.
"""
import ctypes
import math

import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from diffusion_unet_attention_b200 import _lib  # noqa: E402

DEV = torch.device("cuda:0")


def _run(lib, fn, desc, tq, tk, lda, ws=None):
    B, H, N = desc.B, desc.H, desc.N
    a = torch.full((B, H, N, lda), float("nan"), dtype=torch.float32, device=DEV)
    ls = torch.full((B, H, N, 2), float("nan"), dtype=torch.float32, device=DEV)
    stream = ctypes.c_void_p(torch.cuda.current_stream(DEV).cuda_stream)
    if fn == "qk_stats":
        st = lib.sdattn_qk_stats(ctypes.byref(desc), tq.data_ptr(), tk.data_ptr(), a.data_ptr(), ls.data_ptr(),
                                 ws.data_ptr(), ws.numel(), stream)
    else:
        st = lib.sdattn_qk_stats_noalloc(ctypes.byref(desc), tq.data_ptr(), tk.data_ptr(), a.data_ptr(),
                                         ls.data_ptr(), stream)
    assert st == 0, _lib.STATUS.get(st, st)
    torch.cuda.synchronize()
    return a, ls


# Column splits with 148 SMs in brackets (the plan depends on the SM count).
@pytest.mark.parametrize("B,H,N,M,d", [
    (1, 4, 128, 8192, 40),      # [16 splits] four row tiles of partials and counters
    (2, 8, 512, 4096, 40),      # [2 splits]
    (2, 8, 4096, 4096, 40),     # [2 splits] 64x64-latent self-attention
    (2, 8, 1024, 1024, 80),     # [1 split] 32x32-latent self-attention: one wave unsplit
    (2, 8, 300, 77, 160),       # [1 split] no scratch in use
])
def test_matches_workspace_entry_point_twice(B, H, N, M, d):
    lib = _lib.load()
    desc = _lib.Desc(B, H, N, M, d, _lib.SDATTN_F16, float(np.float32(1 / math.sqrt(d))))
    q, k, _ = synth.make_qkv(synth.Shape("t", B, H, N, M, d), 80, call_id=d)
    tq, tk = (torch.from_numpy(x).to(DEV) for x in (q, k))
    lda = lib.sdattn_a_ld(ctypes.byref(desc))
    ws = torch.zeros(max(lib.sdattn_workspace_bytes(ctypes.byref(desc)), 256), dtype=torch.uint8, device=DEV)
    a_ref, ls_ref = _run(lib, "qk_stats", desc, tq, tk, lda, ws)
    assert torch.isfinite(a_ref[..., :M]).all() and torch.isfinite(ls_ref).all()
    for _ in range(2):
        a, ls = _run(lib, "noalloc", desc, tq, tk, lda)
        assert torch.equal(a[..., :M], a_ref[..., :M])
        assert torch.equal(ls, ls_ref)
    status = ctypes.c_uint32(0)
    assert lib.sdattn_device_error(ctypes.byref(status)) == 0


def test_rejects_shapes_beyond_its_scratch():
    """1060 row tiles of 16384-key rows: with 148 SMs the plan splits each row
    in two (the split shortens the busiest CTA's chain from 512 to 495 block
    times), and the partials (1060 x 128 x 2 float2, 2.17 MB) exceed the 2 MiB
    array.  The split plan follows the SM count, so the case is only known to
    exceed it on 148 SMs.  The buffers are real and full-size, so a call that
    were accepted would still stay inside them."""
    if torch.cuda.get_device_properties(DEV).multi_processor_count != 148:
        pytest.skip("the split plan of this shape is worked out for 148 SMs")
    lib = _lib.load()
    B, H, N, M, d = 1, 1060, 128, 16384, 40
    desc = _lib.Desc(B, H, N, M, d, _lib.SDATTN_F16, 0.15811388)
    q = torch.zeros((B, H, N, d), dtype=torch.float16, device=DEV)
    k = torch.zeros((B, H, M, d), dtype=torch.float16, device=DEV)
    a = torch.empty((B, H, N, M), dtype=torch.float32, device=DEV)
    ls = torch.empty((B, H, N, 2), dtype=torch.float32, device=DEV)
    st = lib.sdattn_qk_stats_noalloc(ctypes.byref(desc), q.data_ptr(), k.data_ptr(), a.data_ptr(), ls.data_ptr(),
                                     None)
    assert _lib.STATUS[st] == "SDATTN_ERR_WORKSPACE"
