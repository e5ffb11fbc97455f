"""sdattn_qk_stats_noalloc: the allocation-free variant of sdattn_qk_stats.

It serves callers that may not allocate device memory (no workspace of their
own): its split-reduction scratch is a fixed array inside the library.  These
checks call it through the C ABI and compare it with sdattn_qk_stats (given a
caller-owned workspace) on the same inputs, twice in a row, since every call
reuses the one array that the previous call left behind.

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
A_TOL, L_TOL, S_RTOL = 1e-4, 1e-4, 1e-4      # the parity tolerances of the other GPU tests


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


@pytest.mark.parametrize("B,H,N,M,d", [
    (1, 1, 256, 4096, 40),      # 16 column splits: the scratch carries partials and counters
    (2, 8, 4096, 4096, 40),     # 64x64-latent self-attention (2 splits)
    (2, 8, 1024, 1024, 80),     # 32x32-latent self-attention
    (2, 8, 300, 77, 160),       # a single split: no scratch in use
])
def test_matches_workspace_entry_point_twice(B, H, N, M, d):
    lib = _lib.load()
    desc = _lib.Desc(B, H, N, M, d, _lib.SDATTN_F16, float(np.float32(1 / math.sqrt(d))))
    q, k, _ = synth.make_qkv(synth.Shape("t", B, H, N, M, d), 80, call_id=d)
    tq, tk = (torch.from_numpy(x).to(DEV) for x in (q, k))
    lda = lib.sdattn_a_ld(ctypes.byref(desc))
    ws = torch.zeros(max(lib.sdattn_workspace_bytes(ctypes.byref(desc)), 256), dtype=torch.uint8, device=DEV)
    a_ref, ls_ref = _run(lib, "qk_stats", desc, tq, tk, lda, ws)
    for _ in range(2):
        a, ls = _run(lib, "noalloc", desc, tq, tk, lda)
        assert torch.isfinite(a[..., :M]).all() and torch.isfinite(ls).all()
        assert (a[..., :M] - a_ref[..., :M]).abs().max().item() <= A_TOL
        assert (ls[..., 0] - ls_ref[..., 0]).abs().max().item() <= L_TOL
        assert ((ls[..., 1] / ls_ref[..., 1]) - 1).abs().max().item() <= S_RTOL
    status = ctypes.c_uint32(0)
    assert lib.sdattn_device_error(ctypes.byref(status)) == 0


def test_rejects_shapes_beyond_its_scratch():
    # 149 row tiles of an 8192-key row split 16 ways need about 2.4 MB of partials
    lib = _lib.load()
    desc = _lib.Desc(1, 149, 128, 8192, 40, _lib.SDATTN_F16, 0.15811388)
    p = torch.empty(16, dtype=torch.float32, device=DEV)
    st = lib.sdattn_qk_stats_noalloc(ctypes.byref(desc), p.data_ptr(), p.data_ptr(), p.data_ptr(), p.data_ptr(),
                                     None)
    assert _lib.STATUS[st] == "SDATTN_ERR_WORKSPACE"
