"""The C ABI library loads, exports what include/sdattn.h declares, and rejects
bad arguments on the host before any CUDA call (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from diffusion_unet_attention_b200 import _lib, build
    build.build()
    return _lib.load()


def _desc(B=2, H=8, N=4096, M=4096, d=40, dtype=0, scale=0.158113883):
    from diffusion_unet_attention_b200 import _lib
    return _lib.Desc(B, H, N, M, d, dtype, scale)


def test_header_declarations_are_exported(lib):
    from diffusion_unet_attention_b200 import _lib
    hdr = open(os.path.join(ROOT, "include", "sdattn.h")).read()
    declared = set(re.findall(r"\b(sdattn_[a-z0-9_]+)\s*\(", hdr))
    assert declared == set(_lib.EXPORTS)
    for name in declared:
        assert hasattr(lib, name), name


def test_a_ld_and_workspace(lib):
    for M, ld in [(4096, 4096), (77, 80), (1, 4), (64, 64), (129, 132)]:
        assert lib.sdattn_a_ld(ctypes.byref(_desc(M=M))) == ld
    for M, ld in [(4096, 4096), (77, 80), (1, 8), (64, 64), (129, 136)]:
        assert lib.sdattn_a16_ld(ctypes.byref(_desc(M=M))) == ld
    assert lib.sdattn_a_ld(ctypes.byref(_desc(d=64))) == -1
    ws = lib.sdattn_workspace_bytes(ctypes.byref(_desc()))
    # tickets for 2*8*32 row tiles plus 16 splits of 128 float2 per tile
    assert ws >= 2 * 8 * 32 * 128 * 16 * 8
    assert lib.sdattn_workspace_bytes(ctypes.byref(_desc(N=0))) == 0


@pytest.mark.parametrize("kw,status", [
    (dict(B=0), 1), (dict(N=0), 1), (dict(M=-1), 1), (dict(scale=float("inf")), 1),
    (dict(scale=float("nan")), 1), (dict(scale=0.0), 1), (dict(scale=-0.1), 1), (dict(d=64), 2), (dict(d=128), 2), (dict(dtype=7), 2),
])
def test_bad_descriptor(lib, kw, status):
    d = _desc(**kw)
    p = ctypes.c_void_p(4096)
    assert lib.sdattn_flash(ctypes.byref(d), p, p, p, p, None, None, 0, None) == status
    assert lib.sdattn_qk_stats(ctypes.byref(d), p, p, p, p, p, 1 << 30, None) == status
    assert lib.sdattn_softmax_av(ctypes.byref(d), p, p, p, p, None) == status
    assert lib.sdattn_qk_scores(ctypes.byref(d), p, p, p, None) == status
    assert lib.sdattn_row_stats(ctypes.byref(d), p, p, p, 1 << 30, None) == status
    assert lib.sdattn_qk_stats_f16a(ctypes.byref(d), p, p, p, p, p, 1 << 30, None) == status
    assert lib.sdattn_softmax_av_f16a(ctypes.byref(d), p, p, p, p, None) == status
    assert lib.sdattn_a16_ld(ctypes.byref(d)) == -1


def test_null_and_misaligned_pointers(lib):
    d = _desc()
    ok = ctypes.c_void_p(1 << 20)
    bad = ctypes.c_void_p((1 << 20) + 8)
    assert lib.sdattn_flash(None, ok, ok, ok, ok, None, None, 0, None) == 1
    assert lib.sdattn_flash(ctypes.byref(d), None, ok, ok, ok, None, None, 0, None) == 1
    assert lib.sdattn_flash(ctypes.byref(d), ok, ok, bad, ok, None, None, 0, None) == 3
    assert lib.sdattn_flash(ctypes.byref(d), ok, ok, ok, ok, bad, None, 0, None) == 3
    assert lib.sdattn_softmax_av(ctypes.byref(d), ok, ok, ok, None, None) == 1
    assert lib.sdattn_softmax_av(ctypes.byref(d), bad, ok, ok, ok, None) == 3
    assert lib.sdattn_qk_stats(ctypes.byref(d), ok, ok, ok, bad, ok, 1 << 30, None) == 3
    assert lib.sdattn_qk_scores(ctypes.byref(d), ok, None, ok, None) == 1
    assert lib.sdattn_qk_scores(ctypes.byref(d), ok, ok, bad, None) == 3
    assert lib.sdattn_row_stats(ctypes.byref(d), ok, None, ok, 1 << 30, None) == 1
    assert lib.sdattn_row_stats(ctypes.byref(d), bad, ok, ok, 1 << 30, None) == 3
    assert lib.sdattn_qk_stats_f16a(ctypes.byref(d), ok, ok, bad, ok, ok, 1 << 30, None) == 3
    assert lib.sdattn_softmax_av_f16a(ctypes.byref(d), ok, ok, None, ok, None) == 1
    assert lib.sdattn_softmax_av_f16a(ctypes.byref(d), ok, ok, ok, bad, None) == 3


def test_workspace_checked(lib):
    d = _desc()
    ok = ctypes.c_void_p(1 << 20)
    need = lib.sdattn_workspace_bytes(ctypes.byref(d))
    assert lib.sdattn_qk_stats(ctypes.byref(d), ok, ok, ok, ok, None, need, None) == 4
    assert lib.sdattn_qk_stats(ctypes.byref(d), ok, ok, ok, ok, ok, 4096, None) == 4
    assert lib.sdattn_qk_stats_f16a(ctypes.byref(d), ok, ok, ok, ok, ok, 4096, None) == 4
    # row statistics: the workspace is needed only when rows are split (few
    # rows); a size without a pointer is always refused
    assert lib.sdattn_row_stats(ctypes.byref(d), ok, ok, None, 16, None) == 4
    few = _desc(B=1, H=1, N=16, M=4096)
    assert lib.sdattn_row_stats(ctypes.byref(few), ok, ok, None, 0, None) == 4
    assert lib.sdattn_workspace_bytes(ctypes.byref(few)) >= 16 * 8 * 8
    # flash: the workspace is optional, but a size without a pointer, a short
    # one or a misaligned one is refused before anything is enqueued
    bad = ctypes.c_void_p((1 << 20) + 8)
    assert lib.sdattn_flash(ctypes.byref(d), ok, ok, ok, ok, None, None, 16, None) == 4
    assert lib.sdattn_flash(ctypes.byref(d), ok, ok, ok, ok, None, ok, 4096, None) == 4
    assert lib.sdattn_flash(ctypes.byref(d), ok, ok, ok, ok, None, bad, need, None) == 3


def test_group_norm_and_geglu_arguments(lib):
    from diffusion_unet_attention_b200 import _lib
    ok = ctypes.c_void_p(1 << 20)
    bad = ctypes.c_void_p((1 << 20) + 8)
    good = _lib.GNDesc(2, 320, 64, 64, 32, 0, 1e-6)
    for kw, status in [(dict(C=321), 1), (dict(G=0), 1), (dict(B=0), 1), (dict(eps=-1.0), 1),
                       (dict(eps=float("nan")), 1), (dict(dtype=3), 2), (dict(H=3, W=3), 2),
                       (dict(C=32 * 65, H=64, W=64), 2)]:
        f = dict(B=2, C=320, H=64, W=64, G=32, dtype=0, eps=1e-6)
        f.update(kw)
        d = _lib.GNDesc(f["B"], f["C"], f["H"], f["W"], f["G"], f["dtype"], f["eps"])
        assert lib.sdattn_group_norm(ctypes.byref(d), ok, ok, ok, ok, None) == status, kw
    assert lib.sdattn_group_norm(None, ok, ok, ok, ok, None) == 1
    assert lib.sdattn_group_norm(ctypes.byref(good), ok, None, ok, ok, None) == 1
    assert lib.sdattn_group_norm(ctypes.byref(good), bad, ok, ok, ok, None) == 3
    assert lib.sdattn_geglu(0, 1280, 0, ok, ok, None) == 1
    assert lib.sdattn_geglu(10, 4, 0, ok, ok, None) == 1
    assert lib.sdattn_geglu(10, 1284, 0, ok, ok, None) == 2
    assert lib.sdattn_geglu(10, 1280, 5, ok, ok, None) == 2
    assert lib.sdattn_geglu(10, 1280, 0, None, ok, None) == 1
    assert lib.sdattn_geglu(10, 1280, 0, ok, bad, None) == 3


def test_winograd_arguments(lib):
    """Shape rules, workspace size and argument checks of the Winograd calls,
    all decided on the host (the pointers below are never dereferenced)."""
    from diffusion_unet_attention_b200 import _lib

    def cd(N=2, C=320, K=320, H=64, W=64, dtype=0):
        return ctypes.byref(_lib.ConvDesc(N, C, K, H, W, dtype))

    # U [36][K][C] 16-bit; workspace: V [36][T][C] 16-bit (256-byte rounded) + M [36][K][ldm] fp32
    assert lib.sdattn_wino_filter_bytes(cd()) == 36 * 320 * 320 * 2
    T = 2 * 16 * 16
    assert lib.sdattn_wino_workspace_bytes(cd()) == (36 * T * 320 * 2 + 255) // 256 * 256 + 36 * 320 * T * 4
    T = 1 * 4 * 3   # 13 x 10 -> 4 x 3 tiles, ldm 12
    assert lib.sdattn_wino_workspace_bytes(cd(N=1, C=24, K=40, H=13, W=10)) == \
        (36 * T * 24 * 2 + 255) // 256 * 256 + 36 * 40 * 12 * 4
    for bad in [dict(C=12), dict(W=4097), dict(dtype=7), dict(N=0), dict(K=0), dict(H=0)]:
        assert lib.sdattn_wino_filter_bytes(cd(**bad)) == 0, bad
        assert lib.sdattn_wino_workspace_bytes(cd(**bad)) == 0, bad
    fake = ctypes.c_void_p(1 << 20)   # 16-byte aligned, never touched
    need = lib.sdattn_wino_workspace_bytes(cd())
    conv = lib.sdattn_wino_conv3x3
    assert conv(cd(), fake, fake, None, fake, fake, need - 1, None) == 4      # workspace too small
    assert conv(cd(), fake, fake, None, fake, None, need, None) == 4          # no workspace
    assert conv(cd(C=12), fake, fake, None, fake, fake, need, None) == 2      # C not a multiple of 8
    assert conv(cd(N=0), fake, fake, None, fake, fake, need, None) == 1
    assert conv(cd(), ctypes.c_void_p((1 << 20) + 8), fake, None, fake, fake, need, None) == 3
    assert conv(cd(), fake, fake, ctypes.c_void_p((1 << 20) + 2), fake, fake, need, None) == 3   # bias
    assert conv(cd(), None, fake, None, fake, fake, need, None) == 1
    assert lib.sdattn_wino_filter(cd(), fake, ctypes.c_void_p((1 << 20) + 4), None) == 3
    assert lib.sdattn_wino_filter(cd(C=20), fake, fake, None) == 2


def test_flash_tf32_arguments(lib):
    """fp32 inputs go only through sdattn_flash_tf32, and it takes only them."""
    fake = ctypes.c_void_p(1 << 20)
    f32 = _desc(dtype=2)
    assert lib.sdattn_flash_tf32(ctypes.byref(_desc(dtype=0)), fake, fake, fake, fake, None, None) == 2
    assert lib.sdattn_flash_tf32(ctypes.byref(_desc(dtype=2, d=64)), fake, fake, fake, fake, None, None) == 2
    assert lib.sdattn_flash_tf32(ctypes.byref(f32), fake, None, fake, fake, None, None) == 1
    assert lib.sdattn_flash_tf32(ctypes.byref(f32), fake, fake, fake, ctypes.c_void_p((1 << 20) + 4), None, None) == 3
    assert lib.sdattn_flash_tf32(ctypes.byref(_desc(dtype=2, scale=0.0)), fake, fake, fake, fake, None, None) == 1
    # the 16-bit entry points reject fp32 descriptors
    assert lib.sdattn_a_ld(ctypes.byref(f32)) == -1
    assert lib.sdattn_flash(ctypes.byref(f32), fake, fake, fake, fake, None, None, 0, None) == 2


def test_status_strings(lib):
    for s in range(7):
        assert lib.sdattn_status_string(s)
    assert lib.sdattn_status_string(99) == b"unknown status"
    assert lib.sdattn_version() >= 100


def test_python_api_refuses_cpu_tensors():
    import torch
    import diffusion_unet_attention_b200 as sd
    q = torch.zeros(1, 1, 8, 40, dtype=torch.float16)
    with pytest.raises(ValueError):
        sd.flash(q, q, q)
    with pytest.raises(ValueError):
        sd.qk_stats(q, q)
