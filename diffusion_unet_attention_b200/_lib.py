"""ctypes declarations of libsdattn's C ABI (include/sdattn.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind these symbols.  Loading fails loudly when the shared library is
missing; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsdattn.so")

SDATTN_F16 = 0
SDATTN_BF16 = 1
SDATTN_F32 = 2

STATUS = {
    0: "SDATTN_OK",
    1: "SDATTN_ERR_INVALID_ARG",
    2: "SDATTN_ERR_UNSUPPORTED",
    3: "SDATTN_ERR_ALIGNMENT",
    4: "SDATTN_ERR_WORKSPACE",
    5: "SDATTN_ERR_CUDA",
    6: "SDATTN_ERR_TIMEOUT",
}

# Every symbol include/sdattn.h declares.
EXPORTS = ("sdattn_a_ld", "sdattn_workspace_bytes", "sdattn_qk_stats", "sdattn_softmax_av", "sdattn_flash",
           "sdattn_flash_f32o", "sdattn_flash_tf32",
           "sdattn_qk_scores", "sdattn_row_stats", "sdattn_a16_ld", "sdattn_qk_stats_f16a",
           "sdattn_softmax_av_f16a", "sdattn_group_norm", "sdattn_geglu", "sdattn_qk_stats_noalloc",
           "sdattn_wino_filter_bytes", "sdattn_wino_workspace_bytes", "sdattn_wino_filter", "sdattn_wino_conv3x3",
           "sdattn_device_error", "sdattn_status_string", "sdattn_version")


class Desc(ctypes.Structure):
    """sdattn_desc: shape of one attention call."""
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32), ("M", ctypes.c_int32),
                ("d", ctypes.c_int32), ("dtype", ctypes.c_int32), ("scale", ctypes.c_float)]


class GNDesc(ctypes.Structure):
    """sdattn_gn_desc: shape of one group normalisation."""
    _fields_ = [("B", ctypes.c_int32), ("C", ctypes.c_int32), ("H", ctypes.c_int32), ("W", ctypes.c_int32),
                ("G", ctypes.c_int32), ("dtype", ctypes.c_int32), ("eps", ctypes.c_float)]


class ConvDesc(ctypes.Structure):
    """sdattn_conv_desc: shape of one 3x3 convolution."""
    _fields_ = [("N", ctypes.c_int32), ("C", ctypes.c_int32), ("K", ctypes.c_int32), ("H", ctypes.c_int32),
                ("W", ctypes.c_int32), ("dtype", ctypes.c_int32)]


class SdattnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {STATUS.get(status, status)}")
        self.status = status


_lib = None


def load(path: str = LIB_PATH):
    """Loads libsdattn and declares its symbols (raises if it is missing)."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libsdattn.so not built at {path}; run "
                          "`python -m diffusion_unet_attention_b200.build`")
    lib = ctypes.CDLL(path)
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    dp = ctypes.POINTER(Desc)
    lib.sdattn_a_ld.argtypes = [dp]
    lib.sdattn_a_ld.restype = ctypes.c_int64
    lib.sdattn_workspace_bytes.argtypes = [dp]
    lib.sdattn_workspace_bytes.restype = sz
    lib.sdattn_qk_stats.argtypes = [dp, vp, vp, vp, vp, vp, sz, vp]
    lib.sdattn_qk_stats.restype = ctypes.c_int
    lib.sdattn_softmax_av.argtypes = [dp, vp, vp, vp, vp, vp]
    lib.sdattn_softmax_av.restype = ctypes.c_int
    lib.sdattn_flash_f32o.argtypes = [dp, vp, vp, vp, vp, vp, vp]
    lib.sdattn_flash_f32o.restype = ctypes.c_int
    lib.sdattn_flash_tf32.argtypes = [dp, vp, vp, vp, vp, vp, vp]
    lib.sdattn_flash_tf32.restype = ctypes.c_int
    lib.sdattn_qk_scores.argtypes = [dp, vp, vp, vp, vp]
    lib.sdattn_qk_scores.restype = ctypes.c_int
    lib.sdattn_row_stats.argtypes = [dp, vp, vp, vp, sz, vp]
    lib.sdattn_row_stats.restype = ctypes.c_int
    lib.sdattn_a16_ld.argtypes = [dp]
    lib.sdattn_a16_ld.restype = ctypes.c_int64
    lib.sdattn_qk_stats_f16a.argtypes = [dp, vp, vp, vp, vp, vp, sz, vp]
    lib.sdattn_qk_stats_f16a.restype = ctypes.c_int
    lib.sdattn_softmax_av_f16a.argtypes = [dp, vp, vp, vp, vp, vp]
    lib.sdattn_softmax_av_f16a.restype = ctypes.c_int
    lib.sdattn_flash.argtypes = [dp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.sdattn_flash.restype = ctypes.c_int
    lib.sdattn_group_norm.argtypes = [ctypes.POINTER(GNDesc), vp, vp, vp, vp, vp]
    lib.sdattn_group_norm.restype = ctypes.c_int
    lib.sdattn_geglu.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, vp, vp, vp]
    lib.sdattn_geglu.restype = ctypes.c_int
    cp = ctypes.POINTER(ConvDesc)
    lib.sdattn_wino_filter_bytes.argtypes = [cp]
    lib.sdattn_wino_filter_bytes.restype = sz
    lib.sdattn_wino_workspace_bytes.argtypes = [cp]
    lib.sdattn_wino_workspace_bytes.restype = sz
    lib.sdattn_wino_filter.argtypes = [cp, vp, vp, vp]
    lib.sdattn_wino_filter.restype = ctypes.c_int
    lib.sdattn_wino_conv3x3.argtypes = [cp, vp, vp, vp, vp, vp, sz, vp]
    lib.sdattn_wino_conv3x3.restype = ctypes.c_int
    lib.sdattn_qk_stats_noalloc.argtypes = [dp, vp, vp, vp, vp, vp]
    lib.sdattn_qk_stats_noalloc.restype = ctypes.c_int
    lib.sdattn_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32)]
    lib.sdattn_device_error.restype = ctypes.c_int
    lib.sdattn_status_string.argtypes = [ctypes.c_int]
    lib.sdattn_status_string.restype = ctypes.c_char_p
    lib.sdattn_version.argtypes = []
    lib.sdattn_version.restype = ctypes.c_int32
    if path == LIB_PATH:
        _lib = lib
    return lib


def check(fn: str, status: int) -> None:
    if status != 0:
        raise SdattnError(fn, status)
