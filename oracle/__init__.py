"""fp64 CPU oracle for O = softmax(scale * Q K^T) V and its row statistics.

TEST INFRASTRUCTURE ONLY: the tests, the package's smoke check and the
benchmark's CPU-baseline leg use it; the CUDA product path must never import
it.  It shares no code with the CUDA library; both sides are fed by the seeded
generator in `synth`, which holds no attention arithmetic.

The arithmetic lives in `oracle.c` (plain C, fp64, one query row per loop
iteration); this module compiles it with gcc on first use and calls it
through ctypes.  The definition it follows is exact attention, which both forms
in "Speed Is All You Need: On-Device Acceleration of Large Diffusion Models via
GPU-Aware Optimizations" (news summary, section on the three optimisations,
partially fused softmax and FlashAttention paragraphs) must reproduce.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_SO = os.path.join(_HERE, "_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False, src: str = _SRC, out: str = _SO) -> str:
    """Compile `src` into the shared object `out` with gcc (fp64, OpenMP)."""
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
           "-shared", "-fPIC", "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def load(path: str | None = None):
    """Load (building if needed) the oracle library and declare its symbols."""
    global _lib
    with _lock:
        if path is None and _lib is not None:
            return _lib
        so = path or build()
        lib = ctypes.CDLL(so)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.oracle_attention.restype = ctypes.c_int
        lib.oracle_attention.argtypes = [ctypes.c_int64] * 5 + [ctypes.c_double] + [dp] * 6
        lib.oracle_set_threads.argtypes = [ctypes.c_int]
        lib.oracle_set_threads.restype = None
        lib.oracle_max_threads.restype = ctypes.c_int
        if path is None:
            _lib = lib
        return lib


def _ptr(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double)) if a is not None else None


def attention(q, k, v, scale: float, want_a: bool = False, threads: int | None = None,
              lib=None):
    """Exact attention in fp64.

    q: [B,H,N,d], k and v: [B,H,M,d] (any real dtype; widened exactly to fp64).
    scale: the score scale (the fp32 value the GPU uses, widened).
    Returns a dict with O [B,H,N,d], L and S [B,H,N], and A [B,H,N,M] if asked.
    """
    lib = lib or load()
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    B, H, N, d = q.shape
    M = k.shape[2]
    if k.shape != (B, H, M, d) or v.shape != (B, H, M, d):
        raise ValueError("q [B,H,N,d], k and v [B,H,M,d] expected")
    o = np.empty((B, H, N, d), dtype=np.float64)
    ls = np.empty((B, H, N, 2), dtype=np.float64)
    a = np.empty((B, H, N, M), dtype=np.float64) if want_a else None
    if threads:
        lib.oracle_set_threads(int(threads))
    rc = lib.oracle_attention(B, H, N, M, d, float(scale), _ptr(q), _ptr(k), _ptr(v),
                              _ptr(o), _ptr(ls), _ptr(a))
    if rc != 0:
        raise RuntimeError("oracle_attention failed")
    out = {"O": o, "L": ls[..., 0].copy(), "S": ls[..., 1].copy()}
    if want_a:
        out["A"] = a
    return out


def max_threads() -> int:
    return int(load().oracle_max_threads())
