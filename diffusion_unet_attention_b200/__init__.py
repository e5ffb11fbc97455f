"""B200 (sm_100a) attention for Stable Diffusion's UNet transformer blocks.

    O = softmax(scale * Q K^T) V,   Q [B,H,N,d], K and V [B,H,M,d], d in {40, 80, 160}

Two forms, after "Speed Is All You Need: On-Device Acceleration of Large
Diffusion Models via GPU-Aware Optimizations" (news summary, section on the
three optimisations, attention-efficiency paragraphs):

* partially fused softmax: `qk_stats` writes the fp32 score matrix A and the
  per-row statistics LS = (L_i, S_i) (row max, shifted sum of exponentials);
  `softmax_av` fuses the normalisation with the product by V;
* FlashAttention: `flash` tiles over keys with an online softmax in one kernel.

Variants of the partially fused form: the page's reduction as a kernel of its
own over a stored A (`qk_scores`, `row_stats`, then `softmax_av`), and A
stored in fp16 (`qk_stats_f16a`, `softmax_av_f16a`).  Beside attention, the
two specialised UNet kernels of the same section: `group_norm` and `geglu`.

This module only marshals torch tensors (device memory and streams) into the
C ABI of libsdattn.so; all arithmetic runs in the CUDA kernels.  There is no
CPU fallback: calls fail if the library or a CUDA device is missing.
"""
from __future__ import annotations

import ctypes
import math

import torch

from . import _lib

__all__ = ["qk_stats", "softmax_av", "flash", "flash_f32o", "flash_tf32", "partially_fused", "qk_scores", "row_stats", "qk_stats_f16a",
           "softmax_av_f16a", "group_norm", "geglu", "wino_filter", "conv3x3_winograd", "wino_workspace_bytes",
           "device_error", "a_ld", "a16_ld", "workspace_bytes", "SdattnError", "load_library"]

SdattnError = _lib.SdattnError
load_library = _lib.load

_DTYPES = {torch.float16: _lib.SDATTN_F16, torch.bfloat16: _lib.SDATTN_BF16}
_workspaces: dict[int, torch.Tensor] = {}


def _lib_handle():
    return _lib.load()


def make_desc(B: int, H: int, N: int, M: int, d: int, dtype: torch.dtype, scale: float) -> _lib.Desc:
    if dtype not in _DTYPES:
        raise TypeError(f"dtype {dtype} not supported (float16 or bfloat16)")
    return _lib.Desc(B, H, N, M, d, _DTYPES[dtype], float(scale))


def _scale(scale, d):
    return 1.0 / math.sqrt(d) if scale is None else float(scale)


def _check_qk(q: torch.Tensor, k: torch.Tensor):
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q must be [B,H,N,d] and k [B,H,M,d]")
    if not (q.is_cuda and k.is_cuda):
        raise ValueError("tensors must live on a CUDA device")
    if q.dtype != k.dtype:
        raise TypeError("q and k must share a dtype")
    B, H, N, d = q.shape
    if k.shape[0] != B or k.shape[1] != H or k.shape[3] != d:
        raise ValueError(f"shape mismatch: q {tuple(q.shape)}, k {tuple(k.shape)}")
    return B, H, N, k.shape[2], d


def _contig(t: torch.Tensor) -> torch.Tensor:
    return t if t.is_contiguous() else t.contiguous()


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def a_ld(desc: _lib.Desc) -> int:
    v = _lib_handle().sdattn_a_ld(ctypes.byref(desc))
    if v < 0:
        raise _lib.SdattnError("sdattn_a_ld", 1)
    return int(v)


def a16_ld(desc: _lib.Desc) -> int:
    v = _lib_handle().sdattn_a16_ld(ctypes.byref(desc))
    if v < 0:
        raise _lib.SdattnError("sdattn_a16_ld", 1)
    return int(v)


def workspace_bytes(desc: _lib.Desc) -> int:
    return int(_lib_handle().sdattn_workspace_bytes(ctypes.byref(desc)))


def workspace(desc: _lib.Desc, device: torch.device) -> torch.Tensor:
    """A zero-filled workspace for `desc` on `device`, cached and grown on demand.

    Calls that share it must be ordered on one stream (the library leaves the
    workspace ready for the next call when a call completes)."""
    need = max(workspace_bytes(desc), 256)
    idx = device.index if device.index is not None else torch.cuda.current_device()
    ws = _workspaces.get(idx)
    if ws is None or ws.numel() < need:
        ws = torch.zeros(need, dtype=torch.uint8, device=device)
        _workspaces[idx] = ws
    return ws


def qk_stats(q: torch.Tensor, k: torch.Tensor, scale: float | None = None, out_a: torch.Tensor | None = None,
             out_ls: torch.Tensor | None = None, ws: torch.Tensor | None = None):
    """Partially fused softmax, first kernel.

    Returns (A, LS): A [B,H,N,lda] fp32 with A[..., :M] = scale * Q K^T, and
    LS [B,H,N,2] fp32 = (row max L_i, sum_j exp(A_ij - L_i))."""
    B, H, N, M, d = _check_qk(q, k)
    q, k = _contig(q), _contig(k)
    desc = make_desc(B, H, N, M, d, q.dtype, _scale(scale, d))
    lda = a_ld(desc)
    A = out_a if out_a is not None else torch.empty((B, H, N, lda), dtype=torch.float32, device=q.device)
    LS = out_ls if out_ls is not None else torch.empty((B, H, N, 2), dtype=torch.float32, device=q.device)
    if A.shape != (B, H, N, lda) or A.dtype != torch.float32 or not A.is_contiguous():
        raise ValueError(f"out_a must be contiguous fp32 [B,H,N,{lda}]")
    if LS.shape != (B, H, N, 2) or LS.dtype != torch.float32 or not LS.is_contiguous():
        raise ValueError("out_ls must be contiguous fp32 [B,H,N,2]")
    w = ws if ws is not None else workspace(desc, q.device)
    st = _lib_handle().sdattn_qk_stats(ctypes.byref(desc), q.data_ptr(), k.data_ptr(), A.data_ptr(),
                                       LS.data_ptr(), w.data_ptr(), w.numel(), _stream(q.device))
    _lib.check("sdattn_qk_stats", st)
    return A, LS


def softmax_av(a: torch.Tensor, ls: torch.Tensor, v: torch.Tensor, scale: float | None = None,
               out: torch.Tensor | None = None):
    """Partially fused softmax, second kernel: O = (sum_j exp(A_ij - L_i) V_j) / S_i.

    `a` and `ls` as returned by `qk_stats`; v [B,H,M,d]."""
    B, H, M, d = v.shape
    N = a.shape[2]
    if not v.is_cuda:
        raise ValueError("v must live on a CUDA device")
    desc = make_desc(B, H, N, M, d, v.dtype, _scale(scale, d))
    lda = a_ld(desc)
    if a.shape != (B, H, N, lda) or a.dtype != torch.float32 or not a.is_contiguous():
        raise ValueError(f"a must be contiguous fp32 [B,H,N,{lda}]")
    if ls.shape != (B, H, N, 2) or ls.dtype != torch.float32 or not ls.is_contiguous():
        raise ValueError("ls must be contiguous fp32 [B,H,N,2]")
    v = _contig(v)
    O = out if out is not None else torch.empty((B, H, N, d), dtype=v.dtype, device=v.device)
    st = _lib_handle().sdattn_softmax_av(ctypes.byref(desc), a.data_ptr(), ls.data_ptr(), v.data_ptr(),
                                         O.data_ptr(), _stream(v.device))
    _lib.check("sdattn_softmax_av", st)
    return O


def qk_scores(q: torch.Tensor, k: torch.Tensor, scale: float | None = None, out_a: torch.Tensor | None = None):
    """Three-pass variant, first pass: A [B,H,N,lda] fp32 alone (no statistics)."""
    B, H, N, M, d = _check_qk(q, k)
    q, k = _contig(q), _contig(k)
    desc = make_desc(B, H, N, M, d, q.dtype, _scale(scale, d))
    lda = a_ld(desc)
    A = out_a if out_a is not None else torch.empty((B, H, N, lda), dtype=torch.float32, device=q.device)
    if A.shape != (B, H, N, lda) or A.dtype != torch.float32 or not A.is_contiguous():
        raise ValueError(f"out_a must be contiguous fp32 [B,H,N,{lda}]")
    st = _lib_handle().sdattn_qk_scores(ctypes.byref(desc), q.data_ptr(), k.data_ptr(), A.data_ptr(),
                                        _stream(q.device))
    _lib.check("sdattn_qk_scores", st)
    return A


def row_stats(a: torch.Tensor, M: int, d: int, dtype: torch.dtype = torch.float16, out_ls: torch.Tensor | None = None,
              ws: torch.Tensor | None = None):
    """Three-pass variant, second pass: LS [B,H,N,2] = (L_i, S_i) of a stored
    A [B,H,N,lda] (the stand-alone reduction kernel).  `M` is the number of
    valid columns; `d` and `dtype` only complete the call's descriptor."""
    if a.dim() != 4 or a.dtype != torch.float32 or not a.is_contiguous() or not a.is_cuda:
        raise ValueError("a must be a contiguous fp32 CUDA tensor [B,H,N,lda]")
    B, H, N, lda = a.shape
    desc = make_desc(B, H, N, M, d, dtype, 1.0)
    if lda != a_ld(desc):
        raise ValueError(f"a's row stride {lda} does not match M={M}")
    LS = out_ls if out_ls is not None else torch.empty((B, H, N, 2), dtype=torch.float32, device=a.device)
    if LS.shape != (B, H, N, 2) or LS.dtype != torch.float32 or not LS.is_contiguous():
        raise ValueError("out_ls must be contiguous fp32 [B,H,N,2]")
    w = ws if ws is not None else workspace(desc, a.device)
    st = _lib_handle().sdattn_row_stats(ctypes.byref(desc), a.data_ptr(), LS.data_ptr(), w.data_ptr(), w.numel(),
                                        _stream(a.device))
    _lib.check("sdattn_row_stats", st)
    return LS


def qk_stats_f16a(q: torch.Tensor, k: torch.Tensor, scale: float | None = None,
                  out_a: torch.Tensor | None = None, out_ls: torch.Tensor | None = None,
                  ws: torch.Tensor | None = None):
    """fp16-A variant, first kernel: A16 [B,H,N,lda16] fp16 = fp16(scale Q K^T)
    and LS [B,H,N,2], the statistics of the stored values."""
    B, H, N, M, d = _check_qk(q, k)
    q, k = _contig(q), _contig(k)
    desc = make_desc(B, H, N, M, d, q.dtype, _scale(scale, d))
    lda = a16_ld(desc)
    A = out_a if out_a is not None else torch.empty((B, H, N, lda), dtype=torch.float16, device=q.device)
    LS = out_ls if out_ls is not None else torch.empty((B, H, N, 2), dtype=torch.float32, device=q.device)
    if A.shape != (B, H, N, lda) or A.dtype != torch.float16 or not A.is_contiguous():
        raise ValueError(f"out_a must be contiguous fp16 [B,H,N,{lda}]")
    if LS.shape != (B, H, N, 2) or LS.dtype != torch.float32 or not LS.is_contiguous():
        raise ValueError("out_ls must be contiguous fp32 [B,H,N,2]")
    w = ws if ws is not None else workspace(desc, q.device)
    st = _lib_handle().sdattn_qk_stats_f16a(ctypes.byref(desc), q.data_ptr(), k.data_ptr(), A.data_ptr(),
                                            LS.data_ptr(), w.data_ptr(), w.numel(), _stream(q.device))
    _lib.check("sdattn_qk_stats_f16a", st)
    return A, LS


def softmax_av_f16a(a: torch.Tensor, ls: torch.Tensor, v: torch.Tensor, scale: float | None = None,
                    out: torch.Tensor | None = None):
    """fp16-A variant, second kernel: O from A16 and LS as written by `qk_stats_f16a`."""
    B, H, M, d = v.shape
    N = a.shape[2]
    if not v.is_cuda:
        raise ValueError("v must live on a CUDA device")
    desc = make_desc(B, H, N, M, d, v.dtype, _scale(scale, d))
    lda = a16_ld(desc)
    if a.shape != (B, H, N, lda) or a.dtype != torch.float16 or not a.is_contiguous():
        raise ValueError(f"a must be contiguous fp16 [B,H,N,{lda}]")
    if ls.shape != (B, H, N, 2) or ls.dtype != torch.float32 or not ls.is_contiguous():
        raise ValueError("ls must be contiguous fp32 [B,H,N,2]")
    v = _contig(v)
    O = out if out is not None else torch.empty((B, H, N, d), dtype=v.dtype, device=v.device)
    st = _lib_handle().sdattn_softmax_av_f16a(ctypes.byref(desc), a.data_ptr(), ls.data_ptr(), v.data_ptr(),
                                              O.data_ptr(), _stream(v.device))
    _lib.check("sdattn_softmax_av_f16a", st)
    return O


def flash(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, scale: float | None = None,
          out: torch.Tensor | None = None, return_ls: bool = False, out_ls: torch.Tensor | None = None,
          ws: torch.Tensor | None = None, use_workspace: bool = True):
    """FlashAttention form.  Returns O [B,H,N,d] (and LS [B,H,N,2] if asked).

    With a workspace (`ws`, else the cached one) the kernel may cut a block of
    query rows' key range between two CTAs to even out its last wave;
    `use_workspace=False` runs every block of rows whole."""
    B, H, N, M, d = _check_qk(q, k)
    if v.shape != k.shape or v.dtype != q.dtype or not v.is_cuda:
        raise ValueError("v must match k in shape and q in dtype")
    q, k, v = _contig(q), _contig(k), _contig(v)
    desc = make_desc(B, H, N, M, d, q.dtype, _scale(scale, d))
    O = out if out is not None else torch.empty((B, H, N, d), dtype=q.dtype, device=q.device)
    LS = None
    if return_ls or out_ls is not None:
        LS = out_ls if out_ls is not None else torch.empty((B, H, N, 2), dtype=torch.float32, device=q.device)
        if LS.shape != (B, H, N, 2) or LS.dtype != torch.float32 or not LS.is_contiguous():
            raise ValueError("out_ls must be contiguous fp32 [B,H,N,2]")
    w = (ws if ws is not None else workspace(desc, q.device)) if use_workspace else None
    st = _lib_handle().sdattn_flash(ctypes.byref(desc), q.data_ptr(), k.data_ptr(), v.data_ptr(), O.data_ptr(),
                                    LS.data_ptr() if LS is not None else None,
                                    w.data_ptr() if w is not None else None, w.numel() if w is not None else 0,
                                    _stream(q.device))
    _lib.check("sdattn_flash", st)
    return (O, LS) if (return_ls or out_ls is not None) else O


def flash_f32o(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, scale: float | None = None,
               out: torch.Tensor | None = None, return_ls: bool = False):
    """FlashAttention form with an fp32 O and P carried as two 16-bit parts:
    the form that holds bf16 inputs to the fp16 accuracy bar.  Returns O
    [B,H,N,d] float32 (and LS if asked)."""
    B, H, N, M, d = _check_qk(q, k)
    if v.shape != k.shape or v.dtype != q.dtype or not v.is_cuda:
        raise ValueError("v must match k in shape and q in dtype")
    q, k, v = _contig(q), _contig(k), _contig(v)
    desc = make_desc(B, H, N, M, d, q.dtype, _scale(scale, d))
    O = out if out is not None else torch.empty((B, H, N, d), dtype=torch.float32, device=q.device)
    if O.shape != (B, H, N, d) or O.dtype != torch.float32 or not O.is_contiguous():
        raise ValueError("out must be contiguous fp32 [B,H,N,d]")
    LS = torch.empty((B, H, N, 2), dtype=torch.float32, device=q.device) if return_ls else None
    st = _lib_handle().sdattn_flash_f32o(ctypes.byref(desc), q.data_ptr(), k.data_ptr(), v.data_ptr(), O.data_ptr(),
                                         LS.data_ptr() if LS is not None else None, _stream(q.device))
    _lib.check("sdattn_flash_f32o", st)
    return (O, LS) if return_ls else O


def flash_tf32(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, scale: float | None = None,
               out: torch.Tensor | None = None, return_ls: bool = False):
    """FlashAttention form for fp32 q, k, v [B,H,*,d], read natively (tf32
    tensor-core products, fp32 sums); returns O [B,H,N,d] float32 (and LS if
    asked)."""
    B, H, N, M, d = _check_qk(q, k)
    if q.dtype != torch.float32 or v.dtype != torch.float32 or v.shape != k.shape or not v.is_cuda:
        raise TypeError("q, k, v must be float32 CUDA tensors, v shaped like k")
    q, k, v = _contig(q), _contig(k), _contig(v)
    desc = _lib.Desc(B, H, N, M, d, _lib.SDATTN_F32, float(_scale(scale, d)))
    O = out if out is not None else torch.empty((B, H, N, d), dtype=torch.float32, device=q.device)
    if O.shape != (B, H, N, d) or O.dtype != torch.float32 or not O.is_contiguous():
        raise ValueError("out must be contiguous fp32 [B,H,N,d]")
    LS = torch.empty((B, H, N, 2), dtype=torch.float32, device=q.device) if return_ls else None
    st = _lib_handle().sdattn_flash_tf32(ctypes.byref(desc), q.data_ptr(), k.data_ptr(), v.data_ptr(), O.data_ptr(),
                                         LS.data_ptr() if LS is not None else None, _stream(q.device))
    _lib.check("sdattn_flash_tf32", st)
    return (O, LS) if return_ls else O


def partially_fused(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, scale: float | None = None,
                    variant: str = "fused"):
    """The partially fused form; returns O.

    variant "fused": qk_stats then softmax_av (statistics in the QK^T epilogue);
    "three_pass": qk_scores, row_stats, softmax_av (the stand-alone reduction);
    "f16a": qk_stats_f16a then softmax_av_f16a (A stored in fp16)."""
    if variant == "fused":
        A, LS = qk_stats(q, k, scale)
        return softmax_av(A, LS, v, scale)
    if variant == "three_pass":
        A = qk_scores(q, k, scale)
        LS = row_stats(A, k.shape[2], q.shape[3], q.dtype)
        return softmax_av(A, LS, v, scale)
    if variant == "f16a":
        A, LS = qk_stats_f16a(q, k, scale)
        return softmax_av_f16a(A, LS, v, scale)
    raise ValueError(f"unknown variant {variant!r}")


def group_norm(x: torch.Tensor, gamma: torch.Tensor, beta: torch.Tensor, groups: int, eps: float = 1e-6,
               out: torch.Tensor | None = None):
    """Group normalisation of x [B, C, H, W] (fp16 or bf16, NCHW) with
    per-channel fp32 gamma, beta [C], in one launch."""
    if x.dim() != 4 or not x.is_cuda:
        raise ValueError("x must be a CUDA tensor [B, C, H, W]")
    if x.dtype not in _DTYPES:
        raise TypeError(f"dtype {x.dtype} not supported (float16 or bfloat16)")
    B, C, H, W = x.shape
    gamma = _contig(gamma.to(device=x.device, dtype=torch.float32))
    beta = _contig(beta.to(device=x.device, dtype=torch.float32))
    if gamma.shape != (C,) or beta.shape != (C,):
        raise ValueError("gamma and beta must be [C]")
    x = _contig(x)
    Y = out if out is not None else torch.empty_like(x)
    if Y.shape != x.shape or Y.dtype != x.dtype or not Y.is_contiguous():
        raise ValueError("out must match x")
    desc = _lib.GNDesc(B, C, H, W, int(groups), _DTYPES[x.dtype], float(eps))
    st = _lib_handle().sdattn_group_norm(ctypes.byref(desc), x.data_ptr(), gamma.data_ptr(), beta.data_ptr(),
                                         Y.data_ptr(), _stream(x.device))
    _lib.check("sdattn_group_norm", st)
    return Y


def geglu(x: torch.Tensor, out: torch.Tensor | None = None):
    """The UNet's gated GELU: x [..., 2F] -> x[..., :F] * GELU(x[..., F:]) in one launch."""
    if not x.is_cuda or x.dtype not in _DTYPES:
        raise ValueError("x must be a float16 or bfloat16 CUDA tensor")
    F = x.shape[-1] // 2
    if x.shape[-1] != 2 * F:
        raise ValueError("the last dimension must be even")
    x = _contig(x)
    T = x.numel() // (2 * F)
    Y = out if out is not None else torch.empty(x.shape[:-1] + (F,), dtype=x.dtype, device=x.device)
    if Y.numel() != T * F or Y.dtype != x.dtype or not Y.is_contiguous():
        raise ValueError("out must hold x.shape[:-1] + (F,) values of x's dtype")
    st = _lib_handle().sdattn_geglu(T, F, _DTYPES[x.dtype], x.data_ptr(), Y.data_ptr(), _stream(x.device))
    _lib.check("sdattn_geglu", st)
    return Y


def _conv_desc(N, C, K, H, W, dtype) -> _lib.ConvDesc:
    if dtype not in _DTYPES:
        raise TypeError(f"dtype {dtype} not supported (float16 or bfloat16)")
    return _lib.ConvDesc(N, C, K, H, W, _DTYPES[dtype])


def wino_filter(w: torch.Tensor, out: torch.Tensor | None = None):
    """Winograd F(4x4, 3x3) filter transform of w [K, C, 3, 3] (fp16 or bf16):
    U [36, K, C] of w's dtype, computed once per filter."""
    if w.dim() != 4 or w.shape[2:] != (3, 3) or not w.is_cuda:
        raise ValueError("w must be a CUDA tensor [K, C, 3, 3]")
    K, C = w.shape[:2]
    w = _contig(w)
    desc = _conv_desc(1, C, K, 4, 4, w.dtype)
    U = out if out is not None else torch.empty(36, K, C, dtype=w.dtype, device=w.device)
    if U.shape != (36, K, C) or U.dtype != w.dtype or not U.is_contiguous():
        raise ValueError("out must be [36, K, C] of w's dtype")
    st = _lib_handle().sdattn_wino_filter(ctypes.byref(desc), w.data_ptr(), U.data_ptr(), _stream(w.device))
    _lib.check("sdattn_wino_filter", st)
    return U


def conv3x3_winograd(x: torch.Tensor, U: torch.Tensor, bias: torch.Tensor | None = None,
                     out: torch.Tensor | None = None, ws: torch.Tensor | None = None):
    """The UNet's 3x3 convolution (stride 1, zero padding 1) of x [N, C, H, W]
    with a filter transformed by `wino_filter`, plus an optional fp32 bias [K]:
    input transform, batched tensor-core product, output transform."""
    if x.dim() != 4 or not x.is_cuda:
        raise ValueError("x must be a CUDA tensor [N, C, H, W]")
    N, C, H, W = x.shape
    if U.dim() != 3 or U.shape[0] != 36 or U.shape[2] != C or U.dtype != x.dtype:
        raise ValueError("U must be wino_filter's [36, K, C] of x's dtype")
    K = U.shape[1]
    desc = _conv_desc(N, C, K, H, W, x.dtype)
    need = _lib_handle().sdattn_wino_workspace_bytes(ctypes.byref(desc))
    if need == 0:
        raise _lib.SdattnError("sdattn_wino_workspace_bytes", 2)
    if ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device=x.device)
    if bias is not None:
        bias = _contig(bias.to(device=x.device, dtype=torch.float32))
        if bias.shape != (K,):
            raise ValueError("bias must be [K]")
    x, U = _contig(x), _contig(U)
    Y = out if out is not None else torch.empty(N, K, H, W, dtype=x.dtype, device=x.device)
    if Y.shape != (N, K, H, W) or Y.dtype != x.dtype or not Y.is_contiguous():
        raise ValueError("out must be [N, K, H, W] of x's dtype")
    st = _lib_handle().sdattn_wino_conv3x3(ctypes.byref(desc), x.data_ptr(), U.data_ptr(),
                                           bias.data_ptr() if bias is not None else None, Y.data_ptr(),
                                           ws.data_ptr(), ws.numel() * ws.element_size(), _stream(x.device))
    _lib.check("sdattn_wino_conv3x3", st)
    return Y


def wino_workspace_bytes(N: int, C: int, K: int, H: int, W: int, dtype=torch.float16) -> int:
    return int(_lib_handle().sdattn_wino_workspace_bytes(ctypes.byref(_conv_desc(N, C, K, H, W, dtype))))


def device_error():
    """(status name, detail code) of the device error word; reading clears it.

    After a timeout the cached workspaces are zero-filled anew, since the
    abandoned calls may have left counters or partials in them."""
    detail = ctypes.c_uint32(0)
    st = _lib_handle().sdattn_device_error(ctypes.byref(detail))
    if _lib.STATUS.get(st) == "SDATTN_ERR_TIMEOUT":
        for ws in _workspaces.values():
            ws.zero_()
    return _lib.STATUS.get(st, st), int(detail.value)
