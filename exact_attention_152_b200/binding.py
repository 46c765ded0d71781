"""ctypes binding over libattn.so (include/attn.h).

The C functions keep their names and arguments: pointers are Python ints (or
None), sizes ints, the stream a raw ``cudaStream_t`` handle as an int.  They
return the library's status code.  ``fwd`` is the one convenience wrapper: it
allocates O and LSE with torch, passes ``data_ptr()`` and the current stream,
and raises ``AttnError`` on a non-zero status.  No arithmetic happens here.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libattn.so")

ATTN_OK = 0
ATTN_ERR_INVALID_ARG = 1
ATTN_ERR_UNSUPPORTED = 2
ATTN_ERR_CUDA = 3
ATTN_ERR_TIMEOUT = 4

EXP_MUFU, EXP_SPLIT, EXP_POLY = 0, 1, 2

_lock = threading.Lock()
_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int


def lib() -> ctypes.CDLL:
    """Load libattn.so once; raise ImportError if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"{LIB_PATH} is missing: build it with "
                                  "`python -m exact_attention_152_b200.build` (there is no fallback)")
            l = ctypes.CDLL(LIB_PATH)
            l.attn_fwd.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, ctypes.c_float, _I, _P]
            l.attn_fwd.restype = _I
            l.attn_fwd_config.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, ctypes.c_float, _I,
                                          ctypes.c_float, _I, _P, _P]
            l.attn_fwd_config.restype = _I
            l.attn_fwd_gqa.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, ctypes.c_float, _I,
                                       _P]
            l.attn_fwd_gqa.restype = _I
            l.attn_fwd_window.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I,
                                          ctypes.c_float, _I, _I, _P]
            l.attn_fwd_window.restype = _I
            l.attn_fwd_colmask.argtypes = [_P, _P, _P, _P, _P] + [_I] * 6 + [ctypes.c_float, _I, _P, _I,
                                                                          _P, ctypes.c_size_t, _P]
            l.attn_fwd_colmask.restype = _I
            l.attn_colmask_workspace_size.argtypes = [_I, _I, _I]
            l.attn_colmask_workspace_size.restype = ctypes.c_size_t
            l.attn_fwd_varlen.argtypes = [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I,
                                          ctypes.c_float, _I, _I, _P]
            l.attn_fwd_varlen.restype = _I
            l.attn_fwd_fp8.argtypes = [_P, _P, _P, _P, _P] + [_I] * 6 + [ctypes.c_float] * 4 + [_I, _P]
            l.attn_fwd_fp8.restype = _I
            l.attn_bwd.argtypes = [_P] * 10 + [ctypes.c_size_t] + [_I] * 6 + [ctypes.c_float, _I, _P]
            l.attn_bwd.restype = _I
            l.attn_bwd_window.argtypes = [_P] * 10 + [ctypes.c_size_t] + [_I] * 6 + [ctypes.c_float, _I, _I, _P]
            l.attn_bwd_window.restype = _I
            l.attn_bwd_varlen.argtypes = [_P] * 10 + [ctypes.c_size_t, _P, _P] + [_I] * 7 + \
                [ctypes.c_float, _I, _I, _P]
            l.attn_bwd_varlen.restype = _I
            l.attn_bwd_colmask.argtypes = [_P] * 10 + [ctypes.c_size_t] + [_I] * 6 + \
                [ctypes.c_float, _I, _P, _I, _P]
            l.attn_bwd_colmask.restype = _I
            l.attn_bwd_colmask_workspace_size.argtypes = [_I] * 6
            l.attn_bwd_colmask_workspace_size.restype = ctypes.c_size_t
            l.attn_bwd_noalloc.argtypes = [_P] * 9 + [_I] * 6 + [ctypes.c_float, _I, _P]
            l.attn_bwd_noalloc.restype = _I
            l.attn_bwd_workspace_size.argtypes = [_I, _I, _I, _I]
            l.attn_bwd_workspace_size.restype = ctypes.c_size_t
            l.attn_status_sync.argtypes = [_P]
            l.attn_status_sync.restype = _I
            l.attn_status_string.argtypes = [_I]
            l.attn_status_string.restype = ctypes.c_char_p
            l.attn_last_error.argtypes = []
            l.attn_last_error.restype = ctypes.c_char_p
            l.attn_selftest_timeout.argtypes = [ctypes.c_uint, _P]
            l.attn_selftest_timeout.restype = _I
            _lib = l
    return _lib


def attn_fwd(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, stream) -> int:
    return lib().attn_fwd(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, stream)


def attn_fwd_gqa(q, k, v, o, lse, B, H, Hkv, Nq, Nk, d, scale, causal, stream) -> int:
    return lib().attn_fwd_gqa(q, k, v, o, lse, B, H, Hkv, Nq, Nk, d, scale, causal, stream)


def attn_fwd_window(q, k, v, o, lse, B, H, Hkv, Nq, Nk, d, scale, window_left, window_right,
                    stream) -> int:
    return lib().attn_fwd_window(q, k, v, o, lse, B, H, Hkv, Nq, Nk, d, scale, window_left,
                                 window_right, stream)


def attn_fwd_colmask(q, k, v, o, lse, B, H, Hkv, Nq, Nk, d, scale, causal, mask, Hm, workspace,
                     workspace_bytes, stream) -> int:
    return lib().attn_fwd_colmask(q, k, v, o, lse, B, H, Hkv, Nq, Nk, d, scale, causal, mask, Hm,
                                  workspace, workspace_bytes, stream)


def attn_colmask_workspace_size(B, Hm, Nk) -> int:
    return lib().attn_colmask_workspace_size(B, Hm, Nk)


def attn_fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, num_seqs, max_seqlen_q, total_q,
                    total_k, H, Hkv, d, scale, window_left, window_right, stream) -> int:
    return lib().attn_fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, num_seqs,
                                 max_seqlen_q, total_q, total_k, H, Hkv, d, scale, window_left,
                                 window_right, stream)


def attn_fwd_fp8(q, k, v, o, lse, B, H, Hkv, Nq, Nk, d, scale, q_descale, k_descale, v_descale,
                 causal, stream) -> int:
    return lib().attn_fwd_fp8(q, k, v, o, lse, B, H, Hkv, Nq, Nk, d, scale, q_descale, k_descale,
                              v_descale, causal, stream)


def attn_fwd_config(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, rescale_threshold,
                    exp_mode, rescale_count, stream) -> int:
    return lib().attn_fwd_config(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal,
                                 rescale_threshold, exp_mode, rescale_count, stream)


def attn_bwd(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, B, H, Hkv, Nq, Nk, d,
             scale, causal, stream) -> int:
    return lib().attn_bwd(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, B, H, Hkv,
                          Nq, Nk, d, scale, causal, stream)


def attn_bwd_window(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, B, H, Hkv, Nq, Nk,
                    d, scale, window_left, window_right, stream) -> int:
    return lib().attn_bwd_window(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, B, H,
                                 Hkv, Nq, Nk, d, scale, window_left, window_right, stream)


def attn_bwd_colmask(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, B, H, Hkv, Nq, Nk,
                     d, scale, causal, mask, Hm, stream) -> int:
    return lib().attn_bwd_colmask(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, B, H,
                                  Hkv, Nq, Nk, d, scale, causal, mask, Hm, stream)


def attn_bwd_colmask_workspace_size(B, H, Nq, d, Hm, Nk) -> int:
    return lib().attn_bwd_colmask_workspace_size(B, H, Nq, d, Hm, Nk)


def attn_bwd_varlen(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, cu_seqlens_q,
                    cu_seqlens_k, num_seqs, max_seqlen_k, total_q, total_k, H, Hkv, d, scale,
                    window_left, window_right, stream) -> int:
    return lib().attn_bwd_varlen(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes,
                                 cu_seqlens_q, cu_seqlens_k, num_seqs, max_seqlen_k, total_q, total_k,
                                 H, Hkv, d, scale, window_left, window_right, stream)


def attn_bwd_noalloc(q, k, v, o, dout, lse, dq, dk, dv, B, H, Hkv, Nq, Nk, d, scale, causal,
                     stream) -> int:
    return lib().attn_bwd_noalloc(q, k, v, o, dout, lse, dq, dk, dv, B, H, Hkv, Nq, Nk, d, scale,
                                  causal, stream)


def attn_bwd_workspace_size(B, H, Nq, d) -> int:
    return lib().attn_bwd_workspace_size(B, H, Nq, d)


def attn_status_sync(stream) -> int:
    return lib().attn_status_sync(stream)


def attn_status_string(code: int) -> str:
    return lib().attn_status_string(code).decode()


def attn_last_error() -> str:
    return lib().attn_last_error().decode()


def attn_selftest_timeout(timeout_us: int, stream) -> int:
    return lib().attn_selftest_timeout(timeout_us, stream)


class AttnError(RuntimeError):
    def __init__(self, code: int, where: str):
        msg = f"{where}: {attn_status_string(code)} ({code})"
        if code == ATTN_ERR_CUDA:
            msg += f": {attn_last_error()}"
        super().__init__(msg)
        self.code = code


def check(code: int, where: str = "attn") -> None:
    if code != ATTN_OK:
        raise AttnError(code, where)


def _check_bf16(**tensors):
    import torch
    for name, t in tensors.items():
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or not t.is_cuda:
            raise TypeError(f"{name} must be a bfloat16 CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")


def fwd(q, k, v, causal: bool = False, scale: float | None = None, *, window=None, out=None,
        lse=None, return_lse: bool = True, rescale_threshold: float | None = None,
        exp_mode: int | None = None, rescale_count=None):
    """O (and LSE) for BF16 CUDA tensors q [B,H,Nq,d], k/v [B,Hkv,Nk,d].

    Hkv < H (H % Hkv == 0) selects grouped-query attention (attn_fwd_gqa).
    window=(left, right) selects the key band of attn_fwd_window (-1: no bound;
    it replaces ``causal``).  scale defaults to 1/sqrt(d).  Runs on torch's
    current stream; returns (o, lse) or o.  Raises AttnError on any non-zero status.
    """
    import torch

    for name, t in (("q", q), ("k", k), ("v", v)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or not t.is_cuda:
            raise TypeError(f"{name} must be a bfloat16 CUDA tensor")
        if t.dim() != 4 or not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous [B, H, N, d]")
    B, H, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if tuple(k.shape) != (B, Hkv, Nk, d) or tuple(v.shape) != (B, Hkv, Nk, d):
        raise ValueError("k and v must be [B, Hkv, Nk, d] matching q")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, H, Nq, d), dtype=torch.bfloat16, device=q.device)
    if return_lse and lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    stream = torch.cuda.current_stream(q.device).cuda_stream
    lse_ptr = lse.data_ptr() if lse is not None else None
    knobs = rescale_threshold is not None or exp_mode is not None or rescale_count is not None
    if window is not None:
        if causal or knobs:
            raise ValueError("window replaces causal and takes no softmax knobs")
        rc = attn_fwd_window(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse_ptr,
                             B, H, Hkv, Nq, Nk, d, float(scale), int(window[0]), int(window[1]),
                             stream)
        check(rc, "attn_fwd_window")
        return (out, lse) if return_lse else out
    if Hkv != H:
        if rescale_threshold is not None or exp_mode is not None or rescale_count is not None:
            raise ValueError("the softmax knobs are available for Hkv == H only")
        rc = attn_fwd_gqa(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse_ptr,
                          B, H, Hkv, Nq, Nk, d, float(scale), int(bool(causal)), stream)
    elif rescale_threshold is None and exp_mode is None and rescale_count is None:
        rc = attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse_ptr,
                      B, H, Nq, Nk, d, float(scale), int(bool(causal)), stream)
    else:
        rc = attn_fwd_config(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse_ptr,
                             B, H, Nq, Nk, d, float(scale), int(bool(causal)),
                             8.0 if rescale_threshold is None else float(rescale_threshold),
                             EXP_SPLIT if exp_mode is None else int(exp_mode),
                             rescale_count.data_ptr() if rescale_count is not None else None,
                             stream)
    check(rc, "attn_fwd")
    return (out, lse) if return_lse else out


def fwd_colmask(q, k, v, mask, causal: bool = False, scale: float | None = None, *,
                workspace=None, out=None, lse=None):
    """attn_fwd_colmask on BF16 CUDA tensors q [B,H,Nq,d], k/v [B,Hkv,Nk,d] and
    an int32 CUDA mask [B, Hm, Nk, 4] (Hm = 1 or H): key j is hidden from query
    rows [mask[..., j, 0], mask[..., j, 1]) and [mask[..., j, 2], mask[..., j, 3]),
    and from rows i < j when causal.  workspace: a uint8 CUDA tensor of at least
    attn_colmask_workspace_size(B, Hm, Nk) bytes (allocated when None).
    Returns (o, lse) on torch's current stream."""
    import torch

    _check_bf16(q=q, k=k, v=v)
    B, H, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if tuple(k.shape) != (B, Hkv, Nk, d) or tuple(v.shape) != (B, Hkv, Nk, d):
        raise ValueError("k and v must be [B, Hkv, Nk, d] matching q")
    if not isinstance(mask, torch.Tensor) or mask.dtype != torch.int32 or not mask.is_cuda:
        raise TypeError("mask must be an int32 CUDA tensor")
    if mask.dim() != 4 or mask.shape[0] != B or mask.shape[2] != Nk or mask.shape[3] != 4 \
            or not mask.is_contiguous():
        raise ValueError("mask must be contiguous [B, Hm, Nk, 4]")
    Hm = mask.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    ws_bytes = attn_colmask_workspace_size(B, Hm, Nk)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty((B, H, Nq, d), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    stream = torch.cuda.current_stream(q.device).cuda_stream
    rc = attn_fwd_colmask(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                          B, H, Hkv, Nq, Nk, d, float(scale), int(bool(causal)), mask.data_ptr(), Hm,
                          workspace.data_ptr(), workspace.numel(), stream)
    check(rc, "attn_fwd_colmask")
    return out, lse


def fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, causal: bool = False,
               scale: float | None = None, *, window=None, out=None, lse=None,
               return_lse: bool = True):
    """Packed variable-length batch: q [total_q, H, d], k/v [total_k, Hkv, d]
    BF16 CUDA tensors, cu_seqlens_* int32 CUDA tensors of num_seqs + 1 offsets.
    Returns (o [total_q, H, d], lse [H, total_q]) or o.  ``window`` = (left,
    right) band over positions within each sequence (replaces ``causal``)."""
    import torch

    _check_bf16(q=q, k=k, v=v)
    if q.dim() != 3 or k.dim() != 3 or v.dim() != 3:
        raise ValueError("q, k, v must be [total, heads, d]")
    total_q, H, d = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    if tuple(k.shape) != (total_k, Hkv, d) or tuple(v.shape) != (total_k, Hkv, d):
        raise ValueError("k and v must be [total_k, Hkv, d] matching q")
    for name, c in (("cu_seqlens_q", cu_seqlens_q), ("cu_seqlens_k", cu_seqlens_k)):
        if not isinstance(c, torch.Tensor) or c.dtype != torch.int32 or not c.is_cuda \
                or c.dim() != 1 or not c.is_contiguous():
            raise TypeError(f"{name} must be a contiguous int32 CUDA vector")
    if cu_seqlens_q.numel() != cu_seqlens_k.numel() or cu_seqlens_q.numel() < 1:
        raise ValueError("cu_seqlens_q and cu_seqlens_k need the same num_seqs + 1 entries")
    num_seqs = cu_seqlens_q.numel() - 1
    if window is None:
        window = (-1, 0) if causal else (-1, -1)
    elif causal:
        raise ValueError("window replaces causal")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((total_q, H, d), dtype=torch.bfloat16, device=q.device)
    if return_lse and lse is None:
        lse = torch.empty((H, total_q), dtype=torch.float32, device=q.device)
    stream = torch.cuda.current_stream(q.device).cuda_stream
    rc = attn_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                         lse.data_ptr() if lse is not None else None, cu_seqlens_q.data_ptr(),
                         cu_seqlens_k.data_ptr(), num_seqs, int(max_seqlen_q), total_q, total_k,
                         H, Hkv, d, float(scale), int(window[0]), int(window[1]), stream)
    check(rc, "attn_fwd_varlen")
    return (out, lse) if return_lse else out


def bwd(q, k, v, o, dout, lse, causal: bool = False, scale: float | None = None, *,
        window=None, workspace=None):
    """Gradients (dq, dk, dv) for BF16 CUDA tensors q/o/dout [B,H,Nq,d], k/v
    [B,Hkv,Nk,d] and the forward's fp32 lse [B,H,Nq].  window=(left, right)
    selects the key band of attn_bwd_window (it replaces ``causal``).  The
    workspace (a uint8 CUDA tensor of at least attn_bwd_workspace_size bytes)
    is allocated with torch when not given.  Runs on torch's current stream."""
    import torch

    _check_bf16(q=q, k=k, v=v, o=o, dout=dout)
    B, H, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if tuple(o.shape) != tuple(q.shape) or tuple(dout.shape) != tuple(q.shape):
        raise ValueError("o and dout must match q")
    if tuple(k.shape) != (B, Hkv, Nk, d) or tuple(v.shape) != (B, Hkv, Nk, d):
        raise ValueError("k and v must be [B, Hkv, Nk, d] matching q")
    if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (B, H, Nq):
        raise ValueError("lse must be contiguous float32 [B, H, Nq]")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = attn_bwd_workspace_size(B, H, Nq, d)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    stream = torch.cuda.current_stream(q.device).cuda_stream
    ptrs = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(), lse.data_ptr(),
            dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(),
            workspace.numel() * workspace.element_size())
    if window is not None:
        if causal:
            raise ValueError("window replaces causal")
        rc = attn_bwd_window(*ptrs, B, H, Hkv, Nq, Nk, d, float(scale), int(window[0]),
                             int(window[1]), stream)
        check(rc, "attn_bwd_window")
    else:
        rc = attn_bwd(*ptrs, B, H, Hkv, Nq, Nk, d, float(scale), int(bool(causal)), stream)
        check(rc, "attn_bwd")
    return dq, dk, dv


def bwd_colmask(q, k, v, o, dout, lse, mask, causal: bool = False, scale: float | None = None, *,
                workspace=None):
    """Gradients (dq, dk, dv) of fwd_colmask for BF16 CUDA tensors q/o/dout
    [B,H,Nq,d], k/v [B,Hkv,Nk,d], fp32 lse [B,H,Nq] and the int32 CUDA mask
    [B, Hm, Nk, 4].  The workspace is allocated when not given.  Runs on
    torch's current stream."""
    import torch

    _check_bf16(q=q, k=k, v=v, o=o, dout=dout)
    B, H, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if tuple(o.shape) != tuple(q.shape) or tuple(dout.shape) != tuple(q.shape):
        raise ValueError("o and dout must match q")
    if tuple(k.shape) != (B, Hkv, Nk, d) or tuple(v.shape) != (B, Hkv, Nk, d):
        raise ValueError("k and v must be [B, Hkv, Nk, d] matching q")
    if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (B, H, Nq):
        raise ValueError("lse must be contiguous float32 [B, H, Nq]")
    if not isinstance(mask, torch.Tensor) or mask.dtype != torch.int32 or not mask.is_cuda \
            or mask.dim() != 4 or mask.shape[0] != B or mask.shape[2] != Nk or mask.shape[3] != 4 \
            or not mask.is_contiguous():
        raise ValueError("mask must be a contiguous int32 CUDA tensor [B, Hm, Nk, 4]")
    Hm = mask.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = attn_bwd_colmask_workspace_size(B, H, Nq, d, Hm, Nk)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    stream = torch.cuda.current_stream(q.device).cuda_stream
    rc = attn_bwd_colmask(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(),
                          lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                          workspace.data_ptr(), workspace.numel() * workspace.element_size(), B, H,
                          Hkv, Nq, Nk, d, float(scale), int(bool(causal)), mask.data_ptr(), Hm, stream)
    check(rc, "attn_bwd_colmask")
    return dq, dk, dv


def bwd_varlen(q, k, v, o, dout, lse, cu_seqlens_q, cu_seqlens_k, max_seqlen_k: int,
               causal: bool = False, scale: float | None = None, *, window=None, workspace=None):
    """Gradients (dq, dk, dv) of fwd_varlen: q/o/dout [total_q, H, d], k/v
    [total_k, Hkv, d] BF16 CUDA tensors, lse [H, total_q] fp32, int32 CUDA
    offsets.  ``window`` = (left, right) replaces ``causal``.  The workspace
    (attn_bwd_workspace_size(1, H, total_q, d) bytes) is allocated when not
    given.  Key rows that belong to no sequence are left as torch.empty made
    them.  Runs on torch's current stream."""
    import torch

    _check_bf16(q=q, k=k, v=v, o=o, dout=dout)
    if q.dim() != 3 or k.dim() != 3 or v.dim() != 3:
        raise ValueError("q, k, v must be [total, heads, d]")
    total_q, H, d = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    if tuple(o.shape) != tuple(q.shape) or tuple(dout.shape) != tuple(q.shape):
        raise ValueError("o and dout must match q")
    if tuple(k.shape) != (total_k, Hkv, d) or tuple(v.shape) != (total_k, Hkv, d):
        raise ValueError("k and v must be [total_k, Hkv, d] matching q")
    if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (H, total_q):
        raise ValueError("lse must be contiguous float32 [H, total_q]")
    for name, c in (("cu_seqlens_q", cu_seqlens_q), ("cu_seqlens_k", cu_seqlens_k)):
        if not isinstance(c, torch.Tensor) or c.dtype != torch.int32 or not c.is_cuda \
                or c.dim() != 1 or not c.is_contiguous():
            raise TypeError(f"{name} must be a contiguous int32 CUDA vector")
    if cu_seqlens_q.numel() != cu_seqlens_k.numel() or cu_seqlens_q.numel() < 1:
        raise ValueError("cu_seqlens_q and cu_seqlens_k need the same num_seqs + 1 entries")
    num_seqs = cu_seqlens_q.numel() - 1
    if window is None:
        window = (-1, 0) if causal else (-1, -1)
    elif causal:
        raise ValueError("window replaces causal")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = attn_bwd_workspace_size(1, H, total_q, d)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    stream = torch.cuda.current_stream(q.device).cuda_stream
    rc = attn_bwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(),
                         lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                         workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                         cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), num_seqs,
                         int(max_seqlen_k), total_q, total_k, H, Hkv, d, float(scale),
                         int(window[0]), int(window[1]), stream)
    check(rc, "attn_bwd_varlen")
    return dq, dk, dv


def fwd_fp8(q, k, v, descale=(1.0, 1.0, 1.0), causal: bool = False, scale: float | None = None):
    """FP8 forward: q [B,H,Nq,d], k/v [B,Hkv,Nk,d] uint8 CUDA tensors of E4M3
    codes (or torch.float8_e4m3fn), descale = (q, k, v) scale factors.
    Returns (o BF16 [B,H,Nq,d], lse fp32 [B,H,Nq])."""
    import torch

    for name, t in (("q", q), ("k", k), ("v", v)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda or t.element_size() != 1 \
                or t.dim() != 4 or not t.is_contiguous():
            raise TypeError(f"{name} must be a contiguous 4-D one-byte CUDA tensor of E4M3 codes")
    B, H, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if tuple(k.shape) != (B, Hkv, Nk, d) or tuple(v.shape) != (B, Hkv, Nk, d):
        raise ValueError("k and v must be [B, Hkv, Nk, d] matching q")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = torch.empty((B, H, Nq, d), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    stream = torch.cuda.current_stream(q.device).cuda_stream
    rc = attn_fwd_fp8(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H,
                      Hkv, Nq, Nk, d, float(scale), *(float(x) for x in descale), int(bool(causal)),
                      stream)
    check(rc, "attn_fwd_fp8")
    return o, lse
