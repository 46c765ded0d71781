"""Exact scaled dot-product attention forward for B200 (sm_100a).

The compute path is the C-ABI library ``libattn.so`` (hand-written CUDA:
TMA loads, tcgen05 MMAs into Tensor Memory, online softmax).  This package is a
thin ctypes binding over it; PyTorch is used only for device memory and streams.

The binding is loaded on first use; if ``libattn.so`` is missing the first call
raises ImportError -- there is no fallback of any kind.
"""
from __future__ import annotations

__all__ = [
    "attn_fwd", "attn_fwd_config", "attn_fwd_gqa", "attn_fwd_window", "attn_fwd_varlen",
    "attn_status_sync", "attn_status_string", "attn_last_error", "attn_selftest_timeout", "fwd",
    "fwd_varlen", "attn_fwd_fp8", "fwd_fp8", "attn_bwd", "attn_bwd_window", "attn_bwd_workspace_size", "bwd", "AttnError",
]


def __getattr__(name):
    if name in __all__:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
