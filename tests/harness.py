"""Shared helpers for the parity tests: seeded inputs -> CUDA path and oracle.

The CUDA side is reached only through the C-ABI (exact_attention_152_b200.binding);
the oracle side only through ``oracle``.  They share nothing but the input bits.
"""
from __future__ import annotations

import numpy as np

import oracle
from exact_attention_152_b200 import inputs

# Tolerances of the forward output against the fp64 oracle (BF16 inputs, BF16 O):
MAX_ABS_O = 1e-2
MEAN_ABS_O = 1e-3
MAX_ABS_LSE = 1e-3


def to_device_bf16(bits: np.ndarray):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def run_cuda(q_bits, k_bits, v_bits, scale, causal, **kw):
    """Run attn_fwd (or attn_fwd_config when knobs are given) via the C-ABI.
    Returns (o fp32 numpy, lse numpy)."""
    import torch

    from exact_attention_152_b200 import binding
    q, k, v = (to_device_bf16(x) for x in (q_bits, k_bits, v_bits))
    o, lse = binding.fwd(q, k, v, causal=causal, scale=scale, **kw)
    rc = binding.attn_status_sync(torch.cuda.current_stream().cuda_stream)
    assert rc == 0, f"device status {rc}"
    return o.float().cpu().numpy(), lse.cpu().numpy()


def run_varlen(q_bits, k_bits, v_bits, cu_q, cu_k, max_q, scale, window):
    """Run attn_fwd_varlen via the C-ABI on packed bits (q [total_q, H, d], k/v
    [total_k, Hkv, d], int32 offsets).  Returns (o fp32 numpy, lse numpy [H, total_q])."""
    import torch

    from exact_attention_152_b200 import binding
    q, k, v = (to_device_bf16(x) for x in (q_bits, k_bits, v_bits))
    cq = torch.from_numpy(np.asarray(cu_q, dtype=np.int32)).cuda()
    ck = torch.from_numpy(np.asarray(cu_k, dtype=np.int32)).cuda()
    o, lse = binding.fwd_varlen(q, k, v, cq, ck, max_q, scale=scale, window=window)
    rc = binding.attn_status_sync(torch.cuda.current_stream().cuda_stream)
    assert rc == 0, f"device status {rc}"
    return o.float().cpu().numpy(), lse.cpu().numpy()


def oracle_rows(q_bits, k_bits, v_bits, scale, causal, rows_per_head=None, kv_group=1, band=None):
    """Oracle on selected rows of every (b, h).  rows_per_head: dict bh -> rows or None (all).
    kv_group > 1: query head h reads key/value head h // kv_group.  band: (left,
    right) key band replacing ``causal`` (-1 = no bound)."""
    if band is None:
        band = (-1, 0) if causal else (-1, -1)
    B, H, Nq, d = q_bits.shape
    out = {}
    for b in range(B):
        for h in range(H):
            bh = b * H + h
            rows = np.arange(Nq, dtype=np.int64) if rows_per_head is None else rows_per_head[bh]
            q = inputs.bf16_bits_to_f64(q_bits[b, h, rows])
            k = inputs.bf16_bits_to_f64(k_bits[b, h // kv_group])
            v = inputs.bf16_bits_to_f64(v_bits[b, h // kv_group])
            out[bh] = (rows,) + oracle.attn_rows_window(q, rows, k, v, scale, *band)
    return out


def lse_error(lse_gpu, lse_ref):
    """|LSE difference|; a row with no visible key must be -inf on both sides
    (error 0), -inf on one side only is an infinite error."""
    a = np.asarray(lse_gpu, dtype=np.float64).ravel()
    b = np.asarray(lse_ref, dtype=np.float64).ravel()
    both = np.isneginf(a) & np.isneginf(b)
    e = np.abs(np.where(both, 0.0, a) - np.where(both, 0.0, b))
    return np.where(np.isnan(e), np.inf, e)


def compare(o_gpu, lse_gpu, ref, check_lse=True):
    """Errors of the CUDA output against oracle rows; returns a dict of metrics."""
    B, H = o_gpu.shape[:2]
    errs_o, errs_l = [], []
    for bh, (rows, o_ref, l_ref) in ref.items():
        b, h = divmod(bh, H)
        errs_o.append(np.abs(o_gpu[b, h, rows].astype(np.float64) - o_ref).ravel())
        if check_lse:
            errs_l.append(lse_error(lse_gpu[b, h, rows], l_ref))
    eo = np.concatenate(errs_o)
    m = {"max_abs_o": float(eo.max()) if eo.size else 0.0, "mean_abs_o": float(eo.mean()) if eo.size else 0.0}
    if check_lse:
        el = np.concatenate(errs_l)
        m["max_abs_lse"] = float(el.max()) if el.size else 0.0
    return m


def assert_within(m, check_lse=True):
    assert np.isfinite(m["max_abs_o"]), m
    assert m["max_abs_o"] <= MAX_ABS_O, m
    assert m["mean_abs_o"] <= MEAN_ABS_O, m
    if check_lse:
        assert m["max_abs_lse"] <= MAX_ABS_LSE, m


def random_bits(seed, shape, dist="normal", mult=1.0, tensor="q"):
    return inputs.gen_bf16(seed, tensor, shape, dist, mult)


def compare_varlen(o_gpu, lse_gpu, ref, cu_q):
    """Errors of a packed result (o [total_q, H, d], lse [H, total_q]) against
    oracle.attn_varlen output {(s, h): (rows, o, lse)}."""
    errs_o, errs_l = [], []
    for (s, h), (rows, o_ref, l_ref) in ref.items():
        g = int(cu_q[s]) + rows
        errs_o.append(np.abs(o_gpu[g, h].astype(np.float64) - o_ref).ravel())
        errs_l.append(lse_error(lse_gpu[h, g], l_ref))
    eo = np.concatenate(errs_o) if errs_o else np.zeros(0)
    el = np.concatenate(errs_l) if errs_l else np.zeros(0)
    return {"max_abs_o": float(eo.max()) if eo.size else 0.0,
            "mean_abs_o": float(eo.mean()) if eo.size else 0.0,
            "max_abs_lse": float(el.max()) if el.size else 0.0}
