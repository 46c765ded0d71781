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


# ---------------------------------------------------------------------------
# Element-wise error bound of the BF16 backward
# ---------------------------------------------------------------------------
# Each gradient element is a sum of products in which at most one BF16-rounded
# factor per product carries error, accumulated in fp32 (error ~2^-24 per add,
# negligible), and is itself rounded to BF16 once:
#   dV_j = sum_i P_ij dO_i          P rounded to BF16 before its GEMM:
#        |err| <= u (sum_i P_ij |dO_i|) + u |dV_j|
#   dS_ij = P_ij (dP_ij - D_i)       dS rounded to BF16 before its GEMMs, and
#                                    D_i = <dO_i, O_i> formed from the forward's
#                                    BF16 O, itself within u (|O| + P|V|) of O:
#        |err dS_ij| <= u |dS_ij| + u P_ij sum_c |dO_ic| (|O_ic| + (P|V|)_ic)
#   dK_j = scale sum_i dS_ij Q_i,  dQ_i = scale sum_j dS_ij K_j
#        |err| <= scale sum |err dS| |Q or K| + u |dK_j or dQ_i|
# with u = 2^-8 the unit roundoff of BF16 (8 significant bits, round to
# nearest even).  The exponentials (MUFU, or the polynomial at 1.01e-4
# relative) and the forward's LSE (within ~1e-5) move P by far less than u.
# The GPU tests allow twice the sum (BWD_C = 2); tests/test_bwd_bound.py checks
# that a CPU model of exactly these roundings stays within the sum itself.
BWD_U = 2.0 ** -8
BWD_C = 2.0


def bwd_bound_head(q, k, v, do, scale, visible, chunk=512):
    """Magnitude sums of the bound above for one head, fp64.

    q, do [Nq, d]; k, v [Nk, d]; visible(r0, r1) -> bool [r1 - r0, Nk], the
    keys each of rows r0..r1-1 sees.  Returns (mq [Nq, d], mk [Nk, d],
    mv [Nk, d]) such that |err| <= u * (m + |grad|) element by element."""
    Nq, d = q.shape
    Nk = k.shape[0]
    mq = np.zeros((Nq, d))
    mk = np.zeros((Nk, d))
    mv = np.zeros((Nk, d))
    if Nq == 0 or Nk == 0:
        return mq, mk, mv
    ak, av = np.abs(k), np.abs(v)
    for r0 in range(0, Nq, chunk):
        r1 = min(Nq, r0 + chunk)
        vis = visible(r0, r1)
        s = scale * (q[r0:r1] @ k.T)
        s = np.where(vis, s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        m = np.where(np.isfinite(m), m, 0.0)
        e = np.where(vis, np.exp(s - m), 0.0)
        l = e.sum(axis=1, keepdims=True)
        p = e / np.where(l > 0, l, 1.0)
        o = p @ v
        pv_abs = p @ av
        g = do[r0:r1]
        dp = g @ v.T
        dd = (g * o).sum(axis=1, keepdims=True)
        ds = p * (dp - dd)
        dabs = (np.abs(g) * (np.abs(o) + pv_abs)).sum(axis=1, keepdims=True)
        w = np.abs(ds) + p * dabs
        mq[r0:r1] = scale * (w @ ak)
        mk += scale * (w.T @ np.abs(q[r0:r1]))
        mv += p.T @ np.abs(g)
    return mq, mk, mv


def band_visible(wl, wr, Nk):
    """visible(r0, r1) for the key band i - wl <= j <= i + wr (-1: no bound)."""
    j = np.arange(Nk)[None, :]

    def vis(r0, r1):
        i = np.arange(r0, r1)[:, None]
        ok = np.ones((r1 - r0, Nk), dtype=bool)
        if wl >= 0:
            ok &= j >= i - wl
        if wr >= 0:
            ok &= j <= i + wr
        return ok
    return vis


def colmask_visible(cols, causal):
    """visible(r0, r1) for column intervals cols [Nk, 4] (lo1, hi1, lo2, hi2:
    rows in [lo, hi) do not see the key) plus the causal rule j <= i."""
    lo1, hi1, lo2, hi2 = (cols[:, c][None, :].astype(np.int64) for c in range(4))
    Nk = cols.shape[0]
    j = np.arange(Nk)[None, :]

    def vis(r0, r1):
        i = np.arange(r0, r1)[:, None]
        hidden = ((i >= lo1) & (i < hi1)) | ((i >= lo2) & (i < hi2))
        ok = ~hidden
        if causal:
            ok &= j <= i
        return ok
    return vis


def bwd_bound_dense(q, k, v, do, scale, visible_of):
    """Magnitude sums for [B, H, Nq, d] problems with [B, Hkv, Nk, d] keys and
    values (grouped heads sum into their key/value head).  visible_of(b, h)
    returns the visibility function of that query head."""
    B, H, Nq, d = q.shape
    Hkv = k.shape[1]
    grp = H // Hkv
    mq = np.zeros(q.shape)
    mk = np.zeros(k.shape)
    mv = np.zeros(v.shape)
    for b in range(B):
        for h in range(H):
            a, bk, bv = bwd_bound_head(q[b, h], k[b, h // grp], v[b, h // grp], do[b, h], scale,
                                       visible_of(b, h))
            mq[b, h] = a
            mk[b, h // grp] += bk
            mv[b, h // grp] += bv
    return mq, mk, mv


def bwd_bound_varlen(q, k, v, do, cu_q, cu_k, scale, wl, wr):
    """Magnitude sums for packed batches (q, do [total_q, H, d]; k, v
    [total_k, Hkv, d]); positions count from 0 within each sequence."""
    H, Hkv = q.shape[1], k.shape[1]
    grp = H // Hkv
    mq = np.zeros(q.shape)
    mk = np.zeros(k.shape)
    mv = np.zeros(v.shape)
    for s in range(len(cu_q) - 1):
        a0, a1, c0, c1 = int(cu_q[s]), int(cu_q[s + 1]), int(cu_k[s]), int(cu_k[s + 1])
        for h in range(H):
            a, bk, bv = bwd_bound_head(q[a0:a1, h], k[c0:c1, h // grp], v[c0:c1, h // grp],
                                       do[a0:a1, h], scale, band_visible(wl, wr, c1 - c0))
            mq[a0:a1, h] = a
            mk[c0:c1, h // grp] += bk
            mv[c0:c1, h // grp] += bv
    return mq, mk, mv


def check_grads_elementwise(got, ref, mags, label=""):
    """|got - ref| <= BWD_C * u * (magnitude sums + |ref|) element by element,
    plus a floor of 1e-6 of the problem's largest gradient for fp32 noise."""
    top = max((np.abs(r).max() if r.size else 0.0) for r in ref)
    for name, g, r, m in zip(("dq", "dk", "dv"), got, ref, mags):
        g = np.asarray(g, dtype=np.float64)
        assert np.all(np.isfinite(g)), (label, name)
        err = np.abs(g - r)
        lim = BWD_C * BWD_U * (m + np.abs(r)) + 1e-6 * top + 1e-12
        worst = np.unravel_index(np.argmax(err / lim), err.shape) if err.size else None
        if err.size:
            print(label, name, "max err/bound", float((err / lim).max()), "at", worst)
        assert np.all(err <= lim), (label, name, worst, float(err[worst]), float(lim[worst]))
