"""fp64 CPU oracle for exact attention: forward and backward, dense, key
bands, packed variable-length batches and column-interval masks.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (``exact_attention_152_b200``) never touches it, and
this package never imports the product.

The arithmetic lives in ``attn_oracle.c`` (plain C, fp64, one query row at a
time, written straight from the definition -- see that file's header for the
citations and the readings of the pages).  This module only compiles it with
gcc, marshals numpy arrays and loops over (batch, head) or (sequence, head).

Pins (checks against facts that do not come from this code) live in
``tests/oracle_pins.py``: brute force on tiny shapes, closed forms, invariants
and finite differences for every function here; none is left unpinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``attn_oracle.c`` into ``liboracle.so`` (gcc, -O2, fp-contract off)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    # -ffp-contract=off: no fused multiply-add, so every product and sum rounds
    # exactly as written in fp64.
    cmd = ["gcc", "-O2", "-ffp-contract=off", "-fPIC", "-shared", "-pthread",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            f = lib.oracle_attn_rows_f64
            f.restype = ctypes.c_int
            f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                          ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                          ctypes.c_double, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                          ctypes.c_int]
            w = lib.oracle_attn_rows_window_f64
            w.restype = ctypes.c_int
            w.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                          ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                          ctypes.c_double, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                          ctypes.c_void_p, ctypes.c_int]
            c = lib.oracle_attn_rows_colmask_f64
            c.restype = ctypes.c_int
            c.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                          ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                          ctypes.c_double, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                          ctypes.c_void_p, ctypes.c_int]
            bc = lib.oracle_attn_bwd_colmask_f64
            bc.restype = ctypes.c_int
            bc.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int64] * 3 + [ctypes.c_double, ctypes.c_int] + \
                [ctypes.c_void_p] * 4
            b = lib.oracle_attn_bwd_f64
            b.restype = ctypes.c_int
            b.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int64] * 3 + [ctypes.c_double] + \
                [ctypes.c_int64] * 2 + [ctypes.c_void_p] * 3
            _lib = lib
    return _lib


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def attn_rows(q_rows, rows, k, v, scale, causal, nthreads=None):
    """Attention of selected query rows of ONE (batch, head).

    q_rows: [n, d] fp64 -- the query vectors of rows ``rows`` (int64 [n]).
    k, v:   [Nk, d] fp64.
    Returns (o [n, d] fp64, lse [n] fp64, natural log).
    """
    lib = _load()
    q_rows = np.ascontiguousarray(q_rows, dtype=np.float64)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    n, d = q_rows.shape
    nk = k.shape[0]
    assert rows.shape == (n,) and k.shape == (nk, d) and v.shape == (nk, d)
    if causal:
        assert np.all(rows >= 0)
    o = np.empty((n, d), dtype=np.float64)
    lse = np.empty((n,), dtype=np.float64)
    nt = default_threads() if nthreads is None else int(nthreads)
    rc = lib.oracle_attn_rows_f64(q_rows.ctypes.data, rows.ctypes.data, n,
                                  k.ctypes.data if nk else None,
                                  v.ctypes.data if nk else None, nk, d,
                                  float(scale), 1 if causal else 0,
                                  o.ctypes.data, lse.ctypes.data, nt)
    if rc != 0:
        raise RuntimeError("oracle_attn_rows_f64 failed")
    return o, lse


def attn_rows_window(q_rows, rows, k, v, scale, window_left, window_right, nthreads=None):
    """Like ``attn_rows`` with the keys of row i limited to the band
    [i - window_left, i + window_right] (a negative bound is unbounded; causal
    is (-1, 0)).  Rows whose band holds no key get O = 0, LSE = -inf."""
    lib = _load()
    q_rows = np.ascontiguousarray(q_rows, dtype=np.float64)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    n, d = q_rows.shape
    nk = k.shape[0]
    assert rows.shape == (n,) and k.shape == (nk, d) and v.shape == (nk, d)
    o = np.empty((n, d), dtype=np.float64)
    lse = np.empty((n,), dtype=np.float64)
    nt = default_threads() if nthreads is None else int(nthreads)
    rc = lib.oracle_attn_rows_window_f64(q_rows.ctypes.data, rows.ctypes.data, n,
                                         k.ctypes.data if nk else None,
                                         v.ctypes.data if nk else None, nk, d, float(scale),
                                         int(window_left), int(window_right),
                                         o.ctypes.data, lse.ctypes.data, nt)
    if rc != 0:
        raise RuntimeError("oracle_attn_rows_window_f64 failed")
    return o, lse


def attn_rows_colmask(q_rows, rows, k, v, scale, causal, cols, nthreads=None):
    """Like ``attn_rows`` under column intervals: ``cols`` is [Nk, 4] integers,
    key j's (lo1, hi1, lo2, hi2); row i does not see key j when
    lo1 <= i < hi1 or lo2 <= i < hi2 (or j > i when causal).  Rows that see no
    key get O = 0, LSE = -inf."""
    lib = _load()
    q_rows = np.ascontiguousarray(q_rows, dtype=np.float64)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    cols = np.ascontiguousarray(cols, dtype=np.int64)
    n, d = q_rows.shape
    nk = k.shape[0]
    assert rows.shape == (n,) and k.shape == (nk, d) and v.shape == (nk, d)
    assert cols.shape == (nk, 4)
    o = np.empty((n, d), dtype=np.float64)
    lse = np.empty((n,), dtype=np.float64)
    nt = default_threads() if nthreads is None else int(nthreads)
    rc = lib.oracle_attn_rows_colmask_f64(q_rows.ctypes.data, rows.ctypes.data, n,
                                          k.ctypes.data if nk else None,
                                          v.ctypes.data if nk else None, nk, d, float(scale),
                                          1 if causal else 0, cols.ctypes.data if nk else None,
                                          o.ctypes.data, lse.ctypes.data, nt)
    if rc != 0:
        raise RuntimeError("oracle_attn_rows_colmask_f64 failed")
    return o, lse


def attn_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, scale, window_left=-1, window_right=-1,
                rows_per_seq=None, nthreads=None):
    """Variable-length batch: sequences packed back to back without padding
    (FlashAttention 4 page, ja.linux-konsole.com, section "互換性と現状": batching
    sequences of different lengths efficiently, with no padding).

    q: [total_q, H, d], k/v: [total_k, Hkv, d] fp64 (H % Hkv == 0; query head h
    reads key/value head h // (H // Hkv)); sequence s owns query rows
    cu_seqlens_q[s] .. cu_seqlens_q[s+1]-1 and keys cu_seqlens_k[s] ..
    cu_seqlens_k[s+1]-1, positions counted from 0 within the sequence; the band
    applies to those positions.  rows_per_seq: optional dict s -> local rows to
    evaluate (default all).  Returns {(s, h): (local rows, o [n, d], lse [n])}.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    H, Hkv = q.shape[1], k.shape[1]
    assert H % Hkv == 0
    out = {}
    for s in range(len(cu_seqlens_q) - 1):
        q0, q1 = int(cu_seqlens_q[s]), int(cu_seqlens_q[s + 1])
        k0, k1 = int(cu_seqlens_k[s]), int(cu_seqlens_k[s + 1])
        rows = np.arange(q1 - q0, dtype=np.int64) if rows_per_seq is None else \
            np.asarray(rows_per_seq[s], dtype=np.int64)
        for h in range(H):
            hk = h // (H // Hkv)
            out[(s, h)] = (rows,) + attn_rows_window(q[q0 + rows, h], rows, k[k0:k1, hk],
                                                     v[k0:k1, hk], scale, window_left,
                                                     window_right, nthreads)
    return out


def attn_fwd(q, k, v, scale, causal=False, nthreads=None):
    """Full attention over [B, H, N, d] fp64 arrays -> (o [B,H,Nq,d], lse [B,H,Nq])."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, H, nq, d = q.shape
    o = np.empty((B, H, nq, d), dtype=np.float64)
    lse = np.empty((B, H, nq), dtype=np.float64)
    rows = np.arange(nq, dtype=np.int64)
    for b in range(B):
        for h in range(H):
            o[b, h], lse[b, h] = attn_rows(q[b, h], rows, k[b, h], v[b, h],
                                           scale, causal, nthreads)
    return o, lse


def attn_bwd_head(q, k, v, dout, scale, window_left=-1, window_right=-1):
    """Gradients of one (batch, head): returns (dq [nq, d], dk [nk, d], dv [nk, d])
    fp64 for the cotangent dout [nq, d] (see oracle_attn_bwd_f64)."""
    lib = _load()
    q, k, v, dout = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v, dout))
    nq, d = q.shape
    nk = k.shape[0]
    assert k.shape == (nk, d) and v.shape == (nk, d) and dout.shape == (nq, d)
    dq = np.empty((nq, d))
    dk = np.empty((nk, d))
    dv = np.empty((nk, d))
    ptr = lambda a: a.ctypes.data if a.size else None  # noqa: E731
    rc = lib.oracle_attn_bwd_f64(ptr(q), ptr(k), ptr(v), ptr(dout), nq, nk, d, float(scale),
                                 int(window_left), int(window_right), ptr(dq), ptr(dk), ptr(dv))
    if rc != 0:
        raise RuntimeError("oracle_attn_bwd_f64 failed")
    return dq, dk, dv


def attn_bwd(q, k, v, dout, scale, window_left=-1, window_right=-1, nthreads=None):
    """Gradients over [B, H, Nq, d] q/dout and [B, Hkv, Nk, d] k/v (fp64).
    Query head h reads key/value head h // (H // Hkv); the key/value gradients
    of a shared head are the sum over its query heads.  Heads run on a thread
    pool (the C routine releases the GIL); the group sums are added in head
    order, so the result does not depend on the thread count."""
    import concurrent.futures
    q, k, v, dout = (np.asarray(x, dtype=np.float64) for x in (q, k, v, dout))
    B, H = q.shape[:2]
    Hkv = k.shape[1]
    g = H // Hkv
    jobs = [(b, h) for b in range(B) for h in range(H)]
    nt = default_threads() if nthreads is None else int(nthreads)
    with concurrent.futures.ThreadPoolExecutor(max_workers=max(1, nt)) as ex:
        res = list(ex.map(lambda bh: attn_bwd_head(q[bh[0], bh[1]], k[bh[0], bh[1] // g],
                                                   v[bh[0], bh[1] // g], dout[bh[0], bh[1]],
                                                   scale, window_left, window_right), jobs))
    dq = np.empty(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    for (b, h), (a, bk, bv) in zip(jobs, res):
        dq[b, h] = a
        dk[b, h // g] += bk
        dv[b, h // g] += bv
    return dq, dk, dv


def attn_bwd_varlen(q, k, v, dout, cu_seqlens_q, cu_seqlens_k, scale, window_left=-1,
                    window_right=-1, nthreads=None):
    """Gradients of ``attn_varlen``: q/dout [total_q, H, d], k/v [total_k, Hkv, d]
    fp64, each sequence taken alone (positions from 0 within it) and its heads
    through ``attn_bwd``.  Returns (dq, dk, dv) in the packed layouts; rows that
    belong to no sequence are 0 in dq and NaN in dk, dv (not defined)."""
    q, k, v, dout = (np.asarray(x, dtype=np.float64) for x in (q, k, v, dout))
    dq = np.zeros(q.shape)
    dk = np.full(k.shape, np.nan)
    dv = np.full(v.shape, np.nan)
    for s in range(len(cu_seqlens_q) - 1):
        q0, q1 = int(cu_seqlens_q[s]), int(cu_seqlens_q[s + 1])
        k0, k1 = int(cu_seqlens_k[s]), int(cu_seqlens_k[s + 1])
        per_head = lambda x, a, b: x[a:b].transpose(1, 0, 2)[None]  # noqa: E731  [1, heads, n, d]
        g = attn_bwd(per_head(q, q0, q1), per_head(k, k0, k1), per_head(v, k0, k1),
                     per_head(dout, q0, q1), scale, window_left, window_right, nthreads)
        dq[q0:q1] = g[0][0].transpose(1, 0, 2)
        dk[k0:k1] = g[1][0].transpose(1, 0, 2)
        dv[k0:k1] = g[2][0].transpose(1, 0, 2)
    return dq, dk, dv


def attn_bwd_colmask_head(q, k, v, dout, scale, causal, cols):
    """Gradients of one (batch, head) under column intervals (cols [Nk, 4]:
    key j hidden from rows [lo1, hi1) and [lo2, hi2), and from rows i < j when
    causal); see oracle_attn_bwd_colmask_f64."""
    lib = _load()
    q, k, v, dout = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v, dout))
    cols = np.ascontiguousarray(cols, dtype=np.int64)
    nq, d = q.shape
    nk = k.shape[0]
    assert cols.shape == (nk, 4)
    dq, dk, dv = np.empty((nq, d)), np.empty((nk, d)), np.empty((nk, d))
    ptr = lambda a: a.ctypes.data if a.size else None  # noqa: E731
    rc = lib.oracle_attn_bwd_colmask_f64(ptr(q), ptr(k), ptr(v), ptr(dout), nq, nk, d, float(scale),
                                         1 if causal else 0, ptr(cols), ptr(dq), ptr(dk), ptr(dv))
    if rc != 0:
        raise RuntimeError("oracle_attn_bwd_colmask_f64 failed")
    return dq, dk, dv


def attn_bwd_colmask(q, k, v, dout, scale, causal, mask, nthreads=None):
    """Gradients over [B, H, Nq, d] q/dout and [B, Hkv, Nk, d] k/v under the
    column intervals mask [B, Hm, Nk, 4] (Hm = 1: shared by the heads of a
    batch entry); key/value gradients of a shared head summed in head order."""
    import concurrent.futures
    q, k, v, dout = (np.asarray(x, dtype=np.float64) for x in (q, k, v, dout))
    B, H = q.shape[:2]
    g = H // k.shape[1]
    hm = mask.shape[1]
    jobs = [(b, h) for b in range(B) for h in range(H)]
    nt = default_threads() if nthreads is None else int(nthreads)
    with concurrent.futures.ThreadPoolExecutor(max_workers=max(1, nt)) as ex:
        res = list(ex.map(lambda bh: attn_bwd_colmask_head(
            q[bh[0], bh[1]], k[bh[0], bh[1] // g], v[bh[0], bh[1] // g], dout[bh[0], bh[1]], scale,
            causal, mask[bh[0], bh[1] if hm > 1 else 0]), jobs))
    dq = np.empty(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    for (b, h), (a, bk, bv) in zip(jobs, res):
        dq[b, h] = a
        dk[b, h // g] += bk
        dv[b, h // g] += bv
    return dq, dk, dv
