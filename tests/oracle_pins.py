"""Pins for the fp64 oracle: checks against facts that do not come from the oracle.

Each ``pin_*`` takes an ``attn_rows(q_rows, rows, k, v, scale, causal)`` callable
(the oracle's per-head entry) and raises AssertionError when it disagrees with
what the mathematics fixes.  ``test_oracle_pins.py`` runs them on the real
oracle and on deliberately broken copies of it (to show each plausible mistake
is caught by at least one pin).
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "closed_forms.json")


def _rng(seed):
    return np.random.default_rng(seed)


def _full(attn_rows, q, k, v, scale, causal):
    rows = np.arange(q.shape[0], dtype=np.int64)
    return attn_rows(q, rows, k, v, scale, causal)


def brute_force_python(q, k, v, scale, causal):
    """Textbook attention in pure Python floats: S, then softmax without any max
    subtraction, then P.V.  Only for tiny shapes and small logits."""
    nq, d = len(q), len(q[0])
    nk = len(k)
    o, lse = [], []
    for i in range(nq):
        keys = range(min(i + 1, nk)) if causal else range(nk)
        w = {}
        for j in keys:
            w[j] = math.exp(scale * sum(q[i][c] * k[j][c] for c in range(d)))
        z = sum(w.values())
        o.append([sum(w[j] * v[j][c] for j in keys) / z for c in range(d)])
        lse.append(math.log(z))
    return np.array(o), np.array(lse)


def pin_brute_force(attn_rows):
    """Match a brute-force materialised softmax on tiny shapes (both maskings)."""
    for seed, (nq, nk, d) in enumerate([(1, 1, 1), (3, 5, 2), (7, 7, 4), (9, 9, 3), (4, 13, 8)]):
        r = _rng(seed)
        q, k, v = (r.standard_normal((n, d)) for n in (nq, nk, nk))
        for causal in (False, True):
            if causal and nq != nk:
                continue
            scale = 0.7
            o, lse = _full(attn_rows, q, k, v, scale, causal)
            ob, lb = brute_force_python(q.tolist(), k.tolist(), v.tolist(), scale, causal)
            np.testing.assert_allclose(o, ob, rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(lse, lb, rtol=1e-12, atol=1e-12)


def pin_golden(attn_rows):
    """Hand-derived closed forms stored under tests/golden/."""
    with open(GOLDEN) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        q, k, v = (np.array(c[x], dtype=np.float64) for x in ("q", "k", "v"))
        o, lse = _full(attn_rows, q, k, v, c["scale"], c["causal"])
        np.testing.assert_allclose(o, np.array(c["o"]), rtol=1e-13, atol=1e-13, err_msg=c["name"])
        np.testing.assert_allclose(lse, np.array(c["lse"]), rtol=1e-13, atol=1e-13, err_msg=c["name"])


def pin_single_key(attn_rows):
    """One key: softmax weight is exactly 1, so O = V0 bit-exactly and LSE = s0."""
    r = _rng(11)
    q, k, v = r.standard_normal((5, 16)), r.standard_normal((1, 16)), r.standard_normal((1, 16))
    o, lse = _full(attn_rows, q, k, v, 0.3, False)
    assert np.array_equal(o, np.repeat(v, 5, axis=0))
    np.testing.assert_allclose(lse, 0.3 * (q @ k[0]), rtol=1e-14, atol=1e-14)


def pin_identical_keys(attn_rows):
    """All keys equal: uniform weights, O = mean(V), LSE = s + log(Nk)."""
    r = _rng(12)
    nk, d = 37, 8
    q = r.standard_normal((4, d))
    k = np.repeat(r.standard_normal((1, d)), nk, axis=0)
    v = r.standard_normal((nk, d))
    o, lse = _full(attn_rows, q, k, v, 0.9, False)
    np.testing.assert_allclose(o, np.repeat(v.mean(0, keepdims=True), 4, 0), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, 0.9 * (q @ k[0]) + math.log(nk), rtol=1e-13, atol=1e-13)


def pin_zero_scale(attn_rows):
    """scale = 0: every logit is 0, O = mean(V), LSE = log(Nk)."""
    r = _rng(13)
    q, k, v = r.standard_normal((3, 8)), r.standard_normal((10, 8)), r.standard_normal((10, 8))
    o, lse = _full(attn_rows, q, k, v, 0.0, False)
    np.testing.assert_allclose(o, np.repeat(v.mean(0, keepdims=True), 3, 0), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, np.full(3, math.log(10)), rtol=1e-14)


def pin_causal_prefix(attn_rows):
    """Causal row 0 is V0 exactly; causal row i equals unmasked attention over keys 0..i."""
    r = _rng(14)
    n, d = 12, 8
    q, k, v = (r.standard_normal((n, d)) for _ in range(3))
    o, lse = _full(attn_rows, q, k, v, 0.5, True)
    assert np.array_equal(o[0], v[0])
    for i in range(n):
        oi, li = attn_rows(q[i:i + 1], np.array([0], dtype=np.int64), k[:i + 1], v[:i + 1], 0.5, False)
        np.testing.assert_allclose(o[i], oi[0], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse[i], li[0], rtol=1e-13, atol=1e-13)


def pin_rows_sum_to_one(attn_rows):
    """With independently computed logits s, sum_j exp(s_j - LSE) = 1 and
    O = sum_j exp(s_j - LSE) v_j  (normalisation and the LSE together)."""
    r = _rng(15)
    q, k, v = r.standard_normal((6, 8)), r.standard_normal((21, 8)), r.standard_normal((21, 8))
    scale = 0.8
    o, lse = _full(attn_rows, q, k, v, scale, False)
    s = scale * np.einsum("id,jd->ij", q, k)
    p = np.exp(s - lse[:, None])
    np.testing.assert_allclose(p.sum(1), np.ones(6), rtol=1e-13)
    np.testing.assert_allclose(o, p @ v, rtol=1e-12, atol=1e-13)


def pin_shift_invariance(attn_rows):
    """Adding one vector c to every key leaves O unchanged and shifts LSE_i by
    scale * q_i . c (softmax is invariant to a per-row constant)."""
    r = _rng(16)
    q, k, v = r.standard_normal((5, 8)), r.standard_normal((9, 8)), r.standard_normal((9, 8))
    c = r.standard_normal(8)
    o1, l1 = _full(attn_rows, q, k, v, 0.6, False)
    o2, l2 = _full(attn_rows, q, k + c, v, 0.6, False)
    np.testing.assert_allclose(o2, o1, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(l2, l1 + 0.6 * (q @ c), rtol=1e-12, atol=1e-12)


def pin_value_linearity(attn_rows):
    """O is linear in V: O(V A) = O(V) A."""
    r = _rng(17)
    q, k, v = r.standard_normal((4, 6)), r.standard_normal((11, 6)), r.standard_normal((11, 6))
    a = r.standard_normal((6, 6))
    o1, _ = _full(attn_rows, q, k, v, 0.4, False)
    o2, _ = _full(attn_rows, q, k, v @ a, 0.4, False)
    np.testing.assert_allclose(o2, o1 @ a, rtol=1e-11, atol=1e-12)


def pin_key_permutation(attn_rows):
    """Unmasked attention does not depend on the order of the (key, value) pairs."""
    r = _rng(18)
    q, k, v = r.standard_normal((4, 8)), r.standard_normal((15, 8)), r.standard_normal((15, 8))
    perm = r.permutation(15)
    o1, l1 = _full(attn_rows, q, k, v, 0.5, False)
    o2, l2 = _full(attn_rows, q, k[perm], v[perm], 0.5, False)
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l2, l1, rtol=1e-13, atol=1e-13)


def pin_split_merge(attn_rows):
    """Attention over [K1;K2] equals the LSE-weighted merge of the two halves --
    the algebra that lets a tiled method visit the keys block by block."""
    r = _rng(19)
    q, k, v = r.standard_normal((5, 8)), r.standard_normal((20, 8)), r.standard_normal((20, 8))
    o, l = _full(attn_rows, q, k, v, 0.7, False)
    o1, l1 = _full(attn_rows, q, k[:7], v[:7], 0.7, False)
    o2, l2 = _full(attn_rows, q, k[7:], v[7:], 0.7, False)
    lm = np.logaddexp(l1, l2)
    om = np.exp(l1 - lm)[:, None] * o1 + np.exp(l2 - lm)[:, None] * o2
    np.testing.assert_allclose(o, om, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l, lm, rtol=1e-13, atol=1e-13)


def pin_hard_max(attn_rows):
    """As the scale grows the softmax becomes an argmax: O -> V at the largest logit.
    Also exercises logits far beyond exp's range (the max must be subtracted)."""
    r = _rng(20)
    q, k, v = r.standard_normal((6, 8)), r.standard_normal((13, 8)), r.standard_normal((13, 8))
    o, lse = _full(attn_rows, q, k, v, 1e6, False)
    s = q @ k.T
    best = s.argmax(1)
    np.testing.assert_allclose(o, v[best], rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(lse, 1e6 * s.max(1), rtol=1e-12)


def pin_two_keys_sigmoid(attn_rows):
    """Two keys: the weights are the logistic function of the logit difference."""
    r = _rng(21)
    q, k, v = r.standard_normal((8, 4)), r.standard_normal((2, 4)), r.standard_normal((2, 4))
    o, lse = _full(attn_rows, q, k, v, 1.3, False)
    s = 1.3 * (q @ k.T)
    w0 = 1.0 / (1.0 + np.exp(s[:, 1] - s[:, 0]))
    np.testing.assert_allclose(o, w0[:, None] * v[0] + (1 - w0)[:, None] * v[1], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, np.logaddexp(s[:, 0], s[:, 1]), rtol=1e-13, atol=1e-13)


def pin_empty_keys(attn_rows):
    """No visible key: O = 0 and LSE = -inf (this library's definition)."""
    q = np.ones((2, 4))
    k = np.zeros((0, 4))
    o, lse = attn_rows(q, np.arange(2, dtype=np.int64), k, k, 1.0, False)
    assert np.array_equal(o, np.zeros((2, 4)))
    assert np.all(np.isneginf(lse))


def pin_sampled_rows(attn_rows):
    """Evaluating a subset of rows gives the same values as evaluating all rows
    (row sampling is how the oracle checks large problems)."""
    r = _rng(22)
    n, d = 30, 8
    q, k, v = (r.standard_normal((n, d)) for _ in range(3))
    for causal in (False, True):
        o, lse = _full(attn_rows, q, k, v, 0.5, causal)
        rows = np.array([0, 3, 17, 29], dtype=np.int64)
        os_, ls_ = attn_rows(q[rows], rows, k, v, 0.5, causal)
        assert np.array_equal(os_, o[rows]) and np.array_equal(ls_, lse[rows])


# ---------------------------------------------------------------------------
# Sliding-window band.  These take ``attn_rows_window(q_rows, rows, k, v, scale,
# window_left, window_right)``.
# ---------------------------------------------------------------------------
def band_mask_numpy(nq, nk, wl, wr):
    """Visible (i, j) pairs built from numpy's triangle helpers: np.triu(., -wl)
    keeps j - i >= -wl, np.tril(., wr) keeps j - i <= wr."""
    m = np.ones((nq, nk), dtype=bool)
    if wl >= 0:
        m = np.triu(m, -wl)
    if wr >= 0:
        m = np.tril(m, wr)
    return m


def masked_softmax_numpy(q, k, v, scale, mask):
    """Dense masked attention: materialised scores, -inf outside the mask."""
    s = np.where(mask, scale * (q @ k.T), -np.inf)
    o = np.zeros((q.shape[0], v.shape[1]))
    lse = np.full(q.shape[0], -np.inf)
    for i in range(q.shape[0]):
        if not mask[i].any():
            continue
        m = s[i].max()
        e = np.exp(s[i] - m)
        o[i] = (e / e.sum()) @ v
        lse[i] = m + np.log(e.sum())
    return o, lse


WINDOWS = [(0, 0), (2, 1), (-1, 0), (3, -1), (-1, -1), (1, 5), (20, 20), (0, 3), (4, 0)]


def pin_window_brute_force(attn_rows_window):
    """Match materialised masked attention for many bands, Nq != Nk, and rows
    whose band holds no key."""
    for seed, (nq, nk, d) in enumerate([(7, 7, 4), (9, 13, 3), (12, 5, 8), (1, 1, 2)]):
        r = _rng(100 + seed)
        q, k, v = (r.standard_normal((n, d)) for n in (nq, nk, nk))
        for wl, wr in WINDOWS:
            o, lse = attn_rows_window(q, np.arange(nq, dtype=np.int64), k, v, 0.6, wl, wr)
            ob, lb = masked_softmax_numpy(q, k, v, 0.6, band_mask_numpy(nq, nk, wl, wr))
            np.testing.assert_allclose(o, ob, rtol=1e-12, atol=1e-12, err_msg=str((nq, nk, wl, wr)))
            np.testing.assert_allclose(lse, lb, rtol=1e-12, atol=1e-12, err_msg=str((nq, nk, wl, wr)))


def pin_window_diagonal(attn_rows_window):
    """Band (0, 0): each row sees only its own key, so O_i = v_i exactly and
    LSE_i = scale * q_i . k_i."""
    r = _rng(110)
    n, d = 10, 8
    q, k, v = (r.standard_normal((n, d)) for _ in range(3))
    o, lse = attn_rows_window(q, np.arange(n, dtype=np.int64), k, v, 0.45, 0, 0)
    assert np.array_equal(o, v)
    np.testing.assert_allclose(lse, 0.45 * np.einsum("id,id->i", q, k), rtol=1e-14, atol=1e-14)


def pin_window_is_a_key_slice(attn_rows_window):
    """Row i under band (wl, wr) equals unmasked attention over the key slice
    [max(0, i-wl), min(Nk-1, i+wr)] given to the oracle as the whole key set."""
    r = _rng(111)
    n, d = 16, 4
    q, k, v = (r.standard_normal((n, d)) for _ in range(3))
    for wl, wr in [(3, 2), (0, 5), (6, 0)]:
        o, lse = attn_rows_window(q, np.arange(n, dtype=np.int64), k, v, 0.8, wl, wr)
        for i in range(n):
            lo, hi = max(0, i - wl), min(n - 1, i + wr)
            oi, li = attn_rows_window(q[i:i + 1], np.array([0], dtype=np.int64), k[lo:hi + 1],
                                      v[lo:hi + 1], 0.8, -1, -1)
            np.testing.assert_allclose(o[i], oi[0], rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(lse[i], li[0], rtol=1e-13, atol=1e-13)


WINDOW_PINS = [pin_window_brute_force, pin_window_diagonal, pin_window_is_a_key_slice]


# ---------------------------------------------------------------------------
# Column-interval masks.  These take ``attn_rows_colmask(q_rows, rows, k, v,
# scale, causal, cols)`` with cols [Nk, 4] = (lo1, hi1, lo2, hi2) per key.
# ---------------------------------------------------------------------------
BIG = 1 << 20  # beyond every row index used here


def band_as_columns(nk, wl, wr):
    """Column intervals of the band (wl, wr): key j is hidden from rows
    i > j + wl (first interval) and from rows i < j - wr (second)."""
    j = np.arange(nk, dtype=np.int64)
    cols = np.zeros((nk, 4), dtype=np.int64)  # (0, 0): empty
    if wl >= 0:
        cols[:, 0], cols[:, 1] = j + wl + 1, BIG
    if wr >= 0:
        cols[:, 2], cols[:, 3] = -BIG, j - wr
    return cols


def pin_colmask_band(attn_rows_colmask):
    """Column intervals that spell a band give the band's materialised masked
    attention (the mask built from numpy's triangle helpers)."""
    for seed, (nq, nk, d) in enumerate([(7, 7, 4), (9, 13, 3), (12, 5, 8)]):
        r = _rng(200 + seed)
        q, k, v = (r.standard_normal((n, d)) for n in (nq, nk, nk))
        for wl, wr in WINDOWS:
            o, lse = attn_rows_colmask(q, np.arange(nq, dtype=np.int64), k, v, 0.6, False,
                                       band_as_columns(nk, wl, wr))
            ob, lb = masked_softmax_numpy(q, k, v, 0.6, band_mask_numpy(nq, nk, wl, wr))
            np.testing.assert_allclose(o, ob, rtol=1e-12, atol=1e-12, err_msg=str((nq, nk, wl, wr)))
            np.testing.assert_allclose(lse, lb, rtol=1e-12, atol=1e-12, err_msg=str((nq, nk, wl, wr)))


def pin_colmask_documents(attn_rows_colmask):
    """Document mask: keys of a document are hidden from every later row; with
    causal on, each document's rows equal causal attention within that document
    alone (textbook brute force on the slice)."""
    r = _rng(210)
    lens = [3, 5, 1, 4, 2]
    n, d = sum(lens), 4
    q, k, v = (r.standard_normal((n, d)) for _ in range(3))
    cols = np.zeros((n, 4), dtype=np.int64)
    start = 0
    for ln in lens:
        cols[start:start + ln, 0] = start + ln
        cols[start:start + ln, 1] = n
        start += ln
    o, lse = attn_rows_colmask(q, np.arange(n, dtype=np.int64), k, v, 0.9, True, cols)
    start = 0
    for ln in lens:
        sl = slice(start, start + ln)
        ob, lb = brute_force_python(q[sl].tolist(), k[sl].tolist(), v[sl].tolist(), 0.9, True)
        np.testing.assert_allclose(o[sl], ob, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse[sl], lb, rtol=1e-12, atol=1e-12)
        start += ln


def pin_colmask_empty_intervals(attn_rows_colmask):
    """Empty intervals (lo >= hi, in several spellings) hide nothing: the result
    is textbook attention, causal or not."""
    r = _rng(220)
    n, d = 9, 3
    q, k, v = (r.standard_normal((n, d)) for _ in range(3))
    cols = np.array([[0, 0, 5, 5], [7, 2, 3, 3], [9, 9, 100, -100]] * 3, dtype=np.int64)
    for causal in (False, True):
        o, lse = attn_rows_colmask(q, np.arange(n, dtype=np.int64), k, v, 0.7, causal, cols)
        ob, lb = brute_force_python(q.tolist(), k.tolist(), v.tolist(), 0.7, causal)
        np.testing.assert_allclose(o, ob, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse, lb, rtol=1e-12, atol=1e-12)


def pin_colmask_two_intervals(attn_rows_colmask):
    """Row i sees exactly the keys outside both of their intervals: each row
    equals unmasked attention over that key subset, given as the whole key set
    (so the second interval, the half-open ends and non-contiguous key sets are
    all exercised), and rows that see nothing get O = 0, LSE = -inf."""
    r = _rng(230)
    n, nk, d = 11, 10, 3
    q, k, v = (r.standard_normal((n, d)) for n in (n, nk, nk))
    cols = np.array([[2, 5, 8, 11], [0, 3, 3, 3], [4, 4, 0, 6], [1, 9, 10, 11], [0, 11, 0, 0],
                     [6, 7, 2, 3], [0, 2, 9, 11], [3, 8, 8, 10], [5, 11, 0, 5], [7, 10, 1, 2]],
                    dtype=np.int64)
    rows = np.arange(n, dtype=np.int64)
    # second set: every key's second interval is [8, 11), so rows 8..10 see nothing
    cols_b = cols.copy()
    cols_b[:, 2], cols_b[:, 3] = 8, 11
    for c in (cols, cols_b):
        o, lse = attn_rows_colmask(q, rows, k, v, 0.5, False, c)
        for i in range(n):
            keep = [j for j in range(nk)
                    if not (c[j, 0] <= i < c[j, 1]) and not (c[j, 2] <= i < c[j, 3])]
            if not keep:
                assert np.all(o[i] == 0.0) and lse[i] == -np.inf, i
                continue
            ob, lb = brute_force_python(q[i:i + 1].tolist(), k[keep].tolist(), v[keep].tolist(),
                                        0.5, False)
            np.testing.assert_allclose(o[i], ob[0], rtol=1e-12, atol=1e-12, err_msg=str(i))
            np.testing.assert_allclose(lse[i], lb[0], rtol=1e-12, atol=1e-12, err_msg=str(i))
    assert np.all(o[8:] == 0.0) and np.all(lse[8:] == -np.inf)


def pin_colmask_golden(attn_rows_colmask):
    """Hand-derived closed forms under column intervals stored under tests/golden/."""
    with open(os.path.join(os.path.dirname(GOLDEN), "colmask_closed_forms.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        q, k, v = (np.array(c[x], dtype=np.float64) for x in ("q", "k", "v"))
        cols = np.array(c["cols"], dtype=np.int64)
        o, lse = attn_rows_colmask(q, np.arange(q.shape[0], dtype=np.int64), k, v, c["scale"], c["causal"],
                                   cols)
        want_lse = np.array([float(x) for x in c["lse"]])
        np.testing.assert_allclose(o, np.array(c["o"]), rtol=1e-13, atol=1e-13, err_msg=c["name"])
        np.testing.assert_allclose(lse, want_lse, rtol=1e-13, atol=1e-13, err_msg=c["name"])


COLMASK_PINS = [pin_colmask_band, pin_colmask_documents, pin_colmask_empty_intervals,
                pin_colmask_two_intervals, pin_colmask_golden]


def pin_bwd_colmask_finite_differences(attn_bwd_colmask_head, attn_rows_colmask):
    """Every gradient element under column intervals (two intervals per key,
    some rows seeing no key, causal or not) equals the central difference of
    L = sum(dO * O) through the column-interval forward definition."""
    h = 1e-5
    r = _rng(340)
    nq, nk, d = 6, 7, 2
    cols = np.array([[2, 4, 5, 6], [0, 1, 3, 3], [4, 4, 0, 2], [1, 6, 0, 0], [5, 9, 1, 2],
                     [0, 0, 0, 0], [3, 5, 0, 1]], dtype=np.int64)
    rows = np.arange(nq, dtype=np.int64)
    for causal in (False, True):
        q, k, v, dout = (r.standard_normal(s) for s in ((nq, d), (nk, d), (nk, d), (nq, d)))
        grads = attn_bwd_colmask_head(q, k, v, dout, 0.9, causal, cols)

        def loss(q_, k_, v_):
            o, _ = attn_rows_colmask(q_, rows, k_, v_, 0.9, causal, cols)
            return float((o * dout).sum())
        for which, x in enumerate((q, k, v)):
            num = np.zeros_like(x)
            for idx in np.ndindex(*x.shape):
                args = [q.copy(), k.copy(), v.copy()]
                args[which][idx] += h
                lp = loss(*args)
                args[which][idx] -= 2 * h
                lm = loss(*args)
                num[idx] = (lp - lm) / (2 * h)
            np.testing.assert_allclose(grads[which], num, rtol=1e-6, atol=1e-8,
                                       err_msg=f"grad {'qkv'[which]} causal {causal}")


def pin_bwd_colmask_band_is_the_band(attn_bwd_colmask_head, attn_rows_colmask):
    """Intervals that spell a band give the band's gradients (numpy softmax
    Jacobian on the triu/tril mask: dV = P^T dO, dS = P (dP - rowsum(P dP)))."""
    r = _rng(341)
    n, d = 8, 3
    q, k, v, dout = (r.standard_normal((n, d)) for _ in range(4))
    for wl, wr in [(2, 1), (-1, 0), (0, 3)]:
        dq, dk, dv = attn_bwd_colmask_head(q, k, v, dout, 0.6, False, band_as_columns(n, wl, wr))
        m = band_mask_numpy(n, n, wl, wr)
        s = np.where(m, 0.6 * q @ k.T, -np.inf)
        p = np.exp(s - s.max(1, keepdims=True))
        p /= p.sum(1, keepdims=True)
        dp = dout @ v.T
        ds = p * (dp - (p * dp).sum(1, keepdims=True))
        np.testing.assert_allclose(dv, p.T @ dout, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(dq, 0.6 * ds @ k, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(dk, 0.6 * ds.T @ q, rtol=1e-12, atol=1e-12)


BWD_COLMASK_PINS = [pin_bwd_colmask_finite_differences, pin_bwd_colmask_band_is_the_band]


ALL_PINS = [
    pin_brute_force, pin_golden, pin_single_key, pin_identical_keys, pin_zero_scale,
    pin_causal_prefix, pin_rows_sum_to_one, pin_shift_invariance, pin_value_linearity,
    pin_key_permutation, pin_split_merge, pin_hard_max, pin_two_keys_sigmoid,
    pin_empty_keys, pin_sampled_rows,
]


# ---------------------------------------------------------------------------
# Variable-length batches.  These take ``attn_varlen(q, k, v, cu_q, cu_k, scale,
# window_left, window_right)`` returning {(s, h): (rows, o, lse)}.
# ---------------------------------------------------------------------------
def pin_varlen_block_diagonal(attn_varlen):
    """Packed sequences equal one dense masked attention over the whole packed
    index space whose mask is block-diagonal (same sequence) and banded on the
    positions within the sequence; includes an empty sequence, Nq != Nk per
    sequence and grouped key/value heads."""
    r = _rng(120)
    lens_q = [5, 0, 9, 3]
    lens_k = [7, 2, 9, 1]
    H, Hkv, d = 4, 2, 4
    cu_q = np.concatenate([[0], np.cumsum(lens_q)])
    cu_k = np.concatenate([[0], np.cumsum(lens_k)])
    q = r.standard_normal((cu_q[-1], H, d))
    k = r.standard_normal((cu_k[-1], Hkv, d))
    v = r.standard_normal((cu_k[-1], Hkv, d))
    seq_q = np.repeat(np.arange(len(lens_q)), lens_q)
    seq_k = np.repeat(np.arange(len(lens_k)), lens_k)
    pos_q = np.arange(cu_q[-1]) - cu_q[seq_q]
    pos_k = np.arange(cu_k[-1]) - cu_k[seq_k]
    for wl, wr in [(-1, -1), (-1, 0), (1, 1)]:
        got = attn_varlen(q, k, v, cu_q, cu_k, 0.7, wl, wr)
        rel = pos_k[None, :] - pos_q[:, None]
        mask = seq_q[:, None] == seq_k[None, :]
        if wl >= 0:
            mask &= rel >= -wl
        if wr >= 0:
            mask &= rel <= wr
        for h in range(H):
            hk = h // (H // Hkv)
            ob, lb = masked_softmax_numpy(q[:, h], k[:, hk], v[:, hk], 0.7, mask)
            for s in range(len(lens_q)):
                rows, o, lse = got[(s, h)]
                np.testing.assert_allclose(o, ob[cu_q[s] + rows], rtol=1e-12, atol=1e-12)
                np.testing.assert_allclose(lse, lb[cu_q[s] + rows], rtol=1e-12, atol=1e-12)


def pin_varlen_neighbours_do_not_leak(attn_varlen):
    """A sequence's output does not change when the other sequences' data does."""
    r = _rng(121)
    cu = np.array([0, 6, 10, 19])
    q, k, v = (r.standard_normal((19, 2, 4)) for _ in range(3))
    a = attn_varlen(q, k, v, cu, cu, 0.5, -1, 0)
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    for x in (q2, k2, v2):
        x[:6] += 3.0
        x[10:] -= 2.0
    b = attn_varlen(q2, k2, v2, cu, cu, 0.5, -1, 0)
    for h in range(2):
        assert np.array_equal(a[(1, h)][1], b[(1, h)][1])
        assert np.array_equal(a[(1, h)][2], b[(1, h)][2])


VARLEN_PINS = [pin_varlen_block_diagonal, pin_varlen_neighbours_do_not_leak]



# ---------------------------------------------------------------------------
# Backward pass.  These take ``bwd(q, k, v, dout, scale, wl, wr) -> (dq, dk, dv)``
# for one head and ``fwd(q_rows, rows, k, v, scale, wl, wr) -> (o, lse)``.
# ---------------------------------------------------------------------------
def _loss(fwd, q, k, v, dout, scale, wl, wr):
    o, _ = fwd(q, np.arange(q.shape[0], dtype=np.int64), k, v, scale, wl, wr)
    return float((o * dout).sum())


def pin_bwd_finite_differences(bwd, fwd):
    """Each gradient element equals the central difference of
    L(Q, K, V) = sum(dO * O(Q, K, V)) computed with the forward definition
    (step 1e-5 in fp64: truncation ~1e-10, rounding ~1e-11)."""
    h = 1e-5
    for seed, (nq, nk, d, wl, wr) in enumerate([(4, 6, 3, -1, -1), (5, 5, 2, -1, 0),
                                                 (6, 4, 3, 1, 1), (3, 7, 2, 0, 2)]):
        r = _rng(300 + seed)
        q, k, v, dout = (r.standard_normal(s) for s in ((nq, d), (nk, d), (nk, d), (nq, d)))
        grads = bwd(q, k, v, dout, 0.8, wl, wr)
        for which, x in enumerate((q, k, v)):
            num = np.zeros_like(x)
            for idx in np.ndindex(*x.shape):
                args = [q.copy(), k.copy(), v.copy()]
                args[which][idx] += h
                lp = _loss(fwd, *args, dout, 0.8, wl, wr)
                args[which][idx] -= 2 * h
                lm = _loss(fwd, *args, dout, 0.8, wl, wr)
                num[idx] = (lp - lm) / (2 * h)
            np.testing.assert_allclose(grads[which], num, rtol=1e-6, atol=1e-8,
                                       err_msg=f"grad {'qkv'[which]} band {(wl, wr)}")


def pin_bwd_single_key(bwd, fwd):
    """One key: the softmax is constant 1, so dQ = dK = 0 exactly and
    dV = sum_i dO_i."""
    r = _rng(310)
    q, dout = r.standard_normal((5, 4)), r.standard_normal((5, 4))
    k, v = r.standard_normal((1, 4)), r.standard_normal((1, 4))
    dq, dk, dv = bwd(q, k, v, dout, 0.6, -1, -1)
    assert np.array_equal(dq, np.zeros_like(dq)) and np.array_equal(dk, np.zeros_like(dk))
    np.testing.assert_allclose(dv[0], dout.sum(0), rtol=1e-14, atol=1e-14)


def pin_bwd_sums(bwd, fwd):
    """Rows of the softmax Jacobian sum to zero, so sum_j dK_j = 0; weights
    sum to one, so sum_j dV_j = sum_i dO_i (unmasked and causal)."""
    r = _rng(311)
    n, d = 9, 5
    q, k, v, dout = (r.standard_normal((n, d)) for _ in range(4))
    for wl, wr in [(-1, -1), (-1, 0), (2, 1)]:
        dq, dk, dv = bwd(q, k, v, dout, 0.7, wl, wr)
        np.testing.assert_allclose(dk.sum(0), np.zeros(d), atol=1e-12)
        np.testing.assert_allclose(dv.sum(0), dout.sum(0), rtol=1e-12, atol=1e-12)


def pin_bwd_linear_in_cotangent(bwd, fwd):
    """The gradients are linear in dO."""
    r = _rng(312)
    q, k, v = r.standard_normal((6, 4)), r.standard_normal((8, 4)), r.standard_normal((8, 4))
    g1, g2 = r.standard_normal((6, 4)), r.standard_normal((6, 4))
    a = bwd(q, k, v, g1, 0.5, -1, -1)
    b = bwd(q, k, v, g2, 0.5, -1, -1)
    c = bwd(q, k, v, 2.0 * g1 - 3.0 * g2, 0.5, -1, -1)
    for x, y, z in zip(a, b, c):
        np.testing.assert_allclose(z, 2.0 * x - 3.0 * y, rtol=1e-11, atol=1e-12)


def pin_bwd_dv_is_pt_dout(bwd, fwd):
    """dV = P^T dO with P the materialised softmax of the (independent)
    numpy masked-attention construction."""
    r = _rng(313)
    nq, nk, d = 7, 9, 3
    q, k, v = r.standard_normal((nq, d)), r.standard_normal((nk, d)), r.standard_normal((nk, d))
    dout = r.standard_normal((nq, d))
    for wl, wr in [(-1, -1), (3, 0)]:
        mask = band_mask_numpy(nq, nk, wl, wr)
        s = np.where(mask, 0.9 * (q @ k.T), -np.inf)
        p = np.exp(s - s.max(1, keepdims=True))
        p /= p.sum(1, keepdims=True)
        _, _, dv = bwd(q, k, v, dout, 0.9, wl, wr)
        np.testing.assert_allclose(dv, p.T @ dout, rtol=1e-12, atol=1e-12)


def pin_bwd_golden(bwd, fwd):
    """Hand-derived gradients stored under tests/golden/."""
    with open(os.path.join(os.path.dirname(GOLDEN), "bwd_closed_forms.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        q, k, v, g = (np.array(c[x], dtype=np.float64) for x in ("q", "k", "v", "dout"))
        dq, dk, dv = bwd(q, k, v, g, c["scale"], *c["window"])
        for name, got in (("dq", dq), ("dk", dk), ("dv", dv)):
            np.testing.assert_allclose(got, np.array(c[name]), rtol=1e-13, atol=1e-13,
                                       err_msg=f"{c['name']} {name}")


BWD_PINS = [pin_bwd_finite_differences, pin_bwd_single_key, pin_bwd_sums,
            pin_bwd_linear_in_cotangent, pin_bwd_dv_is_pt_dout, pin_bwd_golden]


# ---------------------------------------------------------------------------
# Backward of a packed variable-length batch.  These take
# ``attn_bwd_varlen(q, k, v, dout, cu_q, cu_k, scale, wl, wr)`` and
# ``attn_varlen(q, k, v, cu_q, cu_k, scale, wl, wr)``.
# ---------------------------------------------------------------------------
def _varlen_loss(attn_varlen, q, k, v, dout, cu_q, cu_k, scale, wl, wr):
    total = 0.0
    for (s, h), (rows, o, _) in attn_varlen(q, k, v, cu_q, cu_k, scale, wl, wr).items():
        total += float((o * dout[int(cu_q[s]) + rows, h]).sum())
    return total


def pin_bwd_varlen_finite_differences(attn_bwd_varlen, attn_varlen):
    """Every owned gradient element of a packed batch (an empty sequence, a
    sequence without keys, Nq != Nk per sequence, two query heads on one
    key/value head, causal and a band) equals the central difference of
    L = sum(dO * O) through the packed forward definition."""
    h = 1e-5
    cu_q = np.array([0, 3, 3, 7, 9])
    cu_k = np.array([0, 4, 6, 9, 9])
    r = _rng(330)
    d = 2
    q, dout = r.standard_normal((9, 2, d)), r.standard_normal((9, 2, d))
    k, v = r.standard_normal((9, 1, d)), r.standard_normal((9, 1, d))
    for wl, wr in [(-1, 0), (1, 1)]:
        grads = attn_bwd_varlen(q, k, v, dout, cu_q, cu_k, 0.7, wl, wr)
        for which, x in enumerate((q, k, v)):
            num = np.zeros_like(x)
            for idx in np.ndindex(*x.shape):
                args = [q.copy(), k.copy(), v.copy()]
                args[which][idx] += h
                lp = _varlen_loss(attn_varlen, *args, dout, cu_q, cu_k, 0.7, wl, wr)
                args[which][idx] -= 2 * h
                lm = _varlen_loss(attn_varlen, *args, dout, cu_q, cu_k, 0.7, wl, wr)
                num[idx] = (lp - lm) / (2 * h)
            np.testing.assert_allclose(grads[which], num, rtol=1e-6, atol=1e-8,
                                       err_msg=f"grad {'qkv'[which]} band {(wl, wr)}")


def pin_bwd_varlen_rows_outside_sequences(attn_bwd_varlen, attn_varlen):
    """Rows no sequence owns: dQ = 0 there, and the owned gradients do not
    depend on their data (the outside rows are refilled with other values)."""
    cu_q = np.array([1, 4, 6])
    cu_k = np.array([0, 3, 5])
    r = _rng(331)
    q, dout = r.standard_normal((8, 1, 3)), r.standard_normal((8, 1, 3))
    k, v = r.standard_normal((7, 1, 3)), r.standard_normal((7, 1, 3))
    dq, dk, dv = attn_bwd_varlen(q, k, v, dout, cu_q, cu_k, 0.5, -1, 0)
    assert np.all(dq[[0, 6, 7]] == 0.0)
    q2, k2, v2, do2 = q.copy(), k.copy(), v.copy(), dout.copy()
    q2[[0, 6, 7]] += 5.0
    do2[[0, 6, 7]] -= 3.0
    k2[5:] *= -2.0
    v2[5:] += 1.0
    dq2, dk2, dv2 = attn_bwd_varlen(q2, k2, v2, do2, cu_q, cu_k, 0.5, -1, 0)
    assert np.array_equal(dq[1:6], dq2[1:6])
    assert np.array_equal(dk[:5], dk2[:5]) and np.array_equal(dv[:5], dv2[:5])


BWD_VARLEN_PINS = [pin_bwd_varlen_finite_differences, pin_bwd_varlen_rows_outside_sequences]
