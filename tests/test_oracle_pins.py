"""The oracle, pinned to facts that do not come from it (CPU only)."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle
import oracle_pins as pins

PINS = pins.ALL_PINS


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_pin(pin):
    pin(oracle.attn_rows)


@pytest.mark.parametrize("pin", pins.BWD_VARLEN_PINS, ids=[p.__name__ for p in pins.BWD_VARLEN_PINS])
def test_oracle_bwd_varlen_pin(pin):
    pin(oracle.attn_bwd_varlen, oracle.attn_varlen)


def test_bwd_varlen_pin_catches_wrong_offsets():
    """A packed backward that reads each sequence's keys one row too late is
    caught by the finite-difference pin."""
    def shifted(q, k, v, dout, cu_q, cu_k, scale, wl, wr):
        return oracle.attn_bwd_varlen(q, k, v, dout, cu_q, np.minimum(np.asarray(cu_k) + 1, k.shape[0]),
                                      scale, wl, wr)
    with pytest.raises(AssertionError):
        pins.pin_bwd_varlen_finite_differences(shifted, oracle.attn_varlen)


@pytest.mark.parametrize("pin", pins.BWD_COLMASK_PINS, ids=[p.__name__ for p in pins.BWD_COLMASK_PINS])
def test_oracle_bwd_colmask_pin(pin):
    pin(oracle.attn_bwd_colmask_head, oracle.attn_rows_colmask)


@pytest.mark.parametrize("pin", pins.COLMASK_PINS, ids=[p.__name__ for p in pins.COLMASK_PINS])
def test_oracle_colmask_pin(pin):
    pin(oracle.attn_rows_colmask)


@pytest.mark.parametrize("pin", pins.WINDOW_PINS, ids=[p.__name__ for p in pins.WINDOW_PINS])
def test_oracle_window_pin(pin):
    pin(oracle.attn_rows_window)


@pytest.mark.parametrize("pin", pins.VARLEN_PINS, ids=[p.__name__ for p in pins.VARLEN_PINS])
def test_oracle_varlen_pin(pin):
    pin(oracle.attn_varlen)


@pytest.mark.parametrize("pin", pins.BWD_PINS, ids=[p.__name__ for p in pins.BWD_PINS])
def test_oracle_bwd_pin(pin):
    pin(oracle.attn_bwd_head, oracle.attn_rows_window)


def test_bwd_group_sum_and_threads():
    """Grouped key/value heads: the shared head's gradients are the sums over its
    query heads, whatever the thread count."""
    r = np.random.default_rng(7)
    q, g = r.standard_normal((2, 4, 6, 3)), r.standard_normal((2, 4, 6, 3))
    k, v = r.standard_normal((2, 2, 5, 3)), r.standard_normal((2, 2, 5, 3))
    dq, dk, dv = oracle.attn_bwd(q, k, v, g, 0.5, -1, 0, nthreads=1)
    dq2, dk2, dv2 = oracle.attn_bwd(q, k, v, g, 0.5, -1, 0, nthreads=5)
    assert np.array_equal(dk, dk2) and np.array_equal(dv, dv2) and np.array_equal(dq, dq2)
    for b in range(2):
        for hk in range(2):
            parts = [oracle.attn_bwd_head(q[b, h], k[b, hk], v[b, hk], g[b, h], 0.5, -1, 0)
                     for h in (2 * hk, 2 * hk + 1)]
            np.testing.assert_allclose(dk[b, hk], parts[0][1] + parts[1][1], rtol=1e-15, atol=1e-15)
            np.testing.assert_allclose(dv[b, hk], parts[0][2] + parts[1][2], rtol=1e-15, atol=1e-15)


def test_full_tensor_wrapper_matches_rows():
    r = np.random.default_rng(5)
    q, k, v = (r.standard_normal((2, 3, 9, 4)) for _ in range(3))
    o, lse = oracle.attn_fwd(q, k, v, 0.5, causal=True)
    for b in range(2):
        for h in range(3):
            o1, l1 = oracle.attn_rows(q[b, h], np.arange(9), k[b, h], v[b, h], 0.5, True)
            assert np.array_equal(o[b, h], o1) and np.array_equal(lse[b, h], l1)


def test_thread_count_does_not_change_result():
    r = np.random.default_rng(6)
    q, k, v = r.standard_normal((50, 16)), r.standard_normal((70, 16)), r.standard_normal((70, 16))
    rows = np.arange(50)
    a = oracle.attn_rows(q, rows, k, v, 0.25, False, nthreads=1)
    b = oracle.attn_rows(q, rows, k, v, 0.25, False, nthreads=7)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


# ---------------------------------------------------------------------------
# Planted mistakes: each mutant of the oracle's C source must fail some pin.
# The mutants are built in a temporary directory; the real oracle is untouched.
# ---------------------------------------------------------------------------
MUTANTS = {
    "dropped_scale": ("s[j - lo] = jb->scale * dot;", "s[j - lo] = dot;"),
    "causal_off_by_one": ("hi = i + jb->window_right;", "hi = i + jb->window_right - 1;"),
    "window_left_off_by_one": ("lo = i - jb->window_left;", "lo = i - jb->window_left + 1;"),
    "window_right_ignored": ("if (jb->window_right >= 0 && i + jb->window_right < hi)",
                             "if (0 && i + jb->window_right < hi)"),
    "lse_without_max": ("jb->lse[r] = m + log(l);", "jb->lse[r] = log(l);"),
    "unnormalised_weights": ("const double p = s[j] / l;", "const double p = s[j];"),
    "transposed_key_index": ("const double *kj = jb->k + j * d;", "const double *kj = jb->k + j;"),
    "max_sign_flip": ("if (s[j] > m) m = s[j];", "if (s[j] < m) m = s[j];"),
    "wrong_value_row": ("const double *vj = jb->v + (lo + j) * d;",
                        "const double *vj = jb->v + (hi - j) * d;"),
    "value_row_not_offset": ("const double *vj = jb->v + (lo + j) * d;",
                             "const double *vj = jb->v + j * d;"),
    "bwd_dropped_D": ("const double ds = p[j] * (dp[j] - D);", "const double ds = p[j] * dp[j];"),
    "bwd_dk_without_scale": ("dk[j * d + c] += scale * ds * qi[c];", "dk[j * d + c] += ds * qi[c];"),
    "bwd_dq_wrong_operand": ("dq[i * d + c] += scale * ds * k[j * d + c];",
                             "dq[i * d + c] += scale * ds * v[j * d + c];"),
    "bwd_dv_with_ds": ("dv[j * d + c] += p[j] * gi[c];", "dv[j * d + c] += ds * gi[c];"),
    "bwd_dp_against_k": ("for (int64_t c = 0; c < d; ++c) dot += gi[c] * v[j * d + c];",
                         "for (int64_t c = 0; c < d; ++c) dot += gi[c] * k[j * d + c];"),
    "cols_hi_inclusive": ("(c[0] <= i && i < c[1])", "(c[0] <= i && i <= c[1])"),
    "cols_second_interval_ignored": ("(c[2] <= i && i < c[3])", "(0 && i < c[3])"),
    "cols_causal_ignored": ("(jb->causal && j > i)", "(0 && j > i)"),
    "cols_value_not_gathered": ("const double *vj = jb->v + jb->vis[t] * d;",
                                "const double *vj = jb->v + t * d;"),
    "bwd_cols_second_interval_ignored": ("(c[2] <= i && i < c[3]);\n            if (!hidden) vis[n++] = j;",
                                         "(0 && i < c[3]);\n            if (!hidden) vis[n++] = j;"),
    "bwd_cols_dv_not_gathered": ("dv[j * d + c] += p[t] * gi[c];", "dv[t * d + c] += p[t] * gi[c];"),
    "bwd_band_ignored": ("if (window_right >= 0 && i + window_right < hi) hi = i + window_right;",
                         "if (0) hi = i + window_right;"),
}


def _build_mutant(tmp_path, name, old, new):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "attn_oracle.c")).read()
    assert old in src, f"mutation anchor missing for {name}"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    lib = tmp_path / f"lib{name}.so"
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-fPIC", "-shared", "-pthread",
                    "-o", str(lib), str(path), "-lm"], check=True)
    cdll = ctypes.CDLL(str(lib))
    f = cdll.oracle_attn_rows_f64
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_double,
                  ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]

    w = cdll.oracle_attn_rows_window_f64
    w.restype = ctypes.c_int
    w.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_double,
                  ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]

    def call(fn, q_rows, rows, k, v, scale, *mask):
        q_rows = np.ascontiguousarray(q_rows, dtype=np.float64)
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        k = np.ascontiguousarray(k, dtype=np.float64)
        v = np.ascontiguousarray(v, dtype=np.float64)
        n, d = q_rows.shape
        o = np.empty((n, d))
        lse = np.empty(n)
        fn(q_rows.ctypes.data, rows.ctypes.data, n, k.ctypes.data if len(k) else None,
           v.ctypes.data if len(v) else None, k.shape[0], d, float(scale), *mask,
           o.ctypes.data, lse.ctypes.data, 2)
        return o, lse

    def attn_rows(q_rows, rows, k, v, scale, causal):
        return call(f, q_rows, rows, k, v, scale, int(causal))

    def attn_rows_window(q_rows, rows, k, v, scale, wl, wr):
        return call(w, q_rows, rows, k, v, scale, int(wl), int(wr))

    cm = cdll.oracle_attn_rows_colmask_f64
    cm.restype = ctypes.c_int
    cm.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                   ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_double,
                   ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]

    def attn_rows_colmask(q_rows, rows, k, v, scale, causal, cols):
        cols = np.ascontiguousarray(cols, dtype=np.int64)
        return call(cm, q_rows, rows, k, v, scale, int(causal), cols.ctypes.data)

    b = cdll.oracle_attn_bwd_f64
    b.restype = ctypes.c_int
    b.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int64] * 3 + [ctypes.c_double] + \
        [ctypes.c_int64] * 2 + [ctypes.c_void_p] * 3

    def attn_bwd_head(q, k, v, dout, scale, wl, wr):
        q, k, v, dout = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v, dout))
        nq, d = q.shape
        nk = k.shape[0]
        dq, dk, dv = np.empty((nq, d)), np.empty((nk, d)), np.empty((nk, d))
        b(q.ctypes.data, k.ctypes.data, v.ctypes.data, dout.ctypes.data, nq, nk, d, float(scale),
          int(wl), int(wr), dq.ctypes.data, dk.ctypes.data, dv.ctypes.data)
        return dq, dk, dv

    bcm = cdll.oracle_attn_bwd_colmask_f64
    bcm.restype = ctypes.c_int
    bcm.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int64] * 3 + [ctypes.c_double, ctypes.c_int] + \
        [ctypes.c_void_p] * 4

    def attn_bwd_colmask_head(q, k, v, dout, scale, causal, cols):
        q, k, v, dout = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v, dout))
        cols = np.ascontiguousarray(cols, dtype=np.int64)
        nq, d = q.shape
        nk = k.shape[0]
        dq, dk, dv = np.empty((nq, d)), np.empty((nk, d)), np.empty((nk, d))
        bcm(q.ctypes.data, k.ctypes.data, v.ctypes.data, dout.ctypes.data, nq, nk, d, float(scale),
            int(causal), cols.ctypes.data, dq.ctypes.data, dk.ctypes.data, dv.ctypes.data)
        return dq, dk, dv

    return attn_rows, attn_rows_window, attn_bwd_head, attn_rows_colmask, attn_bwd_colmask_head


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    rows_fn, window_fn, bwd_fn, colmask_fn, bwd_cm_fn = _build_mutant(tmp_path, name, old, new)
    failed = []
    for pin_set, args in ((PINS, (rows_fn,)), (pins.WINDOW_PINS, (window_fn,)),
                          (pins.BWD_PINS, (bwd_fn, window_fn)),
                          (pins.COLMASK_PINS, (colmask_fn,)),
                          (pins.BWD_COLMASK_PINS, (bwd_cm_fn, colmask_fn))):
        for pin in pin_set:
            try:
                pin(*args)
            except AssertionError:
                failed.append(pin.__name__)
    assert failed, f"no pin catches the planted mistake {name}"


def test_bwd_colmask_per_head_masks_and_group_sums():
    """attn_bwd_colmask with one mask per query head: a head whose mask hides
    every key gets dQ = 0 and adds nothing to its key/value head's dK, dV,
    which then equal the other head's alone (two query heads on one K/V head)."""
    r = np.random.default_rng(350)
    B, H, N, d = 1, 2, 6, 3
    q, dout = r.standard_normal((B, H, N, d)), r.standard_normal((B, H, N, d))
    k, v = r.standard_normal((B, 1, N, d)), r.standard_normal((B, 1, N, d))
    mask = np.zeros((B, H, N, 4), dtype=np.int32)
    mask[0, 1, :, 0], mask[0, 1, :, 1] = 0, N  # head 1 sees nothing
    dq, dk, dv = oracle.attn_bwd_colmask(q, k, v, dout, 0.8, False, mask)
    assert np.all(dq[0, 1] == 0.0)
    a, bk, bv = oracle.attn_bwd_colmask_head(q[0, 0], k[0, 0], v[0, 0], dout[0, 0], 0.8, False, mask[0, 0])
    np.testing.assert_array_equal(dq[0, 0], a)
    np.testing.assert_array_equal(dk[0, 0], bk)
    np.testing.assert_array_equal(dv[0, 0], bv)
