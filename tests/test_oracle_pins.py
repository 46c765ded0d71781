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


@pytest.mark.parametrize("pin", pins.WINDOW_PINS, ids=[p.__name__ for p in pins.WINDOW_PINS])
def test_oracle_window_pin(pin):
    pin(oracle.attn_rows_window)


@pytest.mark.parametrize("pin", pins.VARLEN_PINS, ids=[p.__name__ for p in pins.VARLEN_PINS])
def test_oracle_varlen_pin(pin):
    pin(oracle.attn_varlen)


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

    return attn_rows, attn_rows_window


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    rows_fn, window_fn = _build_mutant(tmp_path, name, old, new)
    failed = []
    for pin_set, fn in ((PINS, rows_fn), (pins.WINDOW_PINS, window_fn)):
        for pin in pin_set:
            try:
                pin(fn)
            except AssertionError:
                failed.append(pin.__name__)
    assert failed, f"no pin catches the planted mistake {name}"
