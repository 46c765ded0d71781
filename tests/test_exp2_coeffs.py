"""Provenance of the FMA-pipe exp2 cubic in csrc/exp2.cuh (CPU, no GPU).

2^x is evaluated as 2^n * p(f) with n = round-to-nearest(x), f = x - n in
[-1/2, 1/2] and p(f) = 1 + f*(c1 + f*(c2 + f*c3)): the constant term is pinned
to exactly 1 so that exp2(0) == 1 bit-exactly (a lone visible key then gets
weight exactly 1).  c1..c3 minimise the maximum relative error |p(f)/2^f - 1|
over [-1/2, 1/2].  This test solves that minimax problem again, as a linear
program on a dense grid, and checks that the constants compiled into the
kernel are its solution rounded to fp32, with the error bound the kernel's
comments and the parity tolerances rely on."""
import os
import re

import numpy as np
import pytest

CUH = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "exact_attention_152_b200", "csrc", "exp2.cuh")


def _kernel_coeffs():
    src = open(CUH).read()
    out = {}
    for name in ("kExpC1", "kExpC2", "kExpC3"):
        m = re.search(rf"constexpr float {name} = ([0-9a-fx.p+-]+)f;", src)
        assert m, name
        out[name] = np.float32(float.fromhex(m.group(1)))
    return out["kExpC1"], out["kExpC2"], out["kExpC3"]


def _fit():
    linprog = pytest.importorskip("scipy.optimize").linprog
    f = np.linspace(-0.5, 0.5, 20001)
    t = np.exp2(f)
    # variables c1, c2, c3, e; minimise e subject to |(1 + c1 f + c2 f^2 + c3 f^3)/t - 1| <= e
    a = np.stack([f / t, f ** 2 / t, f ** 3 / t], axis=1)
    b = 1.0 - 1.0 / t
    a_ub = np.vstack([np.hstack([a, -np.ones((len(f), 1))]), np.hstack([-a, -np.ones((len(f), 1))])])
    b_ub = np.concatenate([b, -b])
    res = linprog(c=[0, 0, 0, 1], A_ub=a_ub, b_ub=b_ub, bounds=[(None, None)] * 4, method="highs")
    assert res.status == 0
    return res.x


def _horner_f32(c1, c2, c3, f):
    p = np.float32(c3) * f + np.float32(c2)
    p = p * f + np.float32(c1)
    return p * f + np.float32(1.0)


def test_kernel_coefficients_are_the_minimax_fit():
    c1, c2, c3, err = _fit()
    k1, k2, k3 = _kernel_coeffs()
    for fit, kern in ((c1, k1), (c2, k2), (c3, k3)):
        # the kernel holds the fit rounded to fp32 (one fp32 ulp of slack for
        # the LP solver's own tolerance)
        assert abs(np.float64(kern) - fit) <= 2.0 * np.spacing(np.float32(abs(fit))), (kern, fit)
    assert 0.9e-4 < err < 1.05e-4


def test_fp32_horner_error_and_exact_one():
    k1, k2, k3 = _kernel_coeffs()
    f = np.linspace(-0.5, 0.5, 1000001).astype(np.float32)
    rel = np.abs(_horner_f32(k1, k2, k3, f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1).max()
    # below BF16's unit roundoff 2^-8 by a factor of ~38
    assert rel < 1.02e-4, rel
    assert _horner_f32(k1, k2, k3, np.float32(0.0)) == np.float32(1.0)
