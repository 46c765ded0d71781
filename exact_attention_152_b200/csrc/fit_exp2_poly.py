"""Fit the cubic used by the kernel's FMA-pipe exp2.

2^x is evaluated as 2^n * p(f) with n = round-to-nearest(x) and f = x - n in
[-1/2, 1/2].  p(f) = 1 + f*(c1 + f*(c2 + f*c3)): the constant term is pinned to
exactly 1 so that exp2(0) == 1 bit-exactly (a lone visible key then gets weight
exactly 1).  c1..c3 minimise the maximum relative error |p(f)/2^f - 1| over
[-1/2, 1/2]; the minimax problem is solved as a linear program on a dense grid
(scipy.optimize.linprog), then the coefficients are rounded to fp32 and the
error is re-measured with fp32 Horner evaluation.

Run:  python fit_exp2_poly.py   (prints the coefficients pasted into the kernel)
"""
import numpy as np
from scipy.optimize import linprog

f = np.linspace(-0.5, 0.5, 20001)
t = np.exp2(f)
# variables: c1, c2, c3, e ; minimise e
# |(1 + c1 f + c2 f^2 + c3 f^3)/t - 1| <= e
A = np.stack([f / t, f**2 / t, f**3 / t], axis=1)
b = 1.0 - 1.0 / t
A_ub = np.vstack([np.hstack([A, -np.ones((len(f), 1))]), np.hstack([-A, -np.ones((len(f), 1))])])
b_ub = np.concatenate([b, -b])
res = linprog(c=[0, 0, 0, 1], A_ub=A_ub, b_ub=b_ub, bounds=[(None, None)] * 4, method="highs")
c1, c2, c3, e = res.x
c = np.array([c1, c2, c3], dtype=np.float32)
fg = np.linspace(-0.5, 0.5, 1000001).astype(np.float32)
p = np.float32(c[2])
p = p * fg + c[1]
p = p * fg + c[0]
p = p * fg + np.float32(1.0)
rel = np.abs(p.astype(np.float64) / np.exp2(fg.astype(np.float64)) - 1).max()
print(f"c1={c[0]!r}  c2={c[1]!r}  c3={c[2]!r}")
print(f"c1={float(c[0]).hex()} c2={float(c[1]).hex()} c3={float(c[2]).hex()}")
print(f"LP max rel err {e:.3e}; fp32 Horner max rel err {rel:.3e}")
