"""Writes slay_exp2_poly.h: a degree-3 polynomial for 2^f on [-1/2, 1/2].

The tensor-core feature map evaluates part of its exponentials on the FMA pipe instead of
the special-function unit: 2^x = 2^j * 2^f with j = round(x) and f = x - j in [-1/2, 1/2]
(Cody-Waite range reduction), and 2^f from this polynomial.  The coefficients minimise the
largest relative error max |p(f) / 2^f - 1| over a dense grid of the interval (a minimax fit
posed as a linear program); they are then rounded to float32 and the error of the float32
Horner evaluation is measured and written beside them.  The features are stored in bf16,
whose rounding error is 2^-9 relative, so a relative error near 1e-4 is invisible there.

Run from this directory:  python gen_exp2_poly.py  (numpy + scipy).
"""
import os

import numpy as np
from scipy.optimize import linprog

DEGREE = 3


def fit(degree=DEGREE, n=4001):
    f = np.linspace(-0.5, 0.5, n)
    y = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True)          # columns 1, f, f^2, ...
    # variables c_0..c_d, t; minimise t subject to |V c - y| <= t y
    nv = degree + 2
    cost = np.zeros(nv)
    cost[-1] = 1.0
    A = np.vstack([np.hstack([V, -y[:, None]]), np.hstack([-V, -y[:, None]])])
    b = np.concatenate([y, -y])
    res = linprog(cost, A_ub=A, b_ub=b, bounds=[(None, None)] * nv, method="highs")
    assert res.status == 0, res.message
    return res.x[:-1]


def horner_f32(c, f):
    f = f.astype(np.float32)
    p = np.full_like(f, np.float32(c[-1]))
    for ck in c[-2::-1]:
        p = (p * f + np.float32(ck)).astype(np.float32)
    return p


def max_rel_error_f32(c, n=200001):
    f = np.linspace(-0.5, 0.5, n).astype(np.float32)
    p = horner_f32(np.asarray(c, dtype=np.float32), f).astype(np.float64)
    return float(np.max(np.abs(p / np.exp2(f.astype(np.float64)) - 1.0)))


def main():
    c = np.asarray(fit(), dtype=np.float32)
    err = max_rel_error_f32(c)
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "slay_exp2_poly.h")
    with open(path, "w") as fh:
        fh.write("// slay_exp2_poly.h -- written by gen_exp2_poly.py; do not edit.\n")
        fh.write("// 2^f ~= c0 + c1 f + c2 f^2 + c3 f^3 on [-1/2, 1/2], minimax in relative error;\n")
        fh.write("// largest relative error of the float32 Horner evaluation: %.3e\n" % err)
        fh.write("#pragma once\n\n")
        for k, ck in enumerate(c):
            fh.write("#define SLAY_EXP2_C%d %.9ef\n" % (k, float(ck)))
        fh.write("#define SLAY_EXP2_MAX_REL_ERR %.3e\n" % err)
    print("wrote", path, "max rel err %.3e" % err, c)


if __name__ == "__main__":
    main()
