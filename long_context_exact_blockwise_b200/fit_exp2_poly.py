"""Fit the polynomial the softmax uses to evaluate part of its exp2 on FMA units.

Method (standard range reduction plus a minimax fit, written from the
mathematics): write x = n + f with n = round(x) and f in [-1/2, 1/2]; then
2^x = 2^n * 2^f, where 2^n is an exponent-field add and 2^f ~ p(f), a
polynomial of degree DEG.  The coefficients minimise the maximum relative
error max |p(f) - 2^f| / 2^f over a dense grid of [-1/2, 1/2], solved
exactly as a linear program (variables c_0..c_DEG and the bound t; two
linear inequalities per grid point).  The result is then evaluated in
float32 with Horner's rule to report the error the kernel actually sees.

Run: python -m long_context_exact_blockwise_b200.fit_exp2_poly [--deg 3]
"""
from __future__ import annotations

import argparse

import numpy as np


def fit(deg: int, n_grid: int = 4001):
    from scipy.optimize import linprog

    f = np.linspace(-0.5, 0.5, n_grid)
    y = np.exp2(f)
    V = np.vander(f, deg + 1, increasing=True)        # columns f^0 .. f^deg
    # |V c - y| <= t y  <=>  V c - t y <= y  and  -V c - t y <= -y
    A = np.vstack([np.hstack([V, -y[:, None]]), np.hstack([-V, -y[:, None]])])
    b = np.concatenate([y, -y])
    cost = np.zeros(deg + 2)
    cost[-1] = 1.0
    res = linprog(cost, A_ub=A, b_ub=b, bounds=[(None, None)] * (deg + 1) + [(0, None)], method="highs")
    if not res.success:
        raise RuntimeError(res.message)
    return res.x[:-1], res.x[-1]


def float32_error(c):
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    c32 = np.asarray(c, dtype=np.float32)
    p = np.full_like(f, c32[-1])
    for k in range(len(c32) - 2, -1, -1):
        p = (p * f + c32[k]).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--deg", type=int, default=3)
    a = ap.parse_args()
    c, t = fit(a.deg)
    print(f"degree {a.deg}: minimax relative error {t:.3e}; float32 Horner {float32_error(c):.3e}")
    for k, v in enumerate(c):
        print(f"  c{k} = {np.float32(v)!r}  ({v:.12e})")


if __name__ == "__main__":
    main()
