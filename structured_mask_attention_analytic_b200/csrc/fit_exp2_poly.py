"""Coefficients of the cubic that the attention softmax uses for 2^f on the
FMA pipe (``exp2_fma`` in device_common.cuh).

2^t is split as 2^n * 2^f with n = round(t) and f = t - n in [-1/2, 1/2];
2^f is approximated by a cubic c0 + c1 f + c2 f^2 + c3 f^3 whose largest
RELATIVE error over [-1/2, 1/2] is made as small as this fit can: a
least-squares fit at Chebyshev nodes, weighted by 1 / 2^f, with the weights
then raised where the error is largest (Lawson's iteration towards the
minimax fit).  The coefficients are rounded to float32, and the error is
measured again on the rounded cubic evaluated in float32 with Horner's
rule, as the kernel evaluates it.

Usage: ``python -m structured_mask_attention_analytic_b200.csrc.fit_exp2_poly``
prints the coefficients and the error bound.
"""
from __future__ import annotations

import numpy as np


def fit(degree: int = 3, nodes: int = 400, iters: int = 200):
    k = np.arange(nodes)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / nodes)          # Chebyshev nodes on [-1/2, 1/2]
    y = np.exp2(f)
    a = np.vander(f, degree + 1, increasing=True) / y[:, None]   # relative residual rows
    b = np.ones_like(f)
    w = np.ones_like(f)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(a * sw[:, None], b * sw, rcond=None)
        err = np.abs(a @ c - b)
        w = w * err
        w /= w.sum()
    return c


def max_rel_error_float32(c) -> float:
    c32 = np.asarray(c, dtype=np.float32)
    f = np.linspace(-0.5, 0.5, 200001, dtype=np.float32)
    p = c32[-1] * np.ones_like(f)
    for ci in c32[-2::-1]:
        p = (p * f + ci).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)))


def main() -> None:
    c = fit()
    for i, ci in enumerate(np.asarray(c, dtype=np.float32)):
        print(f"c{i} = {float(ci):.9e}f")
    print(f"max relative error (float32 Horner): {max_rel_error_float32(c):.3e}")


if __name__ == "__main__":
    main()
