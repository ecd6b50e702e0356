"""Coefficients of the cubic that approximates 2^f on f in [-1/2, 1/2].

Used by the tensor-core prefill kernel to evaluate part of its exponentials
on the FMA pipe (2^x = 2^n * 2^f, n = round(x): Cody-Waite style range
reduction, n added to the float's exponent field).  The cubic is the
least-squares fit of 2^f at 2001 Chebyshev nodes of [-1/2, 1/2], which is
close to the minimax fit; its relative error bound is printed and is far
below the bfloat16 rounding (2^-9) applied to P right after.

    python reference_sliding_window_b200/csrc/fit_exp2.py
"""

import numpy as np


def fit(degree: int = 3, nodes: int = 2001):
    k = np.arange(nodes)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / nodes)      # Chebyshev nodes in [-1/2, 1/2]
    A = np.vander(f, degree + 1, increasing=True)
    c, *_ = np.linalg.lstsq(A / np.exp2(f)[:, None], np.ones_like(f), rcond=None)  # relative LSQ
    return c


def max_rel_error(c, n: int = 200001) -> float:
    f = np.linspace(-0.5, 0.5, n)
    approx = np.polyval(c[::-1], f)
    return float(np.max(np.abs(approx / np.exp2(f) - 1.0)))


if __name__ == "__main__":
    c = fit()
    for i, ci in enumerate(c):
        print(f"c{i} = {np.float32(ci)!r}")
    print("max relative error on [-1/2, 1/2]:", max_rel_error(c))
