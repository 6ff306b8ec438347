"""Coefficients of the FMA-pipe exp2 used by the tensor-core attention softmax.

Method: Chebyshev interpolation (nodes cos((2k+1) pi / (2n)), scaled to the
interval) of 2^f on [-1/2, 1/2] at degree 4, solved in float64 and rounded to
float32.  The kernel splits x = j + f with j = rint(x) (add and subtract
1.5 * 2^23), evaluates the polynomial in f by Horner's rule and adds j to the
exponent field.  Max relative error of the float32 evaluation: 3.6e-6
(P is then rounded to bf16, whose spacing is 2^-8).

    python rope_context_extension_scaled_b200/csrc/exp2_poly_fit.py
"""

import numpy as np


def fit(deg=4):
    n = deg + 1
    k = np.arange(n)
    nodes = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * n))
    c = np.linalg.solve(np.vander(nodes, n, increasing=True), 2.0 ** nodes)
    return c.astype(np.float32)


if __name__ == "__main__":
    c = fit()
    print(", ".join(f"{float(x):.9g}f" for x in c))
