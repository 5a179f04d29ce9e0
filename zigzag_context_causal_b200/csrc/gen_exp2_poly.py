"""Coefficients of the FMA-pipe 2^x used for part of the softmax exponentials.

2^x = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2].  2^f is replaced
by its degree-3 Chebyshev interpolant on [-1/2, 1/2] (interpolation at the four
Chebyshev nodes, which is within a small factor of the minimax polynomial).
Running this script prints the coefficients (monomial basis, c0..c3) and the
worst relative error over the interval; exp2_poly.h holds the printed values.

    python zigzag_context_causal_b200/csrc/gen_exp2_poly.py
"""
import numpy as np


def coefficients(degree: int = 3):
    k = np.arange(degree + 1)
    nodes = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * (degree + 1)))   # Chebyshev nodes on [-1/2, 1/2]
    vander = np.vander(nodes, degree + 1, increasing=True)
    return np.linalg.solve(vander, 2.0 ** nodes)


def max_rel_error(c) -> float:
    f = np.linspace(-0.5, 0.5, 200001)
    p = np.polyval(c[::-1], f)
    return float(np.max(np.abs(p / 2.0 ** f - 1.0)))


if __name__ == "__main__":
    c = coefficients()
    for i, x in enumerate(c):
        print(f"c{i} = {np.float32(x)!r:>14}  ({x:.17g})")
    print(f"max relative error on [-1/2, 1/2]: {max_rel_error(c):.3e}")
