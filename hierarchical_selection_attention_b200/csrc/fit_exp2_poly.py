"""Coefficients of the degree-4 polynomial for 2^f on [-1/2, 1/2] used by
exp2_poly in lh_sm100.cuh.

Method: interpolate g(f) = 2^f at the 5 Chebyshev nodes of [-1/2, 1/2]
(near-minimax for a smooth function), then round the coefficients to fp32.
Prints the coefficients (hex, as written in the CUDA source) and the maximum
relative error of the fp32 polynomial over the interval.

    python fit_exp2_poly.py
"""
import numpy as np


def coefficients(deg: int = 4) -> np.ndarray:
    k = np.arange(deg + 1)
    nodes = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * (deg + 1)))
    V = np.vander(nodes, deg + 1, increasing=True)
    return np.linalg.solve(V, np.exp2(nodes)).astype(np.float32)


def max_rel_error(c32: np.ndarray) -> float:
    f = np.linspace(-0.5, 0.5, 200001)
    p = np.zeros_like(f)
    for c in c32[::-1].astype(np.float64):
        p = p * f + c
    return float(np.max(np.abs(p / np.exp2(f) - 1.0)))


if __name__ == "__main__":
    c32 = coefficients()
    for i, c in enumerate(c32):
        print(f"c{i} = {float(c).hex()}  ({float(c):.9g})")
    print(f"max relative error on [-1/2, 1/2]: {max_rel_error(c32):.3e}")
