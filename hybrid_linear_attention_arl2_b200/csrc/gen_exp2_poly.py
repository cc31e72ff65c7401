"""Coefficients of the polynomial 2^f ~= c0 + c1 f + ... + cn f^n on f in [-1/2, 1/2]
used by the attention kernel's FMA-pipe exp2 (sm100.cuh, exp2_poly).

Method: interpolation at the Chebyshev nodes of [-1/2, 1/2] (near-minimax for a
smooth function), solved in float64 and rounded to float32.  Prints the
coefficients and the worst relative error of the float32 Horner evaluation over
a dense grid.  Run:  python gen_exp2_poly.py [degree]
"""
import sys

import numpy as np


def coefficients(deg: int) -> np.ndarray:
    k = np.arange(deg + 1)
    nodes = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * (deg + 1)))
    V = np.vander(nodes, deg + 1, increasing=True)
    return np.linalg.solve(V, np.exp2(nodes))


def horner32(c: np.ndarray, f: np.ndarray) -> np.ndarray:
    c = c.astype(np.float32)
    f = f.astype(np.float32)
    acc = np.full_like(f, c[-1])
    for a in c[-2::-1]:
        acc = (acc * f + a).astype(np.float32)
    return acc


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c = coefficients(deg)
    f = np.linspace(-0.5, 0.5, 200001)
    err = np.max(np.abs(horner32(c, f).astype(np.float64) / np.exp2(f) - 1.0))
    print("degree", deg, "coefficients (float32):", ", ".join(f"{float(np.float32(x)):.9g}f" for x in c))
    print(f"max relative error on [-1/2, 1/2]: {err:.3e}")
