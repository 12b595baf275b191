"""Derive the polynomial used by fast_exp2_fma() in csrc/fastmath.cuh.

Method: Chebyshev interpolation (the interpolant through the Chebyshev nodes of the
first kind, a classical near-minimax construction; see e.g. Trefethen, "Approximation
Theory and Approximation Practice", ch. 4 and 16) of 2^f on f in [-1/2, 1/2], converted
to monomial coefficients for Horner evaluation in fp32.  The reduced argument is
f = x - rint(x), so |f| <= 1/2.  Prints the coefficients and the max relative error
of the fp32 Horner evaluation on a dense grid.

    python rope_attention_fwd_b200/csrc/gen_exp2_poly.py [degree]
"""
import sys

import numpy as np


def coefficients(deg):
    k = np.arange(deg + 1)
    nodes = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * (deg + 1)))  # Chebyshev nodes on [-1/2, 1/2]
    V = np.vander(nodes, deg + 1, increasing=True)
    return np.linalg.solve(V, np.exp2(nodes))  # c0 + c1 f + ... + cdeg f^deg


def max_rel_err_fp32(c):
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    cf = c.astype(np.float32)
    p = np.full_like(f, cf[-1])
    for a in cf[-2::-1]:
        p = (p * f + a).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1)))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c = coefficients(deg)
    print("degree", deg, "coefficients (f^0 .. f^deg):")
    for a in c:
        print(f"  {np.float32(a).item():.9e}f")
    print("max relative error (fp32 Horner):", max_rel_err_fp32(c))
