"""Coefficients of the degree-3 polynomial used for 2^f, f in [-0.5, 0.5], on the FMA pipe.

Method: weighted least squares on 4096 Chebyshev nodes, minimising the relative
error of p(f) against 2^f (a near-minimax fit). Max relative error 7.7e-5,
below the fp16 rounding of the probabilities (4.9e-4). Prints the fp32 values
written into exp2_poly2() in fastmath.cuh (highest power first there).
"""
import numpy as np


def coefficients(degree=3, nodes=4096):
    k = np.arange(nodes)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / nodes)
    t = np.exp2(f)
    A = np.vstack([f ** i for i in range(degree + 1)]).T
    c, *_ = np.linalg.lstsq(A / t[:, None], np.ones_like(t), rcond=None)
    return c.astype(np.float32)


if __name__ == "__main__":
    c = coefficients()
    f = np.linspace(-0.5, 0.5, 200001)
    p = sum(float(c[i]) * f ** i for i in range(len(c)))
    print([f"{float(x):.9g}f" for x in c], "max rel err", float(np.max(np.abs(p / np.exp2(f) - 1))))
