"""Coefficients of the degree-4 polynomial for 2^f, f in [-1/2, 1/2], used by the softmax
kernels' FMA-pipe exponentials (veda_ptx.cuh, exp2_fma_x2).

Relative error is minimised by least squares at Chebyshev nodes, reweighted by Lawson's
iteration (weights multiplied by the current error) toward the minimax fit. Prints the
coefficients rounded to fp32 and the maximum relative error in fp64.
"""
import numpy as np


def fit(degree: int = 4, nodes: int = 4001, iterations: int = 200):
    f = 0.5 * np.cos(np.pi * (np.arange(nodes) + 0.5) / nodes)
    y = np.exp2(f)
    a = np.vander(f, degree + 1, increasing=True) / y[:, None]
    b = np.ones_like(f)
    w = np.full_like(f, 1.0 / nodes)
    c = None
    for _ in range(iterations):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(a * sw[:, None], b * sw, rcond=None)
        w = w * np.abs(a @ c - b)
        w /= w.sum()
    return c.astype(np.float32), float(np.abs(a @ c - b).max())


if __name__ == "__main__":
    coeffs, err = fit()
    for k, v in enumerate(coeffs):
        print(f"C{k} = {float(v)!r}")
    print(f"max relative error (fp64): {err:.3g}")
