"""Fit the degree-3 polynomial for 2^f on [0, 1) used by the kernel's
FMA-pipe exp2 (sm100_ptx.cuh, exp2_poly2).

Remez exchange on the relative error (p(f) - 2^f) / 2^f: solve for the
polynomial that equioscillates on deg + 2 reference points, move the
reference to the extrema of the new error, repeat.  Prints the coefficients
as fp32 hex floats and the max relative error of the fp32 Horner evaluation.

    python exact_blockwise_head_b200/csrc/fit_exp2_poly.py
"""
import numpy as np


def remez_exp2(deg=3, iters=50, grid=200001):
    n = deg + 2
    x = 0.5 - 0.5 * np.cos(np.pi * np.arange(n) / (n - 1))
    g = np.linspace(0.0, 1.0, grid)
    for _ in range(iters):
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], g) - 2.0 ** g) / 2.0 ** g
        idx = [0]
        sgn = np.sign(np.diff(err))
        idx += [k for k in range(1, len(sgn)) if sgn[k] != sgn[k - 1]]
        idx.append(len(g) - 1)
        if len(idx) == n:
            x = g[np.array(idx)]
    return c


def horner_f32(c, f):
    cf = np.float32(c)
    p = np.full_like(f, cf[-1])
    for k in range(len(cf) - 2, -1, -1):
        p = (p.astype(np.float64) * f + cf[k]).astype(np.float32)  # one rounding per FMA
    return p


if __name__ == "__main__":
    c = remez_exp2()
    f = np.linspace(0, 1, 1_000_001, dtype=np.float32)[:-1]
    p = horner_f32(c, f)
    rel = np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1).max()
    for k, v in enumerate(np.float32(c)):
        print(f"C{k} = {float(v).hex()}  ({float(v):.8f})")
    print(f"max relative error of the fp32 evaluation on [0, 1): {rel:.3e}")
