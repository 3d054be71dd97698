"""Fits the polynomial the attention softmax uses for part of its exp2.

2^x is split (Cody and Waite's range reduction) as 2^n * 2^f with n the
nearest integer to x and f = x - n in [-1/2, 1/2]; 2^f is approximated by a
degree-3 polynomial whose coefficients minimise the maximum relative error
on that interval: a Remez exchange on the relative error, with deg + 2
alternation points started from Chebyshev nodes.

Run ``python fit_exp2_poly.py`` to print the coefficients (as float32) and
the maximum relative error of the float32 Horner evaluation; attn_sm100.cu
holds the printed values.
"""
import numpy as np


def remez_rel(deg=3, lo=-0.5, hi=0.5, iters=40):
    k = deg + 2
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * np.arange(k)[::-1] / (k - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # sum_j c_j x^j / 2^x - 1 = (-1)^i E at the k points
        A = np.zeros((k, deg + 2))
        for i, xi in enumerate(x):
            w = 2.0 ** (-xi)
            A[i, :deg + 1] = [xi ** j * w for j in range(deg + 1)]
            A[i, deg + 1] = -((-1) ** i)
        c = np.linalg.solve(A, np.ones(k))[:deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        idx = [0] + [i for i in range(1, len(grid) - 1)
                     if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0] + [len(grid) - 1]
        cand, vals = grid[idx], np.abs(err[idx])
        x = np.sort(cand[np.argsort(-vals)[:k]])
    return c, np.abs(err).max()


def eval_f32(c, f):
    f = f.astype(np.float32)
    c = c.astype(np.float32)
    r = c[3]
    for j in (2, 1, 0):
        r = (r * f + c[j]).astype(np.float32)
    return r


if __name__ == "__main__":
    c, e = remez_rel()
    c32 = c.astype(np.float32)
    f = np.linspace(-0.5, 0.5, 1000001)
    rel = np.abs(eval_f32(c32, f).astype(np.float64) / 2.0 ** f - 1.0).max()
    print("coefficients c0..c3 (float32):", [float(v) for v in c32])
    print("hex:", [hex(np.float32(v).view(np.uint32)) for v in c32])
    print(f"max relative error: fit {e:.3e}, float32 evaluation {rel:.3e}")
