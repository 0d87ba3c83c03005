"""Coefficients of the cubic that attention kernels use for part of their 2^f.

    python block_sparse_local_b200/csrc/gen_exp2_poly.py

Remez exchange (minimax in relative error) for p(f) ~ 2^f on [-1/2, 1/2],
degree 3, in float64; prints the float32 coefficients that exp2_poly() in
device_ptx.cuh holds and the relative error bound of their float32 Horner
evaluation (about 7.5e-5, well under the 2^-9 rounding of the bf16 P).
"""
import numpy as np


def remez(n=3, a=-0.5, b=0.5, iters=40, grid=200001):
    k = np.arange(n + 2)
    x = (a + b) / 2 + (b - a) / 2 * np.cos(np.pi * k[::-1] / (n + 1))
    g = np.linspace(a, b, grid)
    coef = None
    for _ in range(iters):
        # p(x_i) + (-1)^i E 2^x_i = 2^x_i  (equioscillating relative error)
        A = np.zeros((n + 2, n + 2))
        for i, xi in enumerate(x):
            A[i, :n + 1] = xi ** np.arange(n + 1)
            A[i, n + 1] = (-1) ** i * 2.0 ** xi
        coef = np.linalg.solve(A, 2.0 ** x)[:n + 1]
        err = np.polyval(coef[::-1], g) / 2.0 ** g - 1
        d = np.diff(err)
        cand = np.concatenate(([0], np.where(np.sign(d[:-1]) != np.sign(d[1:]))[0] + 1,
                               [len(g) - 1]))
        sel = []
        for ci in cand:
            if sel and np.sign(err[sel[-1]]) == np.sign(err[ci]):
                if abs(err[ci]) > abs(err[sel[-1]]):
                    sel[-1] = ci
            else:
                sel.append(ci)
        while len(sel) > n + 2:
            sel.pop(0 if abs(err[sel[0]]) < abs(err[sel[-1]]) else -1)
        if len(sel) == n + 2:
            x = g[sel]
    return coef


def coefficients():
    return [float(np.float32(c)) for c in remez()]


def horner_f32(c, f):
    f = np.asarray(f, dtype=np.float32)
    p = np.float32(c[3])
    for i in (2, 1, 0):
        p = (p * f + np.float32(c[i])).astype(np.float32)
    return p


if __name__ == "__main__":
    c = coefficients()
    f = np.linspace(-0.5, 0.5, 100001, dtype=np.float32)
    rel = np.abs(horner_f32(c, f).astype(np.float64) / 2.0 ** f.astype(np.float64) - 1).max()
    for i, v in enumerate(c):
        print(f"c{i} = {v!r}  ({np.float32(v).view(np.uint32):#010x})")
    print(f"max relative error of the float32 evaluation: {rel:.3e}")
