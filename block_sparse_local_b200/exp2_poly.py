"""Derives the polynomial used for part of the exp2 evaluations in the
attention kernel's softmax (evaluated on the FMA pipe instead of MUFU).

    python -m block_sparse_local_b200.exp2_poly

Method: 2^x = 2^j * 2^f with j = round(x) and f = x - j in [-1/2, 1/2]
(Cody & Waite style range reduction); 2^f is replaced by the degree-3
polynomial p that minimises the largest relative error max|p(f)/2^f - 1| on
[-1/2, 1/2] (a linear program over a dense grid).  The coefficients printed
here are the ones in csrc/attn_fwd.cuh.  The approximation's relative error
(about 1e-4) is below the bf16 rounding applied to the probabilities.
"""
import numpy as np
from scipy.optimize import linprog


def fit(degree=3, n=4001):
    f = np.linspace(-0.5, 0.5, n)
    y = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True)      # columns f^0 .. f^deg
    # variables: c_0..c_deg, t ; minimise t s.t. |V c - y| <= t * y
    A = np.vstack([np.hstack([V, -y[:, None]]), np.hstack([-V, -y[:, None]])])
    b = np.concatenate([y, -y])
    cost = np.zeros(degree + 2)
    cost[-1] = 1.0
    res = linprog(cost, A_ub=A, b_ub=b, bounds=[(None, None)] * (degree + 2), method="highs")
    c = res.x[:-1].astype(np.float32)
    p = np.polyval(c[::-1].astype(np.float64), f)
    return c, float(np.max(np.abs(p / y - 1)))


if __name__ == "__main__":
    c, err = fit()
    print("coefficients c0..c3:", ", ".join(f"{x:.9g}f" for x in c))
    print(f"max relative error on [-0.5, 0.5]: {err:.3e}")
