"""Fit the polynomial used for the FMA-pipe 2^x in the fused kernel.

Method: range reduction x = n + f with n = round(x) (so f in [-1/2, 1/2]) and
2^x = 2^n * q(f), where q is the degree-3 polynomial minimising the maximum
RELATIVE error |q(f) / 2^f - 1| on [-1/2, 1/2], found with the Remez exchange
algorithm (equioscillation on degree + 2 reference points).  Coefficients are
rounded to float32 and the resulting float32-evaluated error is reported.

Run: python -m partitioned_attention_state_b200.csrc.fit_exp2_poly
(prints the coefficients written into exp2_poly.h).
"""

from __future__ import annotations

import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def remez(deg=DEG, lo=LO, hi=HI, iters=30):
    n = deg + 2
    # initial reference: Chebyshev extrema
    k = np.arange(n)
    xs = (lo + hi) / 2 + (hi - lo) / 2 * -np.cos(np.pi * k / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # solve sum_j c_j x_i^j - (-1)^i E 2^x_i = 2^x_i  (relative error weight 1/2^x)
        A = np.zeros((n, n))
        for i, x in enumerate(xs):
            A[i, :deg + 1] = x ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * 2.0 ** x
        sol = np.linalg.solve(A, 2.0 ** xs)
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: extrema of the error between sign changes
        idx = []
        sgn = np.sign(err)
        start = 0
        for i in range(1, len(grid)):
            if sgn[i] != sgn[start]:
                seg = slice(start, i)
                idx.append(start + int(np.argmax(np.abs(err[seg]))))
                start = i
        idx.append(start + int(np.argmax(np.abs(err[start:]))))
        if len(idx) != n:
            break
        xs = grid[idx]
    return c, float(np.abs(err).max())


def f32_error(c):
    c32 = np.asarray(c, dtype=np.float32)
    f = np.linspace(LO, HI, 1000001, dtype=np.float32)
    p = np.full_like(f, c32[3])
    for k in (2, 1, 0):
        p = (p * f + c32[k]).astype(np.float32)
    return float(np.abs(p.astype(np.float64) / 2.0 ** f.astype(np.float64) - 1.0).max())


if __name__ == "__main__":
    c, e = remez()
    c32 = np.asarray(c, dtype=np.float32)
    print("minimax relative error (exact coefficients): %.3e" % e)
    print("float32 evaluation error:                    %.3e" % f32_error(c32))
    for k, v in enumerate(c32):
        print(f"c{k} = {float(v).hex()}  ({float(v):.9e})")
