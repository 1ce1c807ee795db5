"""Coefficients of the FMA-pipe exp2 used by the forward softmax.

    python exact_io_aware_77_b200/csrc/gen_exp2_poly.py [degree]

Method (Cody and Waite's argument reduction followed by a minimax polynomial):
2^x = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]; 2^f is replaced by the
polynomial p(f) of the given degree that minimises the maximum RELATIVE error
|p(f) / 2^f - 1| on [-1/2, 1/2], found with the Remez exchange algorithm; 2^n is applied by
adding n to the exponent field of p(f).  Prints the coefficients (lowest degree first) and
the achieved maximum relative error.
"""

import sys

import numpy as np


def remez_relative(degree: int, lo: float = -0.5, hi: float = 0.5, iters: int = 40):
    f = lambda x: np.exp2(x)
    n = degree + 2
    # Chebyshev extrema as the starting reference
    k = np.arange(n)
    ref = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * k[::-1] / (n - 1))
    dense = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # solve p(x_i) - f(x_i) = (-1)^i E f(x_i)  for the coefficients and E
        A = np.zeros((n, n))
        for i, x in enumerate(ref):
            A[i, :degree + 1] = x ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1) ** i) * f(x)
        sol = np.linalg.solve(A, f(ref))
        coef, E = sol[:degree + 1], sol[degree + 1]
        err = np.polyval(coef[::-1], dense) / f(dense) - 1.0
        # new reference: one extremum of the error in each sign-alternating segment
        sign_change = np.where(np.diff(np.sign(err)) != 0)[0]
        bounds = np.concatenate([[0], sign_change + 1, [dense.size]])
        new_ref = []
        for a, b in zip(bounds[:-1], bounds[1:]):
            seg = np.abs(err[a:b])
            new_ref.append(dense[a + int(np.argmax(seg))])
        if len(new_ref) != n:
            break
        ref = np.array(new_ref)
    return coef, float(np.max(np.abs(err)))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    coef, max_rel = remez_relative(deg)
    for i, c in enumerate(coef):
        print(f"c{i} = {np.float32(c)!r}  # {c:.17g}")
    # the error of the float32-rounded coefficients
    x = np.linspace(-0.5, 0.5, 400001)
    c32 = np.array(coef, dtype=np.float32).astype(np.float64)
    print("max relative error (exact coefficients):", max_rel)
    print("max relative error (float32 coefficients):", float(np.max(np.abs(np.polyval(c32[::-1], x) / np.exp2(x) - 1))))
