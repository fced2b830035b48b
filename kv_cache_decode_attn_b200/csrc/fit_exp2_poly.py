"""Fit the polynomial the prefill kernel uses for 2^f on f in [-1/2, 1/2].

Minimax in RELATIVE error, by the Remez exchange algorithm (alternation
theorem for p(f) ~ 2^f with weight 1 / 2^f), in float64.  Prints the
coefficients c0..c3 of p(f) = c0 + f (c1 + f (c2 + f c3)) and the error bound
that the kernel comment and the CPU test quote.

Used by the software exp2 of the prefill softmax: 2^x = 2^n * 2^f with
n = round(x), f = x - n (Cody-Waite style reduction with the round-to-nearest
"magic number" 1.5 * 2^23), 2^f = p(f), and 2^n applied by adding n to the
exponent field.
"""

import numpy as np


def remez_relative(deg=3, lo=-0.5, hi=0.5, iters=30):
    f = lambda x: np.exp2(x)
    n = deg + 2
    # initial reference: Chebyshev extrema
    k = np.arange(n)
    xs = (lo + hi) / 2 + (hi - lo) / 2 * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # solve p(x_i) - f(x_i) = (-1)^i E f(x_i)  (relative equioscillation)
        A = np.zeros((n, n))
        for i, x in enumerate(xs):
            A[i, :deg + 1] = x ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(x)
        sol = np.linalg.solve(A, f(xs))
        c, E = sol[:deg + 1], sol[deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: extrema of the error between sign changes
        idx = [0]
        sign_changes = np.nonzero(np.diff(np.sign(err)))[0]
        bounds = [0] + list(sign_changes + 1) + [len(grid)]
        ext = []
        for a, b in zip(bounds[:-1], bounds[1:]):
            seg = np.abs(err[a:b])
            ext.append(a + int(np.argmax(seg)))
        if len(ext) >= n:
            # keep the n largest alternating extrema
            while len(ext) > n:
                vals = np.abs(err[ext])
                drop = 0 if vals[0] < vals[-1] else len(ext) - 1
                ext.pop(drop)
            xs = grid[ext]
    return c, float(np.abs(err).max())


if __name__ == "__main__":
    c, e = remez_relative()
    print("coefficients (c0..c3):", ", ".join(f"{v:.9e}" for v in c))
    print(f"max relative error on [-0.5, 0.5]: {e:.3e}")
