"""Coefficients of the polynomial exp2 used on the FMA pipe (fastexp.cuh).

Method: Cody-Waite style range reduction x = n + f, n = round(x), f in
[-1/2, 1/2], so 2^x = 2^n * 2^f; 2^f is replaced by the degree-3 polynomial
that minimises the maximum *relative* error on [-1/2, 1/2], found with the
Remez exchange algorithm (equioscillation of the weighted error at deg + 2
points).  Run this file to regenerate the constants:

    python head_partitioned_distance_b200/csrc/exp2_poly.py
"""
import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def remez(deg=DEG, lo=LO, hi=HI, iters=60):
    f = lambda x: np.exp2(x)
    # start from Chebyshev extrema
    k = np.arange(deg + 2)
    x = (lo + hi) / 2 + (hi - lo) / 2 * np.cos(np.pi * k[::-1] / (deg + 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # solve p(x_i) + (-1)^i E f(x_i) = f(x_i)  (relative error weight 1/f)
        A = np.zeros((deg + 2, deg + 2))
        for i, xi in enumerate(x):
            A[i, :deg + 1] = xi ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * f(xi)
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: extrema of the error between sign changes
        sign = np.sign(err)
        idx = np.nonzero(np.diff(sign))[0]
        bounds = np.concatenate(([0], idx + 1, [len(grid)]))
        ext = [b0 + np.argmax(np.abs(err[b0:b1])) for b0, b1 in zip(bounds[:-1], bounds[1:]) if b1 > b0]
        if len(ext) < deg + 2:
            break
        # keep the deg + 2 largest alternating extrema
        while len(ext) > deg + 2:
            vals = np.abs(err[ext])
            drop = 0 if vals[0] < vals[-1] else len(ext) - 1
            ext.pop(drop)
        x = grid[ext]
    err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
    return c, float(np.abs(err).max())


if __name__ == "__main__":
    c, e = remez()
    print(f"// degree-{DEG} minimax (relative) for 2^f on [{LO}, {HI}]; max rel error {e:.3e}")
    for i, ci in enumerate(c):
        print(f"constexpr float kExp2C{i} = {float(np.float32(ci)):.9g}f;")
