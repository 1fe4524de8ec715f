"""Fit the polynomial the forward kernel uses for part of its exponentials.

2^x is split Cody-Waite style into x = n + f with n = round(x) and
f in [-1/2, 1/2]; then 2^x = 2^n * p(f), where p is the degree-4 polynomial
minimising the maximum relative error |p(f) / 2^f - 1| on [-1/2, 1/2],
found here with the Remez exchange algorithm (equioscillation of the weighted
error at n + 2 reference points).  The printed float32 coefficients are
pasted into attn_fwd.cu; tests/test_exp2_poly.py re-derives their error bound.

Usage: python gen_exp2_poly.py [degree]
"""

import sys

import numpy as np

LO, HI = -0.5, 0.5


def remez_relative(deg: int, iters: int = 50):
    """Coefficients c[0..deg] (ascending) minimising max |p(f)/2^f - 1|."""
    n = deg + 2
    # Chebyshev extrema as the initial reference.
    ref = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # Solve p(x_i) - 2^x_i = (-1)^i E 2^x_i for the coefficients and E.
        A = np.zeros((n, n))
        for i, x in enumerate(ref):
            A[i, :deg + 1] = x ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** x
        sol = np.linalg.solve(A, 2.0 ** ref)
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # New reference: the extremum of each run of constant error sign.
        sign = np.sign(err)
        edges = np.flatnonzero(np.diff(sign)) + 1
        runs = np.split(np.arange(grid.size), edges)
        ext = [r[np.argmax(np.abs(err[r]))] for r in runs]
        if len(ext) < n:
            break
        # keep the n alternating extrema with the largest errors
        while len(ext) > n:
            mags = np.abs(err[ext])
            drop = 0 if mags[0] < mags[-1] else len(ext) - 1
            ext.pop(drop)
        new_ref = grid[ext]
        if np.allclose(new_ref, ref, atol=1e-12):
            break
        ref = new_ref
    return c, float(np.max(np.abs(err)))


def main():
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 4
    c, e = remez_relative(deg)
    c32 = c.astype(np.float32)
    print(f"// degree {deg}, max relative error {e:.3e} (float64 coefficients)")
    for i, v in enumerate(c32):
        print(f"constexpr float EXP2_C{i} = {float(v)!r}f;  // {v.view(np.uint32):#010x}")


if __name__ == "__main__":
    main()
