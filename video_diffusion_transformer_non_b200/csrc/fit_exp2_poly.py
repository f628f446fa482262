"""Fits the polynomial used for 2^f, f in [-1/2, 1/2], on the FMA pipe.

Method (Cody & Waite style range reduction, as used for exponentials since
Cody and Waite's "Software Manual for the Elementary Functions", 1980): write
x = j + f with j = round(x) and |f| <= 1/2, so 2^x = 2^j * 2^f; 2^j is added
straight into the exponent field and 2^f comes from a cubic p(f).  The cubic
here minimises the maximum relative error |p(f)/2^f - 1| on [-1/2, 1/2]
(a Remez exchange on the relative error), computed in float64, then rounded
to float32.  Prints the coefficients and the error of the float32 cubic.

    python fit_exp2_poly.py
"""
import numpy as np


def remez_relative(deg=3, iters=30):
    a, b = -0.5, 0.5
    n = deg + 2
    # Chebyshev-like initial reference points
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(a, b, 200001)
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E 2^x_i  for coefficients and E
        A = np.zeros((n, n))
        for i, xi in enumerate(x):
            A[i, :deg + 1] = xi ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** xi
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: extrema of err, one per sign change interval
        idx = [0]
        for k in range(1, grid.size - 1):
            if (err[k] - err[k - 1]) * (err[k + 1] - err[k]) <= 0:
                idx.append(k)
        idx.append(grid.size - 1)
        idx = np.array(sorted(set(idx)))
        cand = grid[idx]
        vals = err[idx]
        # keep alternating-sign extrema with the largest magnitudes
        sel = []
        for xv, ev in zip(cand, vals):
            if sel and np.sign(ev) == np.sign(sel[-1][1]):
                if abs(ev) > abs(sel[-1][1]):
                    sel[-1] = (xv, ev)
            else:
                sel.append((xv, ev))
        while len(sel) > n:
            # drop the smaller end
            if abs(sel[0][1]) < abs(sel[-1][1]):
                sel.pop(0)
            else:
                sel.pop()
        if len(sel) == n:
            x = np.array([s[0] for s in sel])
    return c, np.max(np.abs(err))


def main():
    c, e = remez_relative()
    c32 = c.astype(np.float32)
    f = np.linspace(-0.5, 0.5, 1000001).astype(np.float32)
    p = ((c32[3] * f + c32[2]) * f + c32[1]) * f + c32[0]   # float32 Horner
    rel = np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1)
    print("coefficients c0..c3 (float32):")
    for i, v in enumerate(c32):
        print(f"  c{i} = {float(v)!r:>24}  ({v.view(np.uint32):#010x})")
    print(f"max relative error: minimax {e:.3e}, float32 Horner {rel.max():.3e}")


if __name__ == "__main__":
    main()
