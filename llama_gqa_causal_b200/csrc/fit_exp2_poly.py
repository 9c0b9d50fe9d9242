"""Fit the quadratic used by the prefill kernel's FMA-pipe exp2.

exp2(x) is split as 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]
(Cody & Waite style range reduction); 2^f is replaced by a polynomial p(f)
whose coefficients minimise the maximum relative error on [-1/2, 1/2] (Remez
exchange on the relative error, starting from Chebyshev nodes).  The kernel
rounds p(f) to bf16 afterwards (relative step up to 2^-8 = 3.9e-3) for the
P V product and sums the same p(f) into the row's denominator, so the
quadratic's 1.7e-3 stays below what the probabilities keep and largely
cancels between numerator and denominator; a cubic (7.5e-5) costs one more
packed FMA per pair of exponentials.

    python -m llama_gqa_causal_b200.csrc.fit_exp2_poly
prints the coefficients (c0..c2) and the achieved maximum relative error.
"""
import numpy as np


def remez_rel(deg=2, lo=-0.5, hi=0.5, iters=30):
    f = lambda x: np.exp2(x)
    k = np.arange(deg + 2)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * k[::-1] / (deg + 1))
    for _ in range(iters):
        # solve p(x_i) - f(x_i) = (-1)^i E f(x_i)  (relative equioscillation)
        A = np.zeros((deg + 2, deg + 2))
        for i, xi in enumerate(x):
            A[i, :deg + 1] = xi ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(xi)
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        grid = np.linspace(lo, hi, 200001)
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: extrema of err between sign changes
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        ext = grid[idx]
        ev = err[idx]
        # keep alternating extrema of largest magnitude
        sel = []
        for xi, e in zip(ext, ev):
            if sel and np.sign(e) == np.sign(sel[-1][1]):
                if abs(e) > abs(sel[-1][1]):
                    sel[-1] = (xi, e)
            else:
                sel.append((xi, e))
        if len(sel) >= deg + 2:
            sel = sorted(sel, key=lambda t: -abs(t[1]))[:deg + 2]
            x = np.sort(np.array([t[0] for t in sel]))
    grid = np.linspace(lo, hi, 400001)
    err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
    return c, float(np.abs(err).max())


if __name__ == "__main__":
    c, e = remez_rel()
    c32 = np.float32(c)
    print(f"coefficients c0..c{len(c32) - 1} (float32):", ", ".join(repr(float(v)) for v in c32))
    print("max relative error on [-1/2, 1/2]:", e)
