"""Coefficients of the FMA-pipe exp2 used by the attention softmax (attn_fwd_tc.cu).

exp2(x) = 2^n * 2^f with n = round(x), f = x - n in [-1/2, 1/2] (range reduction by
the round-to-nearest "magic number" 1.5 * 2^23, in the spirit of Cody and Waite), and
2^f approximated by the degree-3 polynomial that minimises the maximum RELATIVE error
on [-1/2, 1/2], found with the Remez exchange algorithm.  Run this file to print the
coefficients and the error bound; the kernel hard-codes the printed values.

The softmax rounds every P to bf16 (relative step 2^-8), so a relative error near
1e-4 is far below the rounding that follows.
"""
import numpy as np


def remez_relative(deg=3, lo=-0.5, hi=0.5, iters=30):
    f = lambda x: np.exp2(x)
    # initial reference: Chebyshev extrema
    k = np.arange(deg + 2)
    ref = (lo + hi) / 2 + (hi - lo) / 2 * np.cos(np.pi * k / (deg + 1))[::-1]
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # solve p(x_i) - f(x_i) = (-1)^i E f(x_i)  (relative equioscillation)
        A = np.zeros((deg + 2, deg + 2))
        for i, x in enumerate(ref):
            A[i, :deg + 1] = x ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(x)
        sol = np.linalg.solve(A, f(ref))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: extrema of the error between sign changes
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        cand = np.array(idx)
        # keep deg+2 alternating extrema with the largest magnitudes
        pts = [cand[0]]
        for i in cand[1:]:
            if np.sign(err[i]) == np.sign(err[pts[-1]]):
                if abs(err[i]) > abs(err[pts[-1]]):
                    pts[-1] = i
            else:
                pts.append(i)
        while len(pts) > deg + 2:
            if abs(err[pts[0]]) < abs(err[pts[-1]]):
                pts.pop(0)
            else:
                pts.pop()
        if len(pts) == deg + 2:
            ref = grid[pts]
    return c, float(np.abs(err).max())


if __name__ == "__main__":
    c, e = remez_relative()
    c32 = c.astype(np.float32)
    for i, v in enumerate(c32):
        print(f"C{i} = {float(v):.9e}f  ({v.view(np.uint32):#010x})")
    print(f"max relative error on [-1/2, 1/2]: {e:.3e}")
