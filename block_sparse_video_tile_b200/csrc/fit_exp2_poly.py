"""Fit the polynomial of the FMA-pipe 2^x used by the attend kernel's softmax.

    python block_sparse_video_tile_b200/csrc/fit_exp2_poly.py

Method (Cody-Waite range reduction + near-minimax polynomial): write
x = j + f with j = round(x) (an integer, applied exactly through the float
exponent field) and f in [-1/2, 1/2], so 2^x = 2^j * 2^f.  2^f is approximated
on [-1/2, 1/2] by the polynomial that interpolates it at the Chebyshev nodes
of the interval (close to the minimax polynomial), refined by a few Remez
exchange steps on the relative error.  The output is the coefficient list
(lowest order first) pasted into attn_kernel.cuh, and the achieved maximum
relative error, which the kernel's tests bound.
"""
import numpy as np


def remez_relative(deg, iters=30):
    """Minimax (relative error) polynomial for 2^f on [-1/2, 1/2]."""
    n = deg + 2
    # initial reference: Chebyshev extrema
    x = 0.5 * np.cos(np.pi * np.arange(n) / (n - 1))[::-1]
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E 2^x_i   (relative equioscillation)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:deg + 1]
        grid = np.linspace(-0.5, 0.5, 200001)
        err = (np.polyval(c[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new reference: extrema of the error on each sign run
        sgn = np.sign(err)
        idx = np.flatnonzero(np.diff(sgn) != 0)
        bounds = np.concatenate([[0], idx + 1, [grid.size]])
        ext = [b0 + np.argmax(np.abs(err[b0:b1])) for b0, b1 in zip(bounds[:-1], bounds[1:])]
        if len(ext) < n:
            break
        # keep n alternating extrema with the largest errors
        while len(ext) > n:
            if abs(err[ext[0]]) < abs(err[ext[-1]]):
                ext.pop(0)
            else:
                ext.pop()
        x = grid[ext]
    return c, float(np.max(np.abs(err)))


if __name__ == "__main__":
    for deg in (3, 4, 5):
        c, e = remez_relative(deg)
        c32 = c.astype(np.float32)
        grid = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
        p = np.zeros_like(grid)
        for a in c32[::-1]:                        # Horner in float32, as the kernel does
            p = p * grid + a
        e32 = float(np.max(np.abs(p.astype(np.float64) - 2.0 ** grid.astype(np.float64))
                           / 2.0 ** grid.astype(np.float64)))
        print(f"degree {deg}: max rel error {e:.3e} (float64), {e32:.3e} (float32 Horner)")
        print("  coefficients:", ", ".join(f"{v:.9e}f" for v in c32))
