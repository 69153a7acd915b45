"""Minimax (Remez exchange) fit of 2^f on [-1/2, 1/2] by a polynomial, on relative error.

Test helper: it regenerates the coefficients of the FMA-pipe exp2 in the kernels' PTX helper
header (a degree-3 polynomial after the range reduction x = n + f, n = rint(x)).

The exchange method: on a reference of deg + 2 points x_0 < ... < x_{deg+1}, solve the linear
system  p(x_i) - 2^{x_i} = (-1)^i E 2^{x_i}  for the deg + 1 coefficients and the levelled error
E (relative error equioscillates with alternating sign); then move every reference point to the
largest |p/2^f - 1| on its sign-alternating stretch of a dense grid, and repeat until the
reference stops moving.  Chebyshev extrema start it."""
import numpy as np


def remez_exp2_rel(deg: int = 3, a: float = -0.5, b: float = 0.5, iters: int = 30, grid_n: int = 200001):
    """Returns (coefficients c_0..c_deg in increasing power, levelled error |E|, max grid error)."""
    n = deg + 2
    x = (a + b) / 2 + (b - a) / 2 * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(a, b, grid_n)
    c, E, err = None, 0.0, None
    for _ in range(iters):
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * np.exp2(x[i])
        sol = np.linalg.solve(A, np.exp2(x))
        c, E = sol[:deg + 1], sol[deg + 1]
        err = np.polyval(c[::-1], grid) / np.exp2(grid) - 1.0
        sign = np.sign(err)
        ext, start = [], 0
        for k in range(1, grid_n + 1):
            if k == grid_n or sign[k] != sign[start]:
                seg = np.arange(start, k)
                ext.append(seg[np.argmax(np.abs(err[seg]))])
                start = k
        ext = np.array(ext)
        while len(ext) > n:                     # keep the n alternating extrema: drop the smaller end
            ext = ext[1:] if abs(err[ext[0]]) < abs(err[ext[-1]]) else ext[:-1]
        new_x = grid[ext]
        if len(new_x) == n and np.allclose(new_x, x, atol=0.0, rtol=0.0):
            break
        if len(new_x) == n:
            x = new_x
    return c, abs(E), float(np.max(np.abs(err)))
