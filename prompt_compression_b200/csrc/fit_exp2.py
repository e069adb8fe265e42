"""Fit the polynomial used by the FMA-pipe exp2 in the scoring epilogue.

2^x = 2^j * 2^f with j = round(x) and f = x - j in [-1/2, 1/2].  2^f is
approximated by a degree-4 polynomial p whose coefficients minimise the
maximum RELATIVE error max |p(f) / 2^f - 1| on [-1/2, 1/2]; they are found
with the Remez exchange algorithm (equioscillation of the weighted error at
n + 2 reference points), written here from its textbook statement.

    python prompt_compression_b200/csrc/fit_exp2.py      # prints the coefficients

The printed values are pasted into exp2_poly.cuh; the GPU test of the
polynomial compares the kernel's results against ex2.approx and exp2f.
"""
import numpy as np

DEG = 4
A, B = -0.5, 0.5


def remez(deg=DEG, iters=30):
    n = deg
    k = np.arange(n + 2)
    x = 0.5 * (A + B) + 0.5 * (B - A) * np.cos(np.pi * (n + 1 - k) / (n + 1))   # Chebyshev extrema
    grid = np.linspace(A, B, 200001)
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i  ->  unknowns c_0..c_n, E
        M = np.zeros((n + 2, n + 2))
        for i, xi in enumerate(x):
            M[i, :n + 1] = xi ** np.arange(n + 1)
            M[i, n + 1] = -((-1) ** i) * 2.0 ** xi
        sol = np.linalg.solve(M, 2.0 ** x)
        c, E = sol[:n + 1], sol[n + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: one extremum per sign-alternating run of the error
        sign = np.sign(err)
        sign[sign == 0] = 1
        runs = np.split(np.arange(grid.size), np.flatnonzero(np.diff(sign)) + 1)
        ext = [r[np.argmax(np.abs(err[r]))] for r in runs]
        if len(ext) < n + 2:
            break
        while len(ext) > n + 2:       # drop the smallest end extremum
            if abs(err[ext[0]]) < abs(err[ext[-1]]):
                ext = ext[1:]
            else:
                ext = ext[:-1]
        x = grid[np.array(ext)]
    err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
    return c, float(np.abs(err).max()), float(abs(E))


def fp32_eval_error(c):
    """Max relative error when p is evaluated in fp32 Horner form with FMA."""
    f = np.linspace(A, B, 100001).astype(np.float32)
    cf = c.astype(np.float32)
    p = np.full_like(f, cf[-1])
    for ci in cf[-2::-1]:
        p = (p.astype(np.float64) * f + ci).astype(np.float32)   # one rounding per step, like FMA
    return float(np.abs(p.astype(np.float64) / 2.0 ** f.astype(np.float64) - 1.0).max())


if __name__ == "__main__":
    c, e, E = remez()
    print(f"degree {DEG} on [{A}, {B}]: max relative error {e:.3e} (levelled {E:.3e}); "
          f"fp32 Horner {fp32_eval_error(c):.3e}")
    for i, ci in enumerate(c.astype(np.float32)):
        print(f"  c{i} = {float(ci):.9e}f  (0x{np.float32(ci).view(np.uint32):08x})")
