"""Coefficients of the polynomial 2^f ~ c0 + c1 f + c2 f^2 + c3 f^3 on f in [-1/2, 1/2] that the
prefill kernel uses for part of its exponentials (csrc/fwd_tc.cuh, ex2_poly2).

The kernel splits x = n + f with n = rint(x) (Cody and Waite's range reduction, "Software Manual
for the Elementary Functions", 1980) and adds n into the exponent field of 2^f.  The polynomial
is the minimax approximation in relative error, found here by the Remez exchange algorithm, then
rounded to fp32; `python exp2_poly.py` prints the coefficients and the error of the rounded
polynomial evaluated in fp32 by Horner's rule, as the kernel evaluates it.
"""
import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def remez(deg=DEGREE, lo=LO, hi=HI, iters=40):
    n = deg + 2  # deg + 1 coefficients and the levelled error
    xs = (lo + hi) / 2 - (hi - lo) / 2 * np.cos(np.pi * np.arange(n) / (n - 1))
    grid = np.linspace(lo, hi, 400001)
    for _ in range(iters):
        a = np.zeros((n, n))
        for i, x in enumerate(xs):
            a[i, :deg + 1] = x ** np.arange(deg + 1)
            a[i, deg + 1] = (-1) ** i * 2.0 ** x  # relative error: E * 2^x
        sol = np.linalg.solve(a, 2.0 ** xs)
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        ext = [0]  # one extremum per run of equal sign
        for k in range(1, grid.size):
            if np.sign(err[k]) != np.sign(err[ext[-1]]):
                ext.append(k)
            elif abs(err[k]) > abs(err[ext[-1]]):
                ext[-1] = k
        if len(ext) >= n:
            xs = grid[np.array(ext[:n])]
    return c


def fp32_horner_error(c32, lo=LO, hi=HI):
    f = np.linspace(lo, hi, 400001).astype(np.float32)
    p = np.full_like(f, c32[-1])
    for ck in c32[-2::-1]:
        p = (p * f + np.float32(ck)).astype(np.float32)
    exact = 2.0 ** f.astype(np.float64)
    return float(np.max(np.abs((p.astype(np.float64) - exact) / exact)))


if __name__ == "__main__":
    c32 = remez().astype(np.float32)
    for k, ck in enumerate(c32):
        print(f"c{k} = {float(ck):.9e}f")
    print(f"max relative error (fp32 Horner) = {fp32_horner_error(c32):.3e}")
