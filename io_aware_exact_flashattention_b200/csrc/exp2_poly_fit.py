"""Derive the polynomial used for part of the kernel's 2^x evaluations.

2^x = 2^n * 2^f with n = round(x) (Cody-Waite range reduction) and
f = x - n in [-1/2, 1/2]; 2^f is approximated by a degree-3 polynomial fitted
by a Remez exchange for minimal maximum relative error on [-1/2, 1/2].  The
coefficients are printed as the C++ constants used in prefill_sm100.cuh, and
the tests re-run this fit and check both the constants and the error bound.

    python io_aware_exact_flashattention_b200/csrc/exp2_poly_fit.py
"""
import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def remez_relative(degree=DEGREE, lo=LO, hi=HI, iters=30):
    """Minimax fit p(f) ~ 2^f minimising max |p(f)/2^f - 1| on [lo, hi]."""
    n = degree + 2
    # Chebyshev extrema as the initial reference
    k = np.arange(n)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i * E * 2^x_i for coefficients and E
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :degree + 1] = x[i] ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:degree + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: extrema of the error between sign changes
        sgn = np.sign(err)
        idx = np.concatenate(([0], np.nonzero(np.diff(sgn))[0] + 1, [len(grid)]))
        ext = [s + np.argmax(np.abs(err[s:e])) for s, e in zip(idx[:-1], idx[1:]) if e > s]
        if len(ext) < n:
            break
        # keep the n extrema with the largest errors, in order
        ext = sorted(sorted(ext, key=lambda j: -abs(err[j]))[:n])
        x = grid[ext]
    err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
    return c, float(np.abs(err).max())


def coefficients_fp32():
    c, e = remez_relative()
    return [float(np.float32(v)) for v in c], e


if __name__ == "__main__":
    c32, e = coefficients_fp32()
    print("// degree-%d minimax fit of 2^f on [%g, %g], max relative error %.3e" % (DEGREE, LO, HI, e))
    for i, v in enumerate(c32):
        print("constexpr float kExp2C%d = %.9ef;" % (i, v))
