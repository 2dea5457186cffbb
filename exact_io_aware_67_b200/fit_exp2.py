"""Derivation of the polynomial the kernels use for part of their base-2
exponentials (computed on the FMA pipe instead of the MUFU unit).

2^x is split as 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]; 2^f
is approximated by a cubic p(f) = c0 + f (c1 + f (c2 + f c3)) whose
coefficients minimise the maximum RELATIVE error on [-1/2, 1/2] (a Remez
exchange on the equioscillation conditions, written here from the
definition; no library fit).  c0 is left free.

    python -m exact_io_aware_67_b200.fit_exp2

prints the coefficients as fp32 hex literals and the achieved bound.
"""
import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def remez(degree=DEGREE, iters=30):
    n = degree + 2                      # reference points for degree+1 coeffs + error
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * (n - 1 - k) / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # solve sum_j c_j x_i^j / 2^x_i + (-1)^i E = 1   (relative error form)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :degree + 1] = x[i] ** np.arange(degree + 1) / 2.0 ** x[i]
            A[i, degree + 1] = (-1) ** i
        sol = np.linalg.solve(A, np.ones(n))
        c = sol[:degree + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: extrema of the error between sign changes
        idx = [0]
        for j in range(1, len(grid) - 1):
            if (err[j] - err[j - 1]) * (err[j + 1] - err[j]) <= 0:
                idx.append(j)
        idx.append(len(grid) - 1)
        idx = sorted(set(idx), key=lambda j: -abs(err[j]))[:n]
        x = np.sort(grid[idx])
    return c, float(np.max(np.abs(err)))


def main():
    c, e = remez()
    c32 = c.astype(np.float32)
    for i, v in enumerate(c32):
        print("c%d = %.9e  (0x%08x)" % (i, v, np.float32(v).view(np.uint32)))
    print("max relative error on [-1/2, 1/2]: %.3e" % e)


if __name__ == "__main__":
    main()
