"""Fit the polynomial used for 2^f, f in [-1/2, 1/2], in the softmax kernel.

Method: minimax approximation of the relative error by the Remez exchange
algorithm (Remez, 1934) on the function 2^f over [-1/2, 1/2], in float64,
then rounding the coefficients to float32 and measuring the error of the
float32 Horner evaluation.  Together with the split x = n + f (n the nearest
integer, computed exactly with the 1.5 * 2^23 rounding constant) and an
exponent-field add this gives 2^x on the FMA pipe (Cody and Waite's argument
reduction).  Run:  python fit_exp2_poly.py [degree]
"""
import sys

import numpy as np


def remez(deg, lo=-0.5, hi=0.5, iters=30):
    f = lambda x: np.exp2(x)
    n = deg + 2
    # initial reference: Chebyshev extrema
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    for _ in range(iters):
        # solve p(x_i) - f(x_i) = (-1)^i E f(x_i)  (relative error equioscillation)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(x[i])
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        g = np.linspace(lo, hi, 200001)
        err = np.polyval(c[::-1], g) / f(g) - 1
        # new reference: extrema of err between sign changes
        idx = [0]
        s = np.sign(err)
        cuts = np.nonzero(np.diff(s))[0]
        bounds = [0] + list(cuts + 1) + [len(g)]
        ext = [b0 + np.argmax(np.abs(err[b0:b1])) for b0, b1 in zip(bounds[:-1], bounds[1:])]
        if len(ext) >= n:
            # keep the n largest consecutive alternating extrema
            while len(ext) > n:
                if abs(err[ext[0]]) < abs(err[ext[-1]]):
                    ext = ext[1:]
                else:
                    ext = ext[:-1]
            x = g[ext]
        del idx
    return c, np.max(np.abs(err))


def eval_f32(c32, f):
    f = f.astype(np.float32)
    p = np.float32(c32[-1])
    for ci in c32[-2::-1]:
        p = (p * f + np.float32(ci)).astype(np.float32)
    return p


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 4
    c, e = remez(deg)
    c32 = c.astype(np.float32)
    g = np.linspace(-0.5, 0.5, 2000001)
    e32 = np.max(np.abs(eval_f32(c32, g).astype(np.float64) / np.exp2(g) - 1))
    print(f"degree {deg}: minimax rel err {e:.3e}, float32 coefficients {e32:.3e}")
    for i, ci in enumerate(c32):
        print(f"  c{i} = {float(ci):.9e}f  (0x{np.float32(ci).view(np.uint32):08x})")
