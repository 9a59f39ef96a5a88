"""Derive the polynomial the attention kernel uses to evaluate part of its exp2 calls on the FMA pipe.

    python docs/exp2_poly.py

exp2(x) = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2] (Cody & Waite style
reduction; the kernel rounds with the 1.5 * 2^23 addition trick and adds n to the exponent
field).  2^f is approximated by the degree-3 polynomial minimising the maximum RELATIVE error
on [-1/2, 1/2], found with the Remez exchange algorithm (equioscillation at degree + 2 points),
then rounded to fp32.  The script prints the coefficients and the error bound of the fp32
Horner evaluation, which the kernel's probabilities (rounded to bf16, relative step 2^-8)
absorb: the bound is ~1e-4.
"""

import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def remez_relative(deg=DEG, iters=30):
    f = lambda x: np.exp2(x)
    # start from Chebyshev extrema
    k = np.arange(deg + 2)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k[::-1] / (deg + 1))
    dense = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # solve p(x_i) - f(x_i) = (-1)^i E f(x_i)  for the coefficients and E
        A = np.zeros((deg + 2, deg + 2))
        for i, xi in enumerate(x):
            A[i, :deg + 1] = xi ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(xi)
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], dense) - f(dense)) / f(dense)
        # new reference: extrema of the error between sign changes
        idx = [0]
        for j in range(1, len(dense) - 1):
            if (err[j] - err[j - 1]) * (err[j + 1] - err[j]) <= 0:
                idx.append(j)
        idx.append(len(dense) - 1)
        cand = dense[idx]
        ev = err[idx]
        # keep deg+2 alternating extrema of largest magnitude
        pts = []
        for xi, e in zip(cand, ev):
            if pts and np.sign(e) == np.sign(pts[-1][1]):
                if abs(e) > abs(pts[-1][1]):
                    pts[-1] = (xi, e)
            else:
                pts.append((xi, e))
        while len(pts) > deg + 2:
            if abs(pts[0][1]) < abs(pts[-1][1]):
                pts.pop(0)
            else:
                pts.pop()
        x = np.array([p[0] for p in pts])
    return c, np.abs(err).max()


def fp32_horner_error(c32):
    xs = np.linspace(LO, HI, 400001).astype(np.float32)
    p = np.float32(c32[3])
    for ci in (c32[2], c32[1], c32[0]):
        p = (p * xs + np.float32(ci)).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(xs.astype(np.float64)) - 1)))


if __name__ == "__main__":
    c, e = remez_relative()
    c32 = [np.float32(v) for v in c]
    print("minimax relative error (real coefficients): %.3e" % e)
    print("fp32 Horner relative error: %.3e" % fp32_horner_error(c32))
    for i, v in enumerate(c32):
        print("c%d = %.9ef  (bits 0x%08x)" % (i, v, np.array(v).view(np.uint32)))
