"""Fit the polynomial of the FMA-pipe base-2 exponential used by the prefill
softmax, and write it into ``exp2_poly.h``.

Method: range reduction x = n + f with n = round-to-nearest(x), so that
f lies in [-1/2, 1/2] (the classic Cody-Waite split of the argument; for
base 2 the split is exact), then 2^x = 2^n * p(f) where p is the degree-3
polynomial minimising the maximum RELATIVE error |p(f) - 2^f| / 2^f on
[-1/2, 1/2], found with the Remez exchange algorithm (equioscillation at
degree + 2 points).  The coefficients are rounded to fp32 and the error of
the fp32 Horner evaluation is reported.

    python paged_kv_cache_408_b200/csrc/exp2_poly_fit.py        # rewrite exp2_poly.h
    python paged_kv_cache_408_b200/csrc/exp2_poly_fit.py --check  # compare with it

Only numpy is needed; nothing here is used at run time.
"""
import os
import sys

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5
HERE = os.path.dirname(os.path.abspath(__file__))
HEADER = os.path.join(HERE, "exp2_poly.h")


def remez(degree=DEGREE, lo=LO, hi=HI, iters=40):
    """Minimax relative-error polynomial for 2^f on [lo, hi]: coefficients
    c0..c_degree (ascending) and the levelled error."""
    n = degree + 2
    # start from Chebyshev extrema
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i  -> unknowns c_0..c_d, E
        A = np.zeros((n, n))
        for j in range(degree + 1):
            A[:, j] = x ** j
        A[:, -1] = -((-1.0) ** np.arange(n)) * np.exp2(x)
        sol = np.linalg.solve(A, np.exp2(x))
        c, E = sol[:-1], sol[-1]
        err = (np.polyval(c[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
        # new reference: one extremum of the error per sign-alternating run
        idx = []
        sgn = np.sign(err)
        start = 0
        for k in range(1, len(grid) + 1):
            if k == len(grid) or sgn[k] != sgn[start]:
                seg = slice(start, k)
                idx.append(start + int(np.argmax(np.abs(err[seg]))))
                start = k
        if len(idx) < n:
            break
        # keep n consecutive alternating extrema with the largest error
        best = max(range(len(idx) - n + 1), key=lambda s: np.abs(err[idx[s:s + n]]).min())
        xn = grid[idx[best:best + n]]
        if np.allclose(xn, x, atol=1e-12):
            break
        x = xn
    return c, abs(E)


def fp32_eval_error(c32):
    """Max relative error of the fp32 Horner evaluation (each step one fused
    multiply-add rounded to fp32, emulated exactly in fp64) over a dense
    fp32 grid of [-1/2, 1/2]."""
    f = np.linspace(LO, HI, 1_000_001).astype(np.float32).astype(np.float64)
    acc = np.full_like(f, np.float64(c32[-1]))
    for cj in c32[-2::-1]:
        acc = (acc * f + np.float64(cj)).astype(np.float32).astype(np.float64)
    return float(np.max(np.abs(acc - np.exp2(f)) / np.exp2(f)))


def header_text(c32, E, E32):
    lines = ["// exp2_poly.h -- written by exp2_poly_fit.py (do not edit): the degree-%d" % DEGREE,
             "// polynomial p(f) ~ 2^f on [-1/2, 1/2] with minimax relative error (Remez",
             "// exchange), coefficients rounded to fp32.  Levelled relative error of the",
             "// exact polynomial %.3e; of the fp32 Horner evaluation %.3e." % (E, E32),
             "#pragma once", "", "namespace pa {", ""]
    for j, cj in enumerate(c32):
        lines.append("constexpr float kExp2Poly%d = %sf;  // %s" % (j, repr(float(cj)), float(cj).hex()))
    lines += ["", "}  // namespace pa", ""]
    return "\n".join(lines)


def fit():
    c, E = remez()
    c32 = c.astype(np.float32)
    return c32, E, fp32_eval_error(c32)


if __name__ == "__main__":
    c32, E, E32 = fit()
    text = header_text(c32, E, E32)
    if "--check" in sys.argv:
        same = os.path.exists(HEADER) and open(HEADER).read() == text
        print("exp2_poly.h is current" if same else "exp2_poly.h differs from the fit")
        sys.exit(0 if same else 1)
    open(HEADER, "w").write(text)
    print(text)
