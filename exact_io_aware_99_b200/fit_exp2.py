"""Fit the polynomial behind the kernels' FMA-pipe exp2.

The forward and backward kernels evaluate part of their exponentials on the
FMA pipe instead of the special-function unit.  Method (Cody-Waite style
range reduction, then a polynomial on the reduced range):

    2^x = 2^n * 2^f,  n = round(x),  f = x - n in [-1/2, 1/2]
    2^f ~= c0 + c1 f + c2 f^2 + c3 f^3

and 2^n is applied by adding n to the exponent field of the polynomial's
result.  The coefficients are the minimax fit of 2^f in *relative* error on
[-1/2, 1/2], computed here with the Remez exchange algorithm on a dense grid,
then rounded to float32.  Run

    python -m exact_io_aware_99_b200.fit_exp2

to print them; ``sm100.cuh`` holds the printed values and a CPU test checks
they agree.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def remez_relative(degree: int = DEGREE, iters: int = 30, grid: int = 200001):
    """Minimax polynomial p of the given degree for g(f) = 2^f on [LO, HI]
    minimising max |p(f)/g(f) - 1|.  Returns (coefficients low->high,
    max relative error)."""
    xs = np.linspace(LO, HI, grid)
    g = np.exp2(xs)
    n = degree + 2
    # initial reference: Chebyshev extrema
    k = np.arange(n)
    ref = 0.5 * (LO + HI) + 0.5 * (HI - LO) * -np.cos(np.pi * k / (n - 1))
    coef = None
    for _ in range(iters):
        # solve p(x_i) - g(x_i) = (-1)^i E g(x_i) for coefficients and E
        A = np.zeros((n, n))
        for i, x in enumerate(ref):
            A[i, :degree + 1] = x ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1) ** i) * np.exp2(x)
        sol = np.linalg.solve(A, np.exp2(ref))
        coef = sol[:degree + 1]
        err = np.polynomial.polynomial.polyval(xs, coef) / g - 1.0
        # new reference: extrema of the error, one per sign run
        sign = np.sign(err)
        sign[sign == 0] = 1
        runs = np.flatnonzero(np.diff(sign)) + 1
        bounds = np.concatenate([[0], runs, [grid]])
        cand = [b0 + int(np.argmax(np.abs(err[b0:b1]))) for b0, b1 in zip(bounds[:-1], bounds[1:])]
        if len(cand) < n:
            break
        # keep the n largest alternating extrema
        while len(cand) > n:
            vals = np.abs(err[cand])
            drop = 0 if vals[0] < vals[-1] else len(cand) - 1
            cand.pop(drop)
        ref = xs[cand]
    err = np.polynomial.polynomial.polyval(xs, coef) / g - 1.0
    return coef, float(np.max(np.abs(err)))


def coefficients_f32():
    coef, _ = remez_relative()
    return [float(np.float32(c)) for c in coef]


def emulate_f32(x: np.ndarray, coef=None) -> np.ndarray:
    """The kernels' steps in float32 arithmetic (for host-side checks):
    clamp to -126, round via the 1.5*2^23 shifter, reduce, Horner, add n to
    the exponent field."""
    c = [np.float32(v) for v in (coef or coefficients_f32())]
    x = np.maximum(np.asarray(x, np.float32), np.float32(-126.0))
    big = np.float32(12582912.0)  # 1.5 * 2^23
    t = (x + big).astype(np.float32)
    nf = (t - big).astype(np.float32)
    f = (x - nf).astype(np.float32)
    p = c[3]
    for ci in (c[2], c[1], c[0]):
        p = (p * f + ci).astype(np.float32)      # fma rounding differs by <= 1 ulp
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


def main():
    coef, err = remez_relative()
    print(f"degree {DEGREE} minimax relative error on [{LO}, {HI}]: {err:.3e}")
    for i, c in enumerate(coefficients_f32()):
        print(f"c{i} = {c!r}  ({np.float32(c).view(np.uint32):#010x})")


if __name__ == "__main__":
    main()
