"""Fit the polynomial used for the FMA-pipe exp2 in the attention kernel and write exp2_poly.cuh.

    python io_aware_exact_24_b200/csrc/exp2_poly_fit.py

Method (textbook, no library code involved):

* Cody & Waite style range reduction: x = n + r with n = round-to-nearest(x)
  and r in [-1/2, 1/2], so 2^x = 2^n * 2^r; 2^n is formed by adding n to the
  exponent field.
* 2^r on [-1/2, 1/2] is approximated by the degree-3 polynomial that minimises
  the maximum *relative* error, found with the Remez exchange algorithm
  (E. Ya. Remez, 1934): solve for coefficients that make the weighted error
  equioscillate on 5 reference points, move the points to the extrema of the
  new error curve, repeat until the levelled error stops changing.

The kernel rounds every probability to bf16 (8 significant bits, relative
spacing 2^-8), so a relative error near 1e-4 is far below what survives.
"""
from __future__ import annotations

import os

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def remez_relative(degree: int = DEGREE, iters: int = 40):
    f = lambda r: np.exp2(r)
    n = degree + 2
    k = np.arange(n)
    ref = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * (n - 1 - k) / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    err_prev = None
    for _ in range(iters):
        # p(r_i) - f(r_i) = (-1)^i * E * f(r_i)
        A = np.zeros((n, n))
        for i, r in enumerate(ref):
            A[i, :degree + 1] = r ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1.0) ** i) * f(r)
        sol = np.linalg.solve(A, f(ref))
        c = sol[:degree + 1]
        e = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: one extremum per sign-alternating run of the error curve
        sign = np.sign(e)
        sign[sign == 0] = 1
        bounds = np.flatnonzero(np.diff(sign)) + 1
        runs = np.split(np.arange(grid.size), bounds)
        ext = [run[np.argmax(np.abs(e[run]))] for run in runs]
        if len(ext) < n:
            break
        # keep the n consecutive extrema with the largest minimum magnitude
        best = max(range(len(ext) - n + 1), key=lambda s: np.abs(e[ext[s:s + n]]).min())
        ref = grid[ext[best:best + n]]
        err = np.abs(e).max()
        if err_prev is not None and abs(err - err_prev) < 1e-15:
            break
        err_prev = err
    return c, float(np.abs(e).max())


def emulated_exp2_f32(x, coeffs):
    """Reference model of the kernel's sequence in float32 (fma modelled in float64)."""
    f32 = np.float32
    x = np.maximum(np.asarray(x, f32), f32(-125.0))
    magic = f32(12582912.0)                      # 1.5 * 2^23
    t = (x + magic).astype(f32)
    nf = (t - magic).astype(f32)
    r = (x - nf).astype(f32)
    c = [f32(v) for v in coeffs]

    def fma(a, b, d):
        # a*b is exact in float64 for float32 inputs; one rounding to float32 after the add
        return (a.astype(np.float64) * b.astype(np.float64) + np.float64(d)).astype(f32)

    p = fma(r, np.full_like(r, c[3]), c[2])     # Horner: ((c3 r + c2) r + c1) r + c0
    p = fma(r, p, c[1])
    p = fma(r, p, c[0])
    bits = (p.view(np.uint32).astype(np.int64) + (t.view(np.uint32).astype(np.int64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def main():
    c, err = remez_relative()
    c32 = [float(np.float32(v)) for v in c]
    xs = np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float32)
    got = emulated_exp2_f32(xs, c32).astype(np.float64)
    rel = np.abs(got / np.exp2(xs.astype(np.float64)) - 1).max()
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "exp2_poly.cuh")
    with open(path, "w") as fh:
        fh.write(
            "// exp2_poly.cuh -- written by exp2_poly_fit.py; do not edit by hand.\n"
            "// 2^r on [-1/2, 1/2], degree-3 minimax in relative error (Remez exchange),\n"
            "// coefficients rounded to fp32.  Levelled relative error of the fit: "
            f"{err:.3e};\n// max relative error of the full fp32 sequence over x in [-125, 8]: {rel:.3e}.\n"
            "#pragma once\n\nnamespace fa {\n"
            + "".join(f"constexpr float kExp2C{i} = {v!r}f;\n" for i, v in enumerate(c32))
            + "constexpr float kExp2MaxRelErr = " + f"{rel:.3e}" + "f;\n}  // namespace fa\n")
    print(path, c32, err, rel)


if __name__ == "__main__":
    main()
