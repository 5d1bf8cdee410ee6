"""Fit the coefficients of exp2_poly.h: 2^f on [-1/2, 1/2] by a polynomial of
degree n that minimises the maximum RELATIVE error (Remez exchange).

  python dynamic_sparse_attention_02_b200/csrc/fit_exp2.py [--degree 3]

prints the coefficients rounded to fp32 as the header's C hex-float lines,
the minimax error of the fp64 fit and the error of the fp32-rounded
coefficients.  The method is the textbook Remez exchange: start from the
Chebyshev extrema, solve for the polynomial whose relative error alternates
with equal magnitude at the n + 2 reference points, move the reference points
to the extrema of the new error curve, repeat.
"""
from __future__ import annotations

import argparse

import numpy as np


def remez(n: int, a: float = -0.5, b: float = 0.5, iters: int = 30, grid: int = 200001):
    """Coefficients c[0..n] (c[j] multiplies f^j) and the max relative error."""
    f = np.exp2
    k = np.arange(n + 2)
    x = (a + b) / 2 + (b - a) / 2 * np.cos(np.pi * k[::-1] / (n + 1))
    g = np.linspace(a, b, grid)
    err = None
    c = None
    for _ in range(iters):
        # p(x_i) - f(x_i) = (-1)^i E f(x_i): equal relative error, alternating sign
        A = np.zeros((n + 2, n + 2))
        for i, xi in enumerate(x):
            A[i, :n + 1] = xi ** np.arange(n + 1)
            A[i, n + 1] = -((-1) ** i) * f(xi)
        sol = np.linalg.solve(A, f(x))
        c = sol[:n + 1]
        err = (np.polyval(c[::-1], g) - f(g)) / f(g)
        # the new reference: the n + 2 largest local extrema of the error curve
        idx = [0]
        for j in range(1, len(g) - 1):
            if (err[j] - err[j - 1]) * (err[j + 1] - err[j]) <= 0:
                idx.append(j)
        idx.append(len(g) - 1)
        idx = sorted(idx, key=lambda j: -abs(err[j]))[:n + 2]
        x = np.sort(g[idx])
    return c, float(np.max(np.abs(err)))


def fp32_coefficients(n: int):
    """(fp32 coefficients, fp64-fit error, error with the fp32 coefficients)."""
    c, e = remez(n)
    c32 = c.astype(np.float32)
    g = np.linspace(-0.5, 0.5, 100001)
    e32 = float(np.max(np.abs((np.polyval(c32[::-1].astype(np.float64), g) - np.exp2(g))
                              / np.exp2(g))))
    return c32, e, e32


def c_hex(v: np.float32) -> str:
    """fp32 value as a C hex-float literal with the trailing zeros of its
    23-bit fraction dropped, as the header writes it."""
    m, ex = np.frexp(np.float64(v))          # v = m * 2^ex, 0.5 <= |m| < 1
    frac = int(round((abs(m) * 2 - 1) * (1 << 24)))  # 24 bits after the point, low bit 0
    digits = f"{frac:06x}".rstrip("0") or "0"
    sign = "-" if v < 0 else ""
    return f"{sign}0x1.{digits}p{ex - 1}f"


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--degree", type=int, default=3)
    n = ap.parse_args().degree
    c32, e, e32 = fp32_coefficients(n)
    for j, v in enumerate(c32):
        print(f"constexpr float kExp2C{j} = {c_hex(v)};")
    print(f"// max relative error: {e:.3g} (fp64 fit), {e32:.3g} (fp32 coefficients)")


if __name__ == "__main__":
    main()
