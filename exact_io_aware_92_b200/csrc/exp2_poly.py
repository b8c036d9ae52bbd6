"""Derive the polynomial the softmax kernel uses to evaluate 2^f on the FMA
pipe for part of its exponentials.

Method: minimax approximation of g(f) = 2^f on [-1/2, 1/2] by a polynomial
of degree 3, minimising the maximum RELATIVE error, found with the Remez
exchange algorithm (solve for coefficients and the levelled error on n+2
reference points, move the references to the extrema of the error, repeat).
The kernel splits x = n + f with n = round(x) (adding 1.5 * 2^23 rounds to
the nearest integer in fp32), evaluates p(f) by Horner's rule with fp32 FMAs
and adds n to the exponent field of p(f).

P's values are rounded to bf16 (8 significant bits) right after, so a
relative error near 2^-13 is far below the rounding it precedes.

Run: python exp2_poly.py  -> prints the fp32 coefficients and the error of
the fp32 Horner evaluation on a dense grid.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def remez(degree: int = DEGREE, iters: int = 30):
    n = degree
    # Chebyshev extrema as the starting reference
    k = np.arange(n + 2)
    ref = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k[::-1] / (n + 1))
    grid = np.linspace(LO, HI, 200001)
    coef = None
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E * 2^x_i   (relative error levelled)
        A = np.zeros((n + 2, n + 2))
        for i, x in enumerate(ref):
            A[i, :n + 1] = x ** np.arange(n + 1)
            A[i, n + 1] = -((-1) ** i) * 2.0 ** x
        sol = np.linalg.solve(A, 2.0 ** ref)
        coef = sol[:n + 1]
        err = (np.polyval(coef[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new references: alternating extrema of the error
        sign = np.sign(err)
        breaks = np.flatnonzero(np.diff(sign) != 0)
        segments = np.split(np.arange(grid.size), breaks + 1)
        ext = [seg[np.argmax(np.abs(err[seg]))] for seg in segments]
        if len(ext) >= n + 2:
            # keep the n+2 largest alternating extrema (contiguous window)
            best, best_val = None, -1
            for s in range(len(ext) - (n + 2) + 1):
                w = ext[s:s + n + 2]
                v = np.min(np.abs(err[w]))
                if v > best_val:
                    best, best_val = w, v
            ref = grid[best]
    return coef, float(np.max(np.abs(err)))


def horner_fp32(coef32: np.ndarray, f: np.ndarray) -> np.ndarray:
    """fp32 Horner evaluation with fused multiply-adds (each FMA rounded once)."""
    acc = np.full(f.shape, coef32[-1], dtype=np.float32)
    f32 = f.astype(np.float32)
    for c in coef32[-2::-1]:
        acc = (acc.astype(np.float64) * f32.astype(np.float64) + np.float64(c)).astype(np.float32)
    return acc


def main():
    coef, err = remez()
    coef32 = coef.astype(np.float32)
    f = np.linspace(LO, HI, 1000001)
    rel = np.abs(horner_fp32(coef32, f).astype(np.float64) - 2.0 ** f) / 2.0 ** f
    print("coefficients c0..c3 (fp32):", [float(c) for c in coef32])
    print(f"levelled relative error (exact arithmetic): {err:.3e}")
    print(f"max relative error of the fp32 Horner form: {rel.max():.3e} "
          f"(2^{np.log2(rel.max()):.2f})")


if __name__ == "__main__":
    main()
