"""Coefficients of the FMA-pipe exp2 used by the forward kernel for part of
each score row (so the special-function unit is not the only exp2 source).

Method: Cody-Waite range reduction x = n + f with n = rint(x), f in [-1/2, 1/2],
then 2^x = 2^n * p(f) with p the degree-3 polynomial that minimises the maximum
*relative* error |p(f) / 2^f - 1| on [-1/2, 1/2], found by the Remez exchange
algorithm below (written for this project; run this file to print the constants
that fwd_sm100.cuh embeds).  2^n is applied by adding n to the exponent field.

The bound needed: P is rounded to bf16 (relative step 2^-8) before the P V
product, so a relative error near 1e-4 in p is far below that rounding.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def _target(x):
    return np.exp2(x)


def remez(degree: int = DEGREE, iters: int = 30) -> tuple[np.ndarray, float]:
    """Minimax relative-error polynomial for 2^f on [LO, HI].

    Returns (coefficients c0..cdegree in increasing order, max relative error).
    """
    n = degree + 2  # reference points
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * (n - 1 - k) / (n - 1))  # Chebyshev extrema
    dense = np.linspace(LO, HI, 200001)
    coef, err = None, None
    for _ in range(iters):
        # Solve p(x_i) - (-1)^i E 2^{x_i} = 2^{x_i}  (relative weighting)
        A = np.zeros((n, n))
        for j in range(degree + 1):
            A[:, j] = x ** j
        A[:, degree + 1] = ((-1.0) ** k) * _target(x)
        sol = np.linalg.solve(A, _target(x))
        coef = sol[: degree + 1]
        # new reference: extrema of the relative error on a dense grid
        r = np.polyval(coef[::-1], dense) / _target(dense) - 1.0
        # locate n alternating extrema
        sign_change = np.where(np.diff(np.sign(r)) != 0)[0]
        edges = np.concatenate(([0], sign_change + 1, [len(dense)]))
        cand = []
        for a, b in zip(edges[:-1], edges[1:]):
            if b > a:
                i = a + int(np.argmax(np.abs(r[a:b])))
                cand.append(i)
        if len(cand) < n:
            break
        # keep the n largest-|error| alternating points
        while len(cand) > n:
            vals = np.abs(r[cand])
            drop = 0 if vals[0] < vals[-1] else len(cand) - 1
            cand.pop(drop)
        x = dense[cand]
        err = float(np.max(np.abs(r)))
    return coef, err


def emulate_f32(xs: np.ndarray, coef) -> np.ndarray:
    """The kernel's arithmetic in float32: clamp, magic-constant rint, Horner
    polynomial, exponent add (no rounding beyond what float32 itself does)."""
    c = [np.float32(v) for v in coef]
    x = np.maximum(xs.astype(np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)  # 1.5 * 2^23
    t = (x + magic).astype(np.float32)
    nf = (t - magic).astype(np.float32)
    f = (x - nf).astype(np.float32)
    p = (c[3] * f + c[2]).astype(np.float32)
    p = (p * f + c[1]).astype(np.float32)
    p = (p * f + c[0]).astype(np.float32)
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


if __name__ == "__main__":
    coef, err = remez()
    print("max relative error (real arithmetic):", err)
    for i, v in enumerate(coef):
        print(f"c{i} = {np.float32(v)!r}f  ({v:.12e})")
