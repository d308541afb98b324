"""Fits the polynomial the FP8 attention kernel uses to evaluate 2^x on the FMA pipe.

    python video_diffusion_transformer_packed_b200/csrc/exp2_poly.py

Method (range reduction for base 2, as in any exp2 built from a polynomial):
x = n + f with n = round(x) and f in [-1/2, 1/2]; 2^x = 2^n * p(f), where p is
a degree-3 polynomial that minimises the largest *relative* error of p(f)
against 2^f on [-1/2, 1/2]. The minimax fit is computed here with a Remez
exchange on the error function e(f) = p(f) * 2^-f - 1, written from the
equioscillation theorem (n + 2 = 5 alternation points). The coefficients are
rounded to float32; the script prints them as hex literals and the resulting
error bound, and the kernel embeds those literals.

Accuracy needed: the probabilities are rounded to e4m3 (4 significant bits)
before the P.V product, so a relative error near 1e-4 (~2^-13) is far below
the rounding the result receives anyway.
"""
from __future__ import annotations

import struct

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def _rel_err(c, f):
    return np.polyval(c[::-1], f) * np.exp2(-f) - 1.0


def remez(degree: int = DEGREE, iters: int = 30) -> np.ndarray:
    """Minimax coefficients c[0..degree] (lowest first) of p(f) ~ 2^f, relative error."""
    m = degree + 2
    # start from Chebyshev extrema
    k = np.arange(m)
    pts = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k[::-1] / (m - 1))
    c = np.zeros(degree + 1)
    for _ in range(iters):
        # solve p(f_i) * 2^-f_i - 1 = (-1)^i E  for c and E
        A = np.zeros((m, m))
        for i, f in enumerate(pts):
            A[i, :degree + 1] = (f ** np.arange(degree + 1)) * np.exp2(-f)
            A[i, degree + 1] = -((-1) ** i)
        sol = np.linalg.solve(A, np.ones(m))
        c = sol[:degree + 1]
        # new alternation points: extrema of the error on a fine grid
        grid = np.linspace(LO, HI, 200001)
        e = _rel_err(c, grid)
        # split the grid at sign changes and take the extreme of each run
        sign = np.sign(e)
        idx = np.flatnonzero(np.diff(sign) != 0)
        bounds = np.concatenate([[0], idx + 1, [len(grid)]])
        ext = [b0 + int(np.argmax(np.abs(e[b0:b1]))) for b0, b1 in zip(bounds[:-1], bounds[1:]) if b1 > b0]
        if len(ext) < m:
            break
        # keep m alternating extrema with the largest errors
        ext = sorted(ext, key=lambda i: -abs(e[i]))[:m]
        pts = np.sort(grid[ext])
    return c


def as_f32(x: float) -> float:
    return struct.unpack("<f", struct.pack("<f", x))[0]


def f32_hex(x: float) -> str:
    return "0x%08X" % struct.unpack("<I", struct.pack("<f", x))[0]


def coefficients_f32():
    return [as_f32(v) for v in remez()]


def max_rel_error_f32(c32) -> float:
    grid = np.linspace(LO, HI, 400001)
    return float(np.max(np.abs(_rel_err(np.array(c32, dtype=np.float64), grid))))


if __name__ == "__main__":
    c32 = coefficients_f32()
    for i, v in enumerate(c32):
        print(f"c{i} = {f32_hex(v)}  // {v:.9g}")
    print(f"max relative error on [-1/2, 1/2] (float32 coefficients, exact arithmetic): "
          f"{max_rel_error_f32(c32):.3e}")
