"""Fit the polynomial the kernel uses to evaluate part of its exponentials on
the FMA pipe instead of the special-function unit.

Method (Cody & Waite, "Software Manual for the Elementary Functions", 1980,
argument reduction; Remez exchange for the minimax fit):
  2^x = 2^j * 2^f,  j = round-to-nearest(x),  f = x - j in [-1/2, 1/2];
  2^f ~ P(f) = c0 + c1 f + c2 f^2 + c3 f^3, the polynomial of degree 3 that
  minimises the maximum *relative* error max |P(f) / 2^f - 1| on [-1/2, 1/2].
The kernel forms j with the float32 "magic number" rounding (x + 1.5 * 2^23
rounds x to an integer in the low mantissa bits), evaluates P by Horner's
rule in float32 and adds j to the exponent field of P's bits.

Run ``python -m patch_res_diffusion_b200.fit_exp2_poly`` to print the
coefficients (float32) and the error bound; the kernel source carries the
printed values.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5
# arguments below this give 0 (2^j must stay a normal float32 exponent)
CLAMP = -125.0


def _solve_levelled(nodes: np.ndarray, degree: int) -> tuple[np.ndarray, float]:
    """Coefficients c and level E with P(x_i) - 2^x_i = (-1)^i E 2^x_i."""
    n = degree + 2
    A = np.zeros((n, n))
    b = np.exp2(nodes)
    for i, x in enumerate(nodes):
        A[i, :degree + 1] = x ** np.arange(degree + 1)
        A[i, degree + 1] = -((-1) ** i) * np.exp2(x)
    sol = np.linalg.solve(A, b)
    return sol[:degree + 1], sol[degree + 1]


def remez(degree: int = DEGREE, iters: int = 30) -> tuple[np.ndarray, float]:
    """Minimax (relative error) polynomial for 2^x on [LO, HI]."""
    k = np.arange(degree + 2)
    nodes = 0.5 * (LO + HI) - 0.5 * (HI - LO) * np.cos(np.pi * k / (degree + 1))
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        c, _ = _solve_levelled(nodes, degree)
        err = np.polyval(c[::-1], grid) / np.exp2(grid) - 1.0
        # new reference: the extremum of each sign-alternating run of the error
        sign = np.sign(err)
        sign[sign == 0] = 1
        runs = np.split(np.arange(grid.size), np.flatnonzero(np.diff(sign)) + 1)
        ext = np.array([r[np.argmax(np.abs(err[r]))] for r in runs])
        if ext.size > degree + 2:  # keep the degree+2 largest alternating extrema
            while ext.size > degree + 2:
                drop = 0 if abs(err[ext[0]]) < abs(err[ext[-1]]) else ext.size - 1
                ext = np.delete(ext, drop)
        nodes = grid[ext]
    c, _ = _solve_levelled(nodes, degree)
    err = np.polyval(c[::-1], grid) / np.exp2(grid) - 1.0
    return c, float(np.abs(err).max())


def coefficients_f32() -> np.ndarray:
    c, _ = remez()
    return c.astype(np.float32)


def emulate_exp2_f32(x: np.ndarray, c: np.ndarray) -> np.ndarray:
    """The kernel's float32 sequence, step by step (fused multiply-adds are
    evaluated in float64 and rounded once, which is exact for float32 inputs
    up to the final rounding)."""
    f32 = np.float32
    x0 = x
    x = np.maximum(np.asarray(x, dtype=f32), f32(CLAMP))
    magic = f32(12582912.0)  # 1.5 * 2^23
    t = (x + magic).astype(f32)
    j = (t - magic).astype(f32)
    f = (x - j).astype(f32)
    p = c[3].astype(f32)
    for ck in (c[2], c[1], c[0]):
        p = (p.astype(np.float64) * f.astype(np.float64) + np.float64(ck)).astype(f32)
    bits = p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))
    out = (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(f32)
    return np.where(np.asarray(x0, dtype=f32) < f32(CLAMP), f32(0.0), out)


if __name__ == "__main__":
    c, e = remez()
    c32 = c.astype(np.float32)
    xs = np.linspace(-30.0, 8.0, 2_000_001, dtype=np.float32)
    rel = np.abs(emulate_exp2_f32(xs, c32).astype(np.float64) / np.exp2(xs.astype(np.float64)) - 1.0)
    print("coefficients (c0..c3):", ", ".join(f"{v!r}f" for v in c32.tolist()))
    print(f"minimax relative error (real arithmetic): {e:.3e}")
    print(f"float32 sequence, max relative error on [-30, 8]: {rel.max():.3e}")
