"""Fit of the polynomial the forward kernel uses to evaluate part of its
exponentials on the FMA pipe instead of the MUFU unit.

Method (written here, from the mathematics): 2^x = 2^n * 2^f with
n = round(x) and f = x - n in [-1/2, 1/2]; 2^f is replaced by the cubic p(f)
that minimises the maximum *relative* error on [-1/2, 1/2], found with the
Remez exchange algorithm (equioscillation at deg + 2 points, iterated).  The
kernel forms n by adding 1.5 * 2^23 (round to nearest), evaluates p with three
FMAs and adds n to the exponent field of p's bit pattern.

    python -m io_aware_exact_35_b200.exp2_poly      # prints the coefficients

The coefficients printed here are the ones in csrc/sm100.cuh (ex2_poly3);
tests/test_exp2_poly.py re-derives them and checks the float32 error bound.
"""

from __future__ import annotations

import numpy as np


def remez_exp2(deg: int = 3, lo: float = -0.5, hi: float = 0.5, iters: int = 40,
               grid: int = 200001):
    """Minimax relative-error polynomial for 2^f on [lo, hi]; returns
    (coefficients c0..c_deg, max relative error)."""
    n = deg + 2
    x = np.cos(np.pi * np.arange(n) / (n - 1))[::-1] * (hi - lo) / 2 + (hi + lo) / 2
    xs = np.linspace(lo, hi, grid)
    c = None
    for _ in range(iters):
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * np.exp2(x[i])
        sol = np.linalg.solve(A, np.exp2(x))
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], xs) / np.exp2(xs) - 1.0
        d = np.diff(err)
        ext = [0] + [i for i in range(1, len(xs) - 1) if d[i - 1] * d[i] < 0] + [len(xs) - 1]
        if len(ext) != n:
            break
        x = xs[ext]
    err = np.polyval(c[::-1], xs) / np.exp2(xs) - 1.0
    return c, float(np.max(np.abs(err)))


def ex2_poly3_f32(x: np.ndarray, c: np.ndarray) -> np.ndarray:
    """float32 model of the kernel's evaluation (same operation order)."""
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)  # 1.5 * 2^23
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    c = np.asarray(c, np.float32).astype(np.float64)

    def fma32(a, b, d):  # one rounding to float32 (a*b is exact in float64)
        return (np.asarray(a, np.float64) * np.asarray(b, np.float64) + d).astype(np.float32)

    p = fma32(c[3], f, c[2])
    p = fma32(p, f, c[1])
    p = fma32(p, f, c[0])
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


if __name__ == "__main__":
    coeffs, e = remez_exp2()
    print("c0..c3 =", ", ".join(f"{float(np.float32(v))!r}f" for v in coeffs),
          f"(max rel err {e:.3e})")
