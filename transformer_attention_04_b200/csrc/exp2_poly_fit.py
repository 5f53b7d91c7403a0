"""Fit the cubic that the attention softmax uses for part of its 2^x evaluations.

Method (Cody-Waite style range reduction + a minimax polynomial fitted here):
  x = n + f with n = round(x) (integer) and f in [-1/2, 1/2];  2^x = 2^n * 2^f.
  2^n is applied by adding n to the float's exponent field; 2^f is a cubic
  c0 + c1 f + c2 f^2 + c3 f^3 whose coefficients minimise the maximum RELATIVE error on
  [-1/2, 1/2]. They are found by a Remez exchange started from a weighted least-squares
  fit on Chebyshev nodes; the result is rounded to float32 and its error re-measured
  in float32 arithmetic with fused multiply-adds, as the kernel evaluates it.

    python transformer_attention_04_b200/csrc/exp2_poly_fit.py

prints the coefficients and the error bound; the kernel's constants are its output.
"""
from __future__ import annotations

import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def remez(deg=DEG, iters=30):
    # start: least squares of 2^f with weight 1/2^f on Chebyshev nodes
    k = np.arange(4000)
    f = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * (k + 0.5) / k.size)
    w = 1.0 / np.exp2(f)
    A = np.vander(f, deg + 1, increasing=True) * w[:, None]
    c = np.linalg.lstsq(A, np.exp2(f) * w, rcond=None)[0]
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        err = (np.polyval(c[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
        # pick deg + 2 alternating extrema
        idx = [0]
        for i in range(1, grid.size - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(grid.size - 1)
        idx = np.array(idx)
        # keep the largest alternating set of size deg + 2
        while idx.size > deg + 2:
            a = np.abs(err[idx])
            j = np.argmin(a)
            idx = np.delete(idx, j)
        x = grid[idx]
        # solve p(x_i) - 2^x_i = (-1)^i E 2^x_i
        s = (-1.0) ** np.arange(deg + 2)
        M = np.hstack([np.vander(x, deg + 1, increasing=True), -(s * np.exp2(x))[:, None]])
        sol = np.linalg.solve(M, np.exp2(x))
        c = sol[:deg + 1]
    return c


def f32_eval_error(c32):
    """Max relative error of the kernel's float32 evaluation over x in [-120, 8] (the kernel
    clamps its argument at -120, where 2^x is already negligible next to a row sum >= 1)."""
    x = np.concatenate([np.linspace(-120.0, 8.0, 2_000_001, dtype=np.float32),
                        np.float32(-1) * np.random.default_rng(0).random(200000, dtype=np.float32) * 20])
    magic = np.float32(12582912.0)  # 1.5 * 2^23: x + magic keeps round(x) in the low bits
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = np.float32(c32[3])
    for ci in (c32[2], c32[1], c32[0]):  # Horner with single roundings, as fma does
        p = (np.float64(p) * np.float64(f) + np.float64(ci)).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    y = bits.view(np.float32).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    return float(np.max(np.abs(y - ref) / ref))


def main():
    c = remez()
    c32 = np.array(c, dtype=np.float32)
    grid = np.linspace(LO, HI, 100001)
    rel = np.max(np.abs(np.polyval(c[::-1], grid) - np.exp2(grid)) / np.exp2(grid))
    print("coefficients c0..c3 (float32):")
    for i, ci in enumerate(c32):
        print(f"  c{i} = {float(ci):.9e}f  (0x{np.float32(ci).view(np.uint32):08x})")
    print(f"minimax relative error on [-1/2, 1/2]: {rel:.3e}")
    print(f"float32 evaluation, x in [-120, 8]: max relative error {f32_eval_error(c32):.3e}")


if __name__ == "__main__":
    main()
