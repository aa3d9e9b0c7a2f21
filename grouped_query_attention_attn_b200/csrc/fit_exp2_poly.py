"""Fit the polynomial the prefill kernel uses for 2^f on [-1/2, 1/2].

Method: Cody & Waite range reduction (x = n + f, n = round(x), applied in the
kernel with the 1.5*2^23 rounding constant) and a minimax polynomial for 2^f
on the reduced range, fitted here with the Remez exchange algorithm for
relative error.  Run:

    python grouped_query_attention_attn_b200/csrc/fit_exp2_poly.py [degree]

It prints the coefficients (low order first), rounded to float32, and the
maximum relative error of the float32 Horner evaluation on a dense grid.
The kernel rounds the result to bf16 (2^-8 relative precision), so degree 3
(max relative error ~1e-4) is enough.
"""

import sys

import numpy as np


def remez_exp2(deg, iters=30):
    lo, hi = -0.5, 0.5
    n = deg + 2
    k = np.arange(n)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * (n - 1 - k) / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    coef = None
    for _ in range(iters):
        f = np.exp2(x)
        # sum_j c_j x^j - f(x) = (-1)^i E f(x)
        A = np.zeros((n, n))
        for j in range(deg + 1):
            A[:, j] = x ** j
        A[:, deg + 1] = -((-1.0) ** k) * f
        sol = np.linalg.solve(A, f)
        coef, E = sol[: deg + 1], sol[deg + 1]
        err = (np.polyval(coef[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
        # new reference: the extrema of the error between sign changes
        sign = np.sign(err)
        cuts = np.where(np.diff(sign) != 0)[0]
        bounds = np.concatenate(([0], cuts + 1, [grid.size]))
        ext = [b0 + np.argmax(np.abs(err[b0:b1])) for b0, b1 in zip(bounds[:-1], bounds[1:])]
        if len(ext) < n:
            break
        ext = np.array(ext)
        # keep the n extrema with the largest errors, alternating
        while ext.size > n:
            drop = np.argmin(np.abs(err[ext]))
            ext = np.delete(ext, drop)
        x = grid[ext]
    return coef, abs(E)


def f32_horner_error(coef32):
    xs = np.linspace(-0.5, 0.5, 2000001).astype(np.float32)
    p = np.float32(coef32[-1]) * np.ones_like(xs)
    for c in coef32[-2::-1]:
        p = (p * xs + np.float32(c)).astype(np.float32)
    ref = np.exp2(xs.astype(np.float64))
    return float(np.max(np.abs(p.astype(np.float64) - ref) / ref))


def main():
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    coef, E = remez_exp2(deg)
    c32 = [np.float32(c) for c in coef]
    print(f"degree {deg}: minimax relative error {E:.3e}")
    print("coefficients (c0 .. c%d), float32:" % deg)
    for i, c in enumerate(c32):
        print(f"  c{i} = {float(c):.9e}f   // {c.view(np.uint32):#010x}")
    print(f"float32 Horner max relative error: {f32_horner_error(c32):.3e}")


if __name__ == "__main__":
    main()
