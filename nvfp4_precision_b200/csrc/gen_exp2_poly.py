"""Fit the polynomial used for 2^f on the FMA pipe.

    python nvfp4_precision_b200/csrc/gen_exp2_poly.py [degree] [--half]

Method: Cody and Waite's range reduction 2^x = 2^n * 2^f.  With --half,
n = round-to-nearest(x) and f = x - n in [-1/2, 1/2] (the reduction the
attention kernel uses: adding 1.5 * 2^23 rounds x to an integer held in the
low mantissa bits, which are then shifted into the exponent field, as in
Schraudolph's fast exponential); otherwise n = floor(x), f in [0, 1).
The polynomial for 2^f with p(0) = 1 is the minimax fit of relative error,
solved as a linear program on a dense grid (minimise t subject to
|p(f_i) - 2^f_i| <= t * 2^f_i).  Prints the fp32 coefficients (c1..cd) and
the relative error of the fp32 Horner evaluation, for the attention kernel.
"""
import sys

import numpy as np
from scipy.optimize import linprog


def fit(degree: int, grid: int = 4097, lo: float = 0.0, hi: float = 1.0):
    f = np.linspace(lo, hi, grid)
    y = np.exp2(f)
    # variables: c1..cd, t ; p(f) = 1 + sum c_k f^k
    A, b = [], []
    for fi, yi in zip(f, y):
        powers = [fi ** k for k in range(1, degree + 1)]
        A.append(powers + [-yi])          #  p - y <= t*y  ->  sum c f^k - t y <= y - 1
        b.append(yi - 1.0)
        A.append([-x for x in powers] + [-yi])  # y - p <= t*y
        b.append(1.0 - yi)
    c = np.zeros(degree + 1)
    c[-1] = 1.0
    res = linprog(c, A_ub=np.array(A), b_ub=np.array(b), bounds=[(None, None)] * (degree + 1), method="highs")
    assert res.success, res.message
    return res.x[:degree].astype(np.float32), float(res.x[-1])


def horner_f32(coef, f):
    """fp32 Horner with a fused multiply-add at each step (computed exactly in
    fp64, then rounded to fp32, which is what an fp32 FMA does)."""
    f = f.astype(np.float32)
    acc = np.full_like(f, coef[-1])
    for ck in coef[-2::-1]:
        acc = (acc.astype(np.float64) * f.astype(np.float64) + np.float64(ck)).astype(np.float32)
    return (acc.astype(np.float64) * f.astype(np.float64) + 1.0).astype(np.float32)


if __name__ == "__main__":
    args = [a for a in sys.argv[1:] if not a.startswith("--")]
    d = int(args[0]) if args else 3
    lo, hi = (-0.5, 0.5) if "--half" in sys.argv else (0.0, 1.0)
    coef, t = fit(d, lo=lo, hi=hi)
    f = np.linspace(lo, hi, 1 << 20, endpoint=True, dtype=np.float32)
    err = np.abs(horner_f32(coef, f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1).max()
    print(f"degree {d}: minimax relative error {t:.3e}; fp32 Horner max relative error {err:.3e}")
    for k, ck in enumerate(coef, 1):
        print(f"  c{k} = {float(ck)!r}f  // 0x{np.float32(ck).view(np.uint32):08X}")
