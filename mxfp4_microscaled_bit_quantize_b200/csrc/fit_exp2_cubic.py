"""Fit of the cubic behind exp2_codes_poly (csrc/attn_fwd_sm100.cu).

The kernel only keeps the E2M1 code of 2^x (round to nearest even on the grid 0, 0.5, 1, 1.5, 2,
3, 4, 6 times 2^e), so the polynomial has to land on the right side of the grid's rounding
midpoints, not match 2^x everywhere. After the range reduction x = n + f with n = round(x) and
f in [-0.5, 0.5], every midpoint 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5 of the grid falls at one of
f = 0 (0.25 = 2^-2), log2 0.75, log2 1.25 or log2 0.875 (1.75 = 2 * 0.875). The cubic
p(f) = 1 + c1 f + c2 f^2 + c3 f^3 has p(0) = 1 by construction and interpolates 2^f at the other
three points: a 3 x 3 linear solve in fp64, then rounding to fp32.

Run it to print the coefficients (as C hex-float literals) and the checks the kernel relies on:
monotone on [-0.5, 0.5], within one fp32 ulp of the midpoints at the interpolation points, and the
worst relative distance to 2^f in between.
"""
from __future__ import annotations

import numpy as np


def fit():
    f = np.log2(np.array([0.75, 0.875, 1.25]))
    a = np.stack([f, f ** 2, f ** 3], axis=1)
    return np.linalg.solve(a, np.exp2(f) - 1.0)


def horner32(coef, f):
    """p(f) as the kernel evaluates it: three fp32 fused multiply-adds (fp64 product and sum of fp32
    operands, rounded once to fp32)."""
    c1, c2, c3 = (np.float32(c) for c in coef)
    f = np.asarray(f, dtype=np.float32)
    r = np.full_like(f, c3)
    r = (r.astype(np.float64) * f + np.float64(c2)).astype(np.float32)
    r = (r.astype(np.float64) * f + np.float64(c1)).astype(np.float32)
    r = (r.astype(np.float64) * f + 1.0).astype(np.float32)
    return r


def main():
    coef = fit()
    c32 = [np.float32(c) for c in coef]
    print("coefficients (fp64):", ", ".join(repr(float(c)) for c in coef))
    print("as fp32 hex floats:  ", ", ".join(float(c).hex().replace("0000000p", "p") + "f" for c in c32))
    f = np.linspace(-0.5, 0.5, 1_000_001).astype(np.float32)
    p = horner32(c32, f)
    print("monotone on [-0.5, 0.5]:", bool(np.all(np.diff(p.astype(np.float64)) >= 0)))
    print("max relative distance to 2^f:", float(np.max(np.abs(p / np.exp2(f.astype(np.float64)) - 1))))
    for target in (0.75, 0.875, 1.25):
        fb = np.float32(np.log2(target))
        got = float(horner32(c32, np.array([fb]))[0])
        print(f"p(log2 {target}) = {got!r} (midpoint {target}, {abs(got - target) / target:.2e} relative)")


if __name__ == "__main__":
    main()
