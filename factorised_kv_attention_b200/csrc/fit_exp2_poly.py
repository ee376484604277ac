"""Regenerate and check the coefficients of exp2_poly2 (kpa_f32x2.cuh).

    python factorised_kv_attention_b200/csrc/fit_exp2_poly.py

Method: 2^x = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2] (Cody-Waite
reduction; n is exact in float32 for |x| < 2^22).  2^f is approximated by a degree-4
polynomial fitted by weighted least squares on a dense grid of [-1/2, 1/2], with the
weights pushed toward the points of largest relative error for a number of passes
(an iteratively reweighted fit that approaches equal relative ripple).  The float32
coefficients are then evaluated exactly as the kernel does (float32 Horner steps, the
2^n scaling by an integer add into the exponent field) over [-126, 8], against float64
2^x, and compared with the constants written in kpa_f32x2.cuh.
"""
from __future__ import annotations

import os
import re
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
DEG = 4


def fit(deg: int = DEG, passes: int = 60) -> np.ndarray:
    f = np.linspace(-0.5, 0.5, 20001)
    y = np.exp2(f)
    V = np.vander(f, deg + 1, increasing=True)
    w = 1.0 / y                                      # relative error
    for _ in range(passes):
        c, *_ = np.linalg.lstsq(V * w[:, None], y * w, rcond=None)
        rel = (V @ c - y) / y
        w = w * (1 + 8 * np.abs(rel) / np.abs(rel).max())
        w /= w.max()
    return c.astype(np.float32)


def evaluate(c32: np.ndarray, x: np.ndarray) -> np.ndarray:
    """The kernel's float32 sequence for 2^x.  Each Horner step is a fused multiply-add
    on the device: here the product is exact in float64 and the sum is rounded once
    to float64 and then to float32 (the double rounding can differ from the device's
    single rounding by one float32 ulp, in rare ties)."""
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    big = np.float32(12582912.0)                     # 1.5 * 2^23
    j = (x + big).astype(np.float32)
    fr = (x - (j - big).astype(np.float32)).astype(np.float32)
    p = np.float32(c32[4])
    for k in (3, 2, 1, 0):
        p = (p.astype(np.float64) * fr.astype(np.float64) + np.float64(c32[k])).astype(np.float32)
    return (p.view(np.int32) + (j.view(np.int32) << 23)).view(np.float32)


def header_coefficients() -> np.ndarray:
    with open(os.path.join(HERE, "kpa_f32x2.cuh")) as fh:
        text = fh.read()
    vals = {}
    for name, lit in re.findall(r"\b(c[0-4]) = (0x[0-9a-fp.+-]+)f", text):
        vals[name] = float.fromhex(lit)
    return np.array([vals[f"c{k}"] for k in range(DEG + 1)], dtype=np.float32)


def max_rel_error(c32: np.ndarray) -> float:
    xs = np.concatenate([np.linspace(-126, 8, 2_000_001).astype(np.float32),
                         (-np.random.default_rng(0).random(100000) * 30).astype(np.float32)])
    got = evaluate(c32, xs).astype(np.float64)
    want = np.exp2(xs.astype(np.float64))
    return float((np.abs(got - want) / want).max())


def main() -> int:
    c = fit()
    print("fitted coefficients:", [float(v).hex() for v in c])
    h = header_coefficients()
    print("header coefficients:", [float(v).hex() for v in h])
    err = max_rel_error(h)
    print(f"max relative error over [-126, 8] of the header's coefficients: {err:.3e}")
    same = bool(np.array_equal(c, h))
    print("header matches the fit:", same)
    return 0 if same and err < 3e-6 else 1


if __name__ == "__main__":
    sys.exit(main())
