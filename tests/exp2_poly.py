"""Derivation of the exp2 polynomial the attention kernel uses on the FMA pipe.

The kernel evaluates part of the softmax exponentials 2^x without the
special-function unit:

* range reduction (Cody-Waite style, one step): with M = 1.5 * 2^23,
  t = x + M rounds x to the nearest integer r = t - M and leaves r in the low
  mantissa bits of t; f = x - r lies in [-1/2, 1/2];
* 2^f by a degree-3 polynomial whose coefficients approximately minimise the
  maximum RELATIVE error on [-1/2, 1/2], fitted here by Lawson's iteratively
  reweighted least squares on Chebyshev nodes;
* 2^x = 2^r * 2^f by adding r << 23 to the bit pattern of the polynomial value
  (the bits of M vanish under the shift).

Run ``python tests/exp2_poly.py`` to print the coefficients
and the error bound; ``EXP2_POLY3`` below are the values compiled into
``csrc/rkv_attention.cu`` (rounded to fp32). The maximum relative error,
7.5e-5, is far below the 2^-9 relative rounding of the bf16 probabilities the
kernel feeds to the PV product.
"""
from __future__ import annotations

import numpy as np

EXP2_POLY3 = (0.9999280735783096, 0.6932609862225388, 0.24261112187715117, 0.05517166493030145)
MAGIC = 12582912.0  # 1.5 * 2^23


def fit(degree: int = 3, nodes: int = 4000, iters: int = 200):
    f = np.cos(np.pi * (np.arange(nodes) + 0.5) / nodes) * 0.5
    y = np.exp2(f)
    a = np.vander(f, degree + 1, increasing=True) / y[:, None]
    w = np.ones_like(f)
    c = None
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(a * sw[:, None], sw, rcond=None)
        e = np.abs(a @ c - 1.0)
        w = w * e
        w /= w.sum()
    return c


def exp2_emulated(x: np.ndarray, coeffs=EXP2_POLY3) -> np.ndarray:
    """The kernel's algorithm in float32 arithmetic (for tests)."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-125.0))
    m = np.float32(MAGIC)
    t = (x + m).astype(np.float32)
    r = (t - m).astype(np.float32)
    f = (x - r).astype(np.float32)
    c0, c1, c2, c3 = (np.float32(v) for v in coeffs)
    p = (c3 * f + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    bits = (t.view(np.uint32).astype(np.uint64) << np.uint64(23)) + p.view(np.uint32).astype(np.uint64)
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


if __name__ == "__main__":
    c = fit()
    g = np.linspace(-0.5, 0.5, 200001)
    err = np.max(np.abs(np.polyval(c[::-1], g) / np.exp2(g) - 1.0))
    print("coefficients", [float(v) for v in c], "max relative error", err)
