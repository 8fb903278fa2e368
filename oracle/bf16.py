"""bf16 <-> fp64, by definition (oracle; test infrastructure only).

bf16 is the upper half of an IEEE binary32: 1 sign bit, 8 exponent bits, 7
stored mantissa bits (8 significant bits for normal numbers). The pages fix the
data type of weights and activations as bf16 and the flow->x0 step as double
([P2] §精度); these two helpers are the only conversions the oracle uses.
"""
from __future__ import annotations

import numpy as np

_MIN_NORMAL = 2.0 ** -126
_SUBNORMAL_ULP = 2.0 ** -133
_MAX_FINITE = (2.0 - 2.0 ** -7) * 2.0 ** 127


def to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns (uint16 array) as fp64."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def from_f64(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest bf16, ties to even; returns uint16 bits.

    Normal range: write x = m * 2**e with 0.5 <= |m| < 1 (frexp), keep 8
    significant bits with round-half-even (``np.rint``), i.e. rint(m * 2**8).
    Below the smallest normal the grid is the fixed subnormal spacing 2**-133.
    Values beyond the largest finite bf16 after rounding become +-inf.
    """
    x = np.asarray(x, dtype=np.float64)
    if not np.all(np.isfinite(x)):
        raise ValueError("bf16 rounding of a non-finite value")
    m, e = np.frexp(x)
    y = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)
    small = np.abs(x) < _MIN_NORMAL
    if np.any(small):
        y = np.where(small, np.rint(x / _SUBNORMAL_ULP) * _SUBNORMAL_ULP, y)
    y = np.where(np.abs(y) > _MAX_FINITE, np.copysign(np.inf, y), y)
    # y is now exactly a bf16 value, hence exactly a binary32 value.
    return (y.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)
