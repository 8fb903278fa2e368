"""The attention kernel's polynomial exp2 (FMA-pipe path), emulated in float32 on the CPU:
coefficients reproduce from their fit, and the full algorithm (range reduction, polynomial,
exponent insertion) stays within 1e-4 relative error of 2^x over the range the softmax uses."""
import importlib.util
import os

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
_spec = importlib.util.spec_from_file_location("exp2_poly", os.path.join(ROOT, "tests", "exp2_poly.py"))
exp2_poly = importlib.util.module_from_spec(_spec)
_spec.loader.exec_module(exp2_poly)


def test_coefficients_reproduce():
    c = exp2_poly.fit()
    assert np.allclose(c, exp2_poly.EXP2_POLY3, rtol=0, atol=1e-9)


def test_emulated_kernel_algorithm_error():
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001), np.arange(-125, 9).astype(np.float64)])
    y = exp2_poly.exp2_emulated(x).astype(np.float64)
    ref = np.exp2(np.maximum(x.astype(np.float32).astype(np.float64), -125.0))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() < 1.0e-4
    assert np.all(y > 0)
    # below the clamp the value stays tiny and positive instead of wrapping
    assert exp2_poly.exp2_emulated(np.array([-1e4, -300.0, -126.0]))[0] < 1e-37
