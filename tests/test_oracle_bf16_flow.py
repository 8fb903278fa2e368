"""Pins of the oracle's bf16 conversion and flow-matching epilogue (CPU only).

The fp64 -> bf16 rounding is checked against hand-worked fixtures and against the
definition "nearest representable value, ties to the even pattern" by brute
force over neighbouring bit patterns; the epilogue against hand-worked values,
the closed-form round trip and its special cases.
"""
import os

import numpy as np
import pytest

from oracle import bf16, flow

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line


def test_bf16_golden_rne():
    for row in _rows("bf16_rne.txt"):
        x_hex, bits_hex = row.split()[:2]
        got = int(bf16.from_f64(np.array([float.fromhex(x_hex)]))[0])
        assert got == int(bits_hex, 16), (x_hex, hex(got), bits_hex)


def test_bf16_every_finite_pattern_round_trips():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    exp = (bits.astype(np.uint32) >> 7) & 0xFF
    finite = bits[exp != 0xFF]
    vals = bf16.to_f64(finite)
    back = bf16.from_f64(vals)
    # -0.0 and +0.0 both map to a zero; all other patterns map to themselves
    nz = vals != 0
    assert np.array_equal(back[nz], finite[nz])
    assert np.all(bf16.to_f64(back[~nz]) == 0)


def test_bf16_to_f64_known_values():
    assert bf16.to_f64(np.array([0x3F80]))[0] == 1.0
    assert bf16.to_f64(np.array([0xC000]))[0] == -2.0
    assert bf16.to_f64(np.array([0x0001]))[0] == 2.0 ** -133
    assert bf16.to_f64(np.array([0x7F7F]))[0] == (2 - 2 ** -7) * 2.0 ** 127


def test_bf16_overflow_boundary():
    """IEEE 754 round-to-nearest-even overflow: the largest finite bf16 is (2 - 2^-7) 2^127
    (0x7F7F); everything below the midpoint (2 - 2^-8) 2^127 to the next power 2^128 rounds
    down to it, the midpoint ties to the even neighbour 2^128, which is out of range, and
    becomes infinity, as does everything above it."""
    top = (2 - 2 ** -7) * 2.0 ** 127
    mid = (2 - 2 ** -8) * 2.0 ** 127
    below = np.nextafter(mid, 0.0)
    for x, want in [(top, 0x7F7F), (below, 0x7F7F), (mid, 0x7F80), (np.nextafter(mid, np.inf), 0x7F80),
                    (1e39, 0x7F80), (-below, 0xFF7F), (-mid, 0xFF80), (-top, 0xFF7F), (-1e300, 0xFF80)]:
        got = int(bf16.from_f64(np.array([x]))[0])
        assert got == want, (x, hex(got), hex(want))


def test_bf16_nearest_by_brute_force():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(20000) * np.exp(rng.uniform(-30, 30, 20000))
    b = bf16.from_f64(x).astype(np.int64)
    y = bf16.to_f64(b.astype(np.uint16))
    # neighbours one pattern up and down (same sign, so the magnitude moves by one step)
    up = bf16.to_f64((b + 1).astype(np.uint16))
    dn = bf16.to_f64(np.maximum(b - 1, 0).astype(np.uint16))
    err = np.abs(x - y)
    assert np.all(err <= np.abs(x - up))
    assert np.all(err <= np.abs(x - dn))
    # exact midpoints must land on an even pattern
    mids = (y + up) / 2
    mb = bf16.from_f64(mids)
    assert np.all(mb % 2 == 0)


def test_flow_golden():
    for row in _rows("flow_x0_renoise.txt"):
        xt, v, eps, s, sn, x0_exp, xn_exp = row.split()
        x0, xn = flow.x0_renoise_f64(float(xt), float(v), float(eps), float(s), float(sn))
        assert float(x0) == float(x0_exp)
        if xn_exp == "none":
            assert xn is None
        else:
            assert float(xn) == float(xn_exp)
        # the same through bf16 I/O (all values are exact in bf16)
        enc = lambda a: bf16.from_f64(np.array([float(a)]))
        bx0, bxn = flow.x0_renoise_bf16(enc(xt), enc(v), enc(eps), float(s), float(sn))
        assert bf16.to_f64(bx0)[0] == float(x0_exp)
        if xn_exp != "none":
            assert bf16.to_f64(bxn)[0] == float(xn_exp)


@pytest.mark.parametrize("sigma", [1.0, 0.75, 0.5, 0.25])
def test_flow_closed_form_round_trip(sigma):
    # build xt on the flow-matching path from a known x0* and noise, with v = eps - x0*
    rng = np.random.default_rng(7)
    x0_true = rng.standard_normal(4096)
    e1 = rng.standard_normal(4096)
    xt = (1 - sigma) * x0_true + sigma * e1
    v = e1 - x0_true
    x0, _ = flow.x0_renoise_f64(xt, v, e1, sigma, -1.0)
    assert np.max(np.abs(x0 - x0_true)) < 1e-14 * 8
    # renoising the recovered x0 with the same noise at sigma reproduces xt
    _, back = flow.x0_renoise_f64(xt, v, e1, sigma, sigma)
    assert np.max(np.abs(back - xt)) < 1e-14 * 8


def test_flow_special_cases():
    rng = np.random.default_rng(3)
    xt, v, eps = rng.standard_normal((3, 1000))
    x0, xn = flow.x0_renoise_f64(xt, v, eps, 0.0, 0.5)
    assert np.array_equal(x0, xt)                       # sigma = 0: nothing to remove
    x0, xn = flow.x0_renoise_f64(xt, v, eps, 0.5, 0.0)
    assert np.array_equal(xn, x0)                       # sigma' = 0: no noise added
    x0, xn = flow.x0_renoise_f64(xt, v, eps, 0.5, 1.0)
    assert np.array_equal(xn, eps)                      # sigma' = 1: pure noise
    assert flow.x0_renoise_f64(xt, v, eps, 0.25, -1.0)[1] is None


def test_sigma_schedule():
    assert flow.sigmas() == [1.0, 0.75, 0.5, 0.25]


def test_cfg_golden():
    for row in _rows("cfg_combine.txt"):
        left, right = row.split("|")
        c, u, sc, xt, eps, s, sn = map(float, left.split())
        v_exp, x0_exp, xn_exp = right.split()
        assert float(flow.cfg_combine_f64(c, u, sc)) == float(v_exp)
        enc = lambda a: bf16.from_f64(np.array([a]))
        bx0, bxn = flow.cfg_x0_renoise_bf16(enc(xt), enc(c), enc(u), enc(eps), sc, s, sn)
        assert bf16.to_f64(bx0)[0] == float(x0_exp)
        if xn_exp == "none":
            assert bxn is None
        else:
            assert bf16.to_f64(bxn)[0] == float(xn_exp)


def test_cfg_special_cases():
    rng = np.random.default_rng(5)
    # bf16-representable inputs: c - u is exact in fp64, so scale 1 / 0 return c / u exactly
    c = bf16.to_f64(bf16.from_f64(rng.standard_normal(5000)))
    u = bf16.to_f64(bf16.from_f64(rng.standard_normal(5000)))
    assert np.array_equal(flow.cfg_combine_f64(c, u, 1.0), c)
    assert np.array_equal(flow.cfg_combine_f64(c, u, 0.0), u)
    assert np.array_equal(flow.cfg_combine_f64(c, c, 5.0), c)      # no disagreement, no guidance
    # linear in the scale: v(s) - u = s * (c - u)
    assert np.allclose(flow.cfg_combine_f64(c, u, 5.0) - u, 5.0 * (c - u), rtol=0, atol=1e-14)
