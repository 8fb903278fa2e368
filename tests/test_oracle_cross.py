"""Pins of the oracle's cross-attention over the cached text K/V (CPU only).

* brute force with scalar loops (math.exp) on tiny inputs, d = 128;
* Q = 0 gives the mean of the text values exactly; one text token gives its value;
* no positions: the output does not depend on which frame a query token belongs to
  nor on the order of the text tokens (a RoPE applied by mistake breaks both);
* the self-attention cache is untouched and does not influence the result; a new
  prompt replaces only the text K/V.
"""
import math

import numpy as np
import pytest

from oracle import bf16
from oracle.layer import OracleLayer, StateError


def _bits(rng, shape, scale=1.0):
    return bf16.from_f64(rng.standard_normal(shape) * scale)


def _layer(H=2):
    return OracleLayer(H, 128, 4, 2, 2, 6, 2, OracleLayer.ABSOLUTE)


def test_cross_brute_force():
    rng = np.random.default_rng(11)
    orc = _layer()
    q, k, v = _bits(rng, (3, 2, 128)), _bits(rng, (5, 2, 128)), _bits(rng, (5, 2, 128))
    orc.set_text_kv(k, v)
    got = orc.cross_attention(q)
    qf, kf, vf = bf16.to_f64(q), bf16.to_f64(k), bf16.to_f64(v)
    for i in range(3):
        for h in range(2):
            s = [math.fsum(qf[i, h, t] * kf[j, h, t] for t in range(128)) / math.sqrt(128) for j in range(5)]
            m = max(s)
            e = [math.exp(x - m) for x in s]
            z = math.fsum(e)
            for t in range(128):
                ref = math.fsum(e[j] * vf[j, h, t] for j in range(5)) / z
                assert abs(got[i, h, t] - ref) <= 1e-13


def test_cross_closed_forms():
    rng = np.random.default_rng(12)
    orc = _layer()
    k, v = _bits(rng, (512, 2, 128)), _bits(rng, (512, 2, 128))
    orc.set_text_kv(k, v)
    q0 = np.zeros((7, 2, 128), dtype=np.uint16)
    mean = bf16.to_f64(v).mean(axis=0)
    assert np.allclose(orc.cross_attention(q0), mean[None], rtol=0, atol=1e-15)
    orc.set_text_kv(k[:1], v[:1])
    one = orc.cross_attention(_bits(rng, (9, 2, 128), 4.0))
    assert np.array_equal(one, np.broadcast_to(bf16.to_f64(v[:1]), one.shape))


def test_cross_has_no_positions():
    rng = np.random.default_rng(13)
    orc = _layer()
    T = orc.T
    k, v = _bits(rng, (37, 2, 128)), _bits(rng, (37, 2, 128))
    orc.set_text_kv(k, v)
    frame = _bits(rng, (T, 2, 128))
    q = np.concatenate([frame, frame, frame])          # three frames with identical bits
    out = orc.cross_attention(q)
    assert np.array_equal(out[:T], out[T:2 * T]) and np.array_equal(out[:T], out[2 * T:])
    perm = rng.permutation(37)
    orc.set_text_kv(k[perm], v[perm])
    assert np.allclose(orc.cross_attention(q), out, rtol=0, atol=1e-14)


def test_cross_independent_of_self_cache_and_prompt_swap():
    rng = np.random.default_rng(14)
    orc = _layer()
    with pytest.raises(StateError):
        orc.cross_attention(np.zeros((1, 2, 128), dtype=np.uint16))
    k, v = _bits(rng, (20, 2, 128)), _bits(rng, (20, 2, 128))
    orc.set_text_kv(k, v)
    q = _bits(rng, (8, 2, 128))
    before = orc.cross_attention(q)
    for f in range(0, 10, 2):                          # commit frames, with evictions
        kc, vc = _bits(rng, (2 * orc.T, 2, 128)), _bits(rng, (2 * orc.T, 2, 128))
        orc.chunk_attention(kc, kc, vc, 2, f, True)
    held = orc.logical_frames()
    kv_bits = orc.logical_kv_bits()
    assert np.array_equal(orc.cross_attention(q), before)
    k2, v2 = _bits(rng, (33, 2, 128)), _bits(rng, (33, 2, 128))
    orc.set_text_kv(k2, v2)                            # a new prompt
    assert orc.logical_frames() == held
    assert all(np.array_equal(a, b) for a, b in zip(orc.logical_kv_bits(), kv_bits))
    assert not np.allclose(orc.cross_attention(q), before)
