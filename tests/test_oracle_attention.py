"""Pins of the oracle's attention and per-layer state machine (CPU only).

* brute force on tiny inputs (scalar loops with math.exp);
* explicit-mask full attention: with a window that covers all history the
  rolling layer must equal full attention over every frame with the
  chunk-granular block-causal mask, RoPE done by an independent complex
  formulation (absolute ids), to 1e-12 (absolute) / 1e-10 (relative);
* closed forms: Q = 0 gives the mean of the visible values, so frame-tagged
  values give the mean visible frame id (pins the visible set through warm-up,
  eviction, wrap and sinks); one visible key gives that key's value exactly;
* relative-mode translation invariance (bitwise) and absolute-mode shift
  equivariance.
"""
import cmath
import math

import numpy as np
import pytest

from oracle import attention, bf16, rope
from oracle.layer import OracleLayer, OrderError


def _bits(rng, shape, scale=1.0):
    return bf16.from_f64(rng.standard_normal(shape) * scale)


def test_attend_brute_force():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((3, 2, 4))
    k = rng.standard_normal((5, 2, 4))
    v = rng.standard_normal((5, 2, 4))
    got = attention.attend(q, k, v)
    for i in range(3):
        for h in range(2):
            s = [sum(q[i, h, t] * k[j, h, t] for t in range(4)) / 2.0 for j in range(5)]
            m = max(s)
            e = [math.exp(x - m) for x in s]
            z = sum(e)
            for t in range(4):
                ref = sum(e[j] / z * v[j, h, t] for j in range(5))
                assert abs(got[i, h, t] - ref) < 1e-14


def test_attend_special_cases():
    rng = np.random.default_rng(4)
    k = rng.standard_normal((7, 3, 8))
    v = rng.standard_normal((7, 3, 8))
    out = attention.attend(np.zeros((2, 3, 8)), k, v)
    assert np.max(np.abs(out - v.mean(axis=0)[None])) < 1e-15
    out = attention.attend(rng.standard_normal((2, 3, 8)), k, np.ones((7, 3, 8)))
    assert np.max(np.abs(out - 1.0)) < 1e-15
    out = attention.attend(rng.standard_normal((4, 3, 8)), k[:1], v[:1])
    assert np.array_equal(out, np.broadcast_to(v[:1], (4, 3, 8)))


# ----------------------------------------------------------------- explicit-mask equality
def _rot_complex(x, t_ids, T, gw, theta=1e4, pairs=(22, 21, 21)):
    n, H, d = x.shape
    out = np.empty_like(x)
    lay = [(a, j, m) for a, m in enumerate(pairs) for j in range(m)]
    for i in range(n):
        pos = (t_ids[i // T], (i % T) // gw, (i % T) % gw)
        for p, (a, j, m) in enumerate(lay):
            r = cmath.exp(1j * pos[a] * theta ** (-j / m))
            for h in range(H):
                z = complex(x[i, h, 2 * p], x[i, h, 2 * p + 1]) * r
                out[i, h, 2 * p], out[i, h, 2 * p + 1] = z.real, z.imag
    return out


def _full_masked(q_rows, q_frames, k_all, v_all, k_frames, chunk_of, T, gw):
    """Full attention over every frame with mask chunk(key) <= chunk(query), absolute RoPE."""
    qr = _rot_complex(q_rows, q_frames, T, gw)
    kr = _rot_complex(k_all, k_frames, T, gw)
    n_q, H, d = q_rows.shape
    qc = chunk_of[q_frames[0]]
    key_chunk = np.repeat([chunk_of[f] for f in k_frames], T)
    out = np.empty((n_q, H, d))
    for h in range(H):
        s = qr[:, h, :] @ kr[:, h, :].T / math.sqrt(d)
        s[:, key_chunk > qc] = -np.inf
        s -= s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        out[:, h, :] = p @ v_all[:, h, :]
    return out


@pytest.mark.parametrize("mode,tol", [(OracleLayer.ABSOLUTE, 1e-12), (OracleLayer.RELATIVE, 1e-10)])
def test_rolling_equals_explicit_mask_when_window_covers_history(mode, tol):
    H, d, gh, gw, C, S, n_chunks = 2, 128, 2, 2, 2, 2, 5
    T = gh * gw
    W = C * n_chunks + 2                       # covers all history: nothing is ever evicted
    lay = OracleLayer(H, d, T, gh, gw, W, S, mode)
    rng = np.random.default_rng(21)
    committed_k, committed_v, frames, chunk_of = [], [], [], {}
    for c in range(n_chunks):
        f0 = c * C
        for f in range(f0, f0 + C):
            chunk_of[f] = c
        for call in range(2):                  # one denoise read, then the commit
            q, k, v = (_bits(rng, (C * T, H, d)) for _ in range(3))
            out = lay.chunk_attention(q, k, v, C, f0, commit=(call == 1))
            k_all = np.concatenate(committed_k + [bf16.to_f64(k)], axis=0)
            v_all = np.concatenate(committed_v + [bf16.to_f64(v)], axis=0)
            ref = _full_masked(bf16.to_f64(q), list(range(f0, f0 + C)), k_all, v_all,
                               frames + list(range(f0, f0 + C)), chunk_of, T, gw)
            assert np.max(np.abs(out - ref)) < tol, (c, call)
        committed_k.append(bf16.to_f64(k))
        committed_v.append(bf16.to_f64(v))
        frames += list(range(f0, f0 + C))


def test_rope_out_bf16_rounds_the_rotated_operands():
    """rope_out_bf16: the attention of the rotated queries and keys rounded to bf16, pinned with
    the independent complex-exponential rotation and full masked attention (absolute ids, a
    window that covers all history); scores x 4 so that the rounding visibly changes the result."""
    H, d, gh, gw, C, S, n_chunks = 2, 128, 2, 2, 2, 2, 3
    T = gh * gw
    W = C * n_chunks + 2
    lay = OracleLayer(H, d, T, gh, gw, W, S, OracleLayer.ABSOLUTE)
    rng = np.random.default_rng(23)
    committed_k, committed_v = [], []
    for c in range(n_chunks):
        f0 = c * C
        q, k, v = _bits(rng, (C * T, H, d), 4.0), _bits(rng, (C * T, H, d)), _bits(rng, (C * T, H, d))
        unrounded = lay.chunk_attention(q, k, v, C, f0, commit=False)   # a read: no state change
        out = lay.chunk_attention(q, k, v, C, f0, commit=True, rope_out_bf16=True)
        assert np.max(np.abs(unrounded - out)) > 1e-4   # the rounding visibly changes the result
        k_all = np.concatenate(committed_k + [bf16.to_f64(k)], axis=0)
        v_all = np.concatenate(committed_v + [bf16.to_f64(v)], axis=0)
        frames = list(range(f0 + C))
        qr = bf16.to_f64(bf16.from_f64(_rot_complex(bf16.to_f64(q), list(range(f0, f0 + C)), T, gw)))
        kr = bf16.to_f64(bf16.from_f64(_rot_complex(k_all, frames, T, gw)))
        ref = np.empty_like(out)
        for h in range(H):
            sc = qr[:, h, :] @ kr[:, h, :].T / math.sqrt(d)
            sc -= sc.max(axis=1, keepdims=True)
            pw = np.exp(sc)
            ref[:, h, :] = (pw / pw.sum(axis=1, keepdims=True)) @ v_all[:, h, :]
        assert np.max(np.abs(out - ref)) < 1e-12, c
        committed_k.append(bf16.to_f64(k))
        committed_v.append(bf16.to_f64(v))


# ----------------------------------------------------------------- visible set closed form
def _visible_frames(f0, C, W, S):
    R = W - S
    vis = list(range(min(S, f0)))
    if f0 > S:
        vis += list(range(max(S, f0 + C - R), f0))
    return vis + list(range(f0, f0 + C))


@pytest.mark.parametrize("W,S,C,refs", [(6, 2, 2, 0), (18, 6, 4, 0), (21, 5, 3, 5), (5, 0, 1, 0), (7, 1, 6, 0)])
def test_zero_query_gives_mean_visible_frame(W, S, C, refs):
    H, d, gh, gw = 1, 128, 1, 2
    T = gh * gw
    lay = OracleLayer(H, d, T, gh, gw, W, S, OracleLayer.ABSOLUTE)

    def tagged(f0, n):
        v = np.repeat(np.arange(f0, f0 + n, dtype=np.float64), T)[:, None, None] * np.ones((1, H, d))
        return bf16.from_f64(v)

    rng = np.random.default_rng(1)
    f0 = 0
    if refs:
        lay.write_chunk(_bits(rng, (refs * T, H, d)), tagged(0, refs), refs, 0)
        f0 = refs
    for _ in range(12):
        for commit in (0, 0, 1):
            q = np.zeros((C * T, H, d), dtype=np.uint16)
            out = lay.chunk_attention(q, _bits(rng, (C * T, H, d)), tagged(f0, C), C, f0, commit)
            expect = float(np.mean(_visible_frames(f0, C, W, S)))
            assert np.max(np.abs(out - expect)) < 1e-12, (f0, commit)
        f0 += C
        assert lay.logical_frames() == _visible_frames(f0 - C, C, W, S)


def test_single_visible_key_returns_its_value():
    lay = OracleLayer(1, 128, 1, 1, 1, window=1, sink=0, rope_mode=OracleLayer.ABSOLUTE)
    rng = np.random.default_rng(8)
    for f0 in range(4):
        q, k, v = (_bits(rng, (1, 1, 128)) for _ in range(3))
        out = lay.chunk_attention(q, k, v, 1, f0, commit=1)
        assert np.array_equal(out, bf16.to_f64(v))


def test_order_is_enforced():
    lay = OracleLayer(1, 128, 1, 1, 1, window=4, sink=1, rope_mode=OracleLayer.ABSOLUTE)
    z = np.zeros((1, 1, 128), dtype=np.uint16)
    with pytest.raises(OrderError):
        lay.chunk_attention(z, z, z, 1, 3, commit=0)
    lay.chunk_attention(z, z, z, 1, 0, commit=0)     # a read does not advance
    with pytest.raises(OrderError):
        lay.chunk_attention(z, z, z, 1, 1, commit=1)


# ----------------------------------------------------------------- invariances
def test_relative_mode_translation_invariance_bitwise():
    """Same raw window contents at chunks 10 and 20 -> bitwise identical outputs (relative ids
    depend only on a frame's place in the window), while absolute ids make them differ."""
    H, d, gh, gw, W, S, C = 2, 128, 2, 2, 6, 2, 2
    T = gh * gw
    period = 10                                     # chunk contents repeat every 10 chunks

    def content(c, call, what):
        rng = np.random.default_rng(1000 * (c % period) + 10 * call + what)
        return _bits(rng, (C * T, H, d))

    outs = {}
    for mode in (OracleLayer.RELATIVE, OracleLayer.ABSOLUTE):
        lay = OracleLayer(H, d, T, gh, gw, W, S, mode)
        lay.write_chunk(_bits(np.random.default_rng(99), (S * T, H, d)),
                        _bits(np.random.default_rng(98), (S * T, H, d)), S, 0)
        for c in range(21):
            f0 = S + c * C
            o = lay.chunk_attention(content(c, 0, 0), content(c, 0, 1), content(c, 0, 2), C, f0, 0)
            outs[(mode, c)] = o
            lay.chunk_attention(content(c, 1, 0), content(c, 1, 1), content(c, 1, 2), C, f0, 1)
    assert np.array_equal(outs[(OracleLayer.RELATIVE, 10)], outs[(OracleLayer.RELATIVE, 20)])
    assert not np.array_equal(outs[(OracleLayer.ABSOLUTE, 10)], outs[(OracleLayer.ABSOLUTE, 20)])


def test_absolute_mode_shift_equivariance():
    rng = np.random.default_rng(17)
    T, gw = 4, 2
    q = rng.standard_normal((T * 2, 2, 128))
    k = rng.standard_normal((T * 5, 2, 128))
    v = rng.standard_normal((T * 5, 2, 128))
    qf, kf = [3, 4], [0, 1, 2, 3, 4]
    ref = None
    for delta in (0, 7, 50, 300):
        qp = rope.token_positions(np.array(qf) + delta, T, gw)
        kp = rope.token_positions(np.array(kf) + delta, T, gw)
        o = attention.attend(rope.rotate(q, qp), rope.rotate(k, kp), v)
        if ref is None:
            ref = o
        assert np.max(np.abs(o - ref)) < 1e-12
