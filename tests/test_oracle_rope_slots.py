"""Pins of the oracle's slot-order relative RoPE (time id = position in the visible window).

ABot-World's relative RoPE ("ABot-World流式因果推理深度解析", §机制三) gives queries and keys
one local coordinate system over the current window. The slot-order reading numbers the
visible frames 0 .. n-1 in logical order (sinks, kept history, chunk); the clamped
re-basing reading (the default relative mode) sends old sinks to id 0 instead. Pins:

* hand-worked window: W=6, S=2, C=2 at frame 10, with one-token frames whose q and k
  have only rotary pair 0 set (omega = 1), so a score is a^2 cos(t_q - t_k) / sqrt(d) in
  closed form; frame-tagged values make the output the softmax-weighted mean frame id,
  computed here from the hand-listed ids (slot order 0..5, clamped re-basing 0,0,2..5);
* without sinks the two readings agree (their ids differ by a constant, which RoPE
  cancels), to 1e-12 through warm-up, eviction and wrap;
* steady-state translation invariance, bitwise;
* the standalone rotation's ids against a hand-worked list.
"""
import math

import numpy as np

from oracle import bf16, rope
from oracle.layer import OracleLayer

D = 128
SLOTS, REL = OracleLayer.RELATIVE_SLOTS, OracleLayer.RELATIVE


def _pair0(n_frames, a):
    x = np.zeros((n_frames, 1, D))
    x[:, 0, 0] = a
    return bf16.from_f64(x)


def _tagged(frames):
    return bf16.from_f64(np.repeat(np.asarray(frames, dtype=np.float64)[:, None, None], D, axis=2))


def _expected_mean_frame(a, t_q, ids):
    """sum_f w_f f / sum_f w_f with w_f = exp(a^2 cos(t_q - t_f) / sqrt(d)); ids: {frame: t}."""
    w = {f: math.exp(a * a * math.cos(t_q - t) / math.sqrt(D)) for f, t in ids.items()}
    return sum(wf * f for f, wf in w.items()) / sum(w.values())


def _run_to_frame_10(mode, a):
    """W=6, S=2, C=2, one token per frame: sinks 0, 1 written first, then chunks committed up
    to frame 10; returns the read of chunk [10, 12) (queries frames 10 and 11)."""
    W, S, C = 6, 2, 2
    lay = OracleLayer(1, D, 1, 1, 1, W, S, mode)
    lay.write_chunk(_pair0(S, a), _tagged([0, 1]), S, 0)
    for f0 in range(2, 10, C):
        lay.chunk_attention(_pair0(C, a), _pair0(C, a), _tagged([f0, f0 + 1]), C, f0, commit=1)
    assert lay.window_frames(C, 10) == [0, 1, 8, 9, 10, 11]
    return lay.chunk_attention(_pair0(C, a), _pair0(C, a), _tagged([10, 11]), C, 10, commit=0)


def test_hand_worked_window_scores():
    a = 3.0
    slot_ids = {0: 0, 1: 1, 8: 2, 9: 3, 10: 4, 11: 5}
    clamped_ids = {0: 0, 1: 0, 8: 2, 9: 3, 10: 4, 11: 5}   # clamp(f - (12 - 6), 0, 5)
    for mode, ids in ((SLOTS, slot_ids), (REL, clamped_ids)):
        out = _run_to_frame_10(mode, a)
        for row, fq in enumerate((10, 11)):
            want = _expected_mean_frame(a, ids[fq], ids)
            assert np.allclose(out[row, 0, :], want, rtol=0, atol=1e-12), (mode, fq)
    # the two readings really differ here (the sinks' ids are the only difference)
    assert abs(_run_to_frame_10(SLOTS, a)[0, 0, 0] - _run_to_frame_10(REL, a)[0, 0, 0]) > 1e-3


def _rollout(mode, W, S, C, chunks, seed, T=4, gh=2, gw=2, H=2):
    rng = np.random.default_rng(seed)
    lay = OracleLayer(H, D, T, gh, gw, W, S, mode)
    outs = []
    f0 = 0
    if S:
        lay.write_chunk(bf16.from_f64(rng.standard_normal((S * T, H, D))),
                        bf16.from_f64(rng.standard_normal((S * T, H, D))), S, 0)
        f0 = S
    for _ in range(chunks):
        for commit in (0, 1):
            q, k, v = (bf16.from_f64(rng.standard_normal((C * T, H, D))) for _ in range(3))
            outs.append(lay.chunk_attention(q, k, v, C, f0, commit))
        f0 += C
    return outs


def test_without_sinks_equals_clamped_rebasing():
    for W, C in ((4, 1), (6, 2), (7, 3)):
        a = _rollout(SLOTS, W, 0, C, 9, seed=W)
        b = _rollout(REL, W, 0, C, 9, seed=W)
        for x, y in zip(a, b):
            assert np.allclose(x, y, rtol=0, atol=1e-12)


def test_with_sinks_differs_from_clamped_rebasing_after_eviction_only():
    a = _rollout(SLOTS, 6, 2, 2, 6, seed=3)
    b = _rollout(REL, 6, 2, 2, 6, seed=3)
    # chunks at frames 2 and 4 see no eviction yet (window end <= W): same scores
    for x, y in zip(a[:4], b[:4]):
        assert np.allclose(x, y, rtol=0, atol=1e-12)
    # from frame 6 on the sinks are older than the window: clamped to 0 in one reading only
    assert all(not np.allclose(x, y, rtol=0, atol=1e-6) for x, y in zip(a[6:], b[6:]))


def test_slot_mode_translation_invariance_bitwise():
    H, gh, gw, W, S, C = 2, 2, 2, 6, 2, 2
    T = gh * gw
    period = 10

    def content(c, call, what):
        return bf16.from_f64(np.random.default_rng(1000 * (c % period) + 10 * call + what).standard_normal((C * T, H, D)))

    lay = OracleLayer(H, D, T, gh, gw, W, S, SLOTS)
    lay.write_chunk(content(-1, 0, 0), content(-1, 0, 1), S, 0)
    outs = {}
    for c in range(21):
        f0 = S + c * C
        outs[c] = lay.chunk_attention(content(c, 0, 0), content(c, 0, 1), content(c, 0, 2), C, f0, 0)
        lay.chunk_attention(content(c, 1, 0), content(c, 1, 1), content(c, 1, 2), C, f0, 1)
    assert np.array_equal(outs[10], outs[20])


def test_rope_apply_slot_ids_hand_worked():
    H, gh, gw, W, S = 1, 1, 2, 6, 2
    T = gh * gw
    lay = OracleLayer(H, D, T, gh, gw, W, S, SLOTS)
    rng = np.random.default_rng(5)
    cases = [
        # (start, n, window_end, ids): sinks keep f, the rest lose max(0, end - W) and clamp
        (0, 4, 4, [0, 1, 2, 3]),
        (10, 2, 12, [4, 5]),
        (0, 2, 12, [0, 1]),
        (8, 4, 12, [2, 3, 4, 5]),
        (1, 3, 30, [1, 0, 0]),
        (40, 2, 30, [5, 5]),
    ]
    for start, n, end, ids in cases:
        x = bf16.from_f64(rng.standard_normal((n * T, H, D)))
        got = lay.rope_apply(x, n, start, end)
        want = rope.rotate(bf16.to_f64(x), rope.token_positions(ids, T, gw))
        assert np.array_equal(got, want), (start, n, end)
