"""Pins of the oracle's rolling cache and 3D RoPE (CPU only).

Cache: a hand-worked fixture, the closed form of what a window of W frames with
S sinks holds after n in-order frames, the ring-slot closed form, and the
"sinks never move" invariant. RoPE: an independent complex-exponential
formulation, the identity at position 0, the 1-radian special case, norm
preservation, the relative-position property of the scores, and the time ids of the
standalone rotation in relative mode against a hand-worked list.
"""
import cmath
import math
import os

import numpy as np
import pytest

from oracle import bf16, rope
from oracle.cache import CapacityError, RollingCache
from oracle.layer import OracleLayer

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ cache
def test_cache_golden_tiny():
    rows = []
    with open(os.path.join(GOLDEN, "rolling_cache_tiny.txt")) as fh:
        for line in fh:
            if line.strip() and not line.startswith("#"):
                rows.append([list(map(int, c.split())) for c in line.split("|")])
    c = RollingCache(window=6, sink=2)
    for (idx,), written, after, next_read in rows:
        c.append(written)
        assert c.slots == after, idx
        nxt = [written[-1] + 1, written[-1] + 2]
        assert c.after_append(nxt) == next_read, idx
        assert c.slots == after                      # a read leaves the cache alone


def _closed_form(n, W, S):
    """Frames held after frames 0..n-1 were appended in order (any chunking that fits)."""
    R = W - S
    return list(range(min(S, n))) + list(range(max(S, n - R), n))


@pytest.mark.parametrize("W,S,C", [(6, 2, 2), (21, 5, 3), (18, 6, 4), (5, 0, 1), (7, 3, 4), (3, 2, 1)])
def test_cache_closed_form(W, S, C):
    c = RollingCache(W, S)
    n = 0
    for _ in range(40):
        c.append(list(range(n, n + C)))
        n += C
        assert c.slots == _closed_form(n, W, S)


def test_cache_mixed_chunk_sizes_and_sink_straddle():
    # five reference frames first (they become the sinks), then chunks of varying size
    W, S = 21, 5
    c = RollingCache(W, S)
    c.append([0, 1, 2, 3, 4])
    n = 5
    rng = np.random.default_rng(0)
    for _ in range(100):
        k = int(rng.integers(1, W - S + 1))
        c.append(list(range(n, n + k)))
        n += k
        assert c.slots == _closed_form(n, W, S)
    # a chunk that straddles the sink boundary: S=6, chunks of 4 (frames 4,5 become sinks)
    c = RollingCache(18, 6)
    c.append([0, 1, 2, 3])
    c.append([4, 5, 6, 7])
    assert c.slots[:6] == [0, 1, 2, 3, 4, 5]


def test_cache_sink_entries_never_move():
    c = RollingCache(6, 2)
    sinks = [object(), object()]
    c.append(sinks)
    for i in range(50):
        c.append([object(), object()])
        assert c.slots[0] is sinks[0] and c.slots[1] is sinks[1]
        assert len(c) == min(6, 2 + 2 * (i + 1))


def test_cache_capacity():
    c = RollingCache(6, 2)
    with pytest.raises(CapacityError):
        c.after_append([0, 1, 2, 3, 4])
    c.append([0, 1, 2, 3])      # exactly W - S fits


def test_ring_slot_closed_form_matches_cache():
    """Ring placement slot(f) = f for f < S, S + (f - S) mod R otherwise puts the frames the
    shift-left cache holds into distinct slots, and reading slots in frame order gives the
    cache's logical order."""
    for W, S, C in [(6, 2, 2), (21, 5, 3), (18, 6, 4), (4, 1, 3)]:
        R = W - S
        c = RollingCache(W, S)
        slot_frame = [-1] * W
        n = 0
        for _ in range(30):
            new = list(range(n, n + C))
            c.append(new)
            for f in new:
                slot_frame[f if f < S else S + (f - S) % R] = f
            n += C
            held = sorted(f for f in slot_frame if f >= 0 and f in c.slots)
            assert held == c.slots                     # same set, logical order = frame order
            assert sorted(f for f in slot_frame if f >= 0) == c.slots


# ------------------------------------------------------------------ RoPE
def _rotate_complex(x, pos, theta, pairs):
    """Independent formulation: pair p as the complex number x[2p] + i x[2p+1], multiplied
    by exp(i * pos_axis * theta**(-j/n)), with the axis layout spelled out by loops."""
    n_tok, H, d = x.shape
    out = np.empty_like(x)
    p = 0
    layout = []
    for axis, n in enumerate(pairs):
        for j in range(n):
            layout.append((axis, j, n))
    for t in range(n_tok):
        for h in range(H):
            for p, (axis, j, n) in enumerate(layout):
                z = complex(x[t, h, 2 * p], x[t, h, 2 * p + 1])
                z *= cmath.exp(1j * pos[t, axis] * theta ** (-j / n))
                out[t, h, 2 * p] = z.real
                out[t, h, 2 * p + 1] = z.imag
    return out


def test_rope_matches_complex_formulation():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((6, 2, 128))
    pos = np.array([[0, 0, 0], [1, 0, 0], [3, 2, 7], [17, 29, 51], [20, 44, 79], [119, 3, 1]])
    got = rope.rotate(x, pos)
    ref = _rotate_complex(x, pos, 1e4, (22, 21, 21))
    assert np.max(np.abs(got - ref)) < 1e-12


def test_rope_identity_at_zero_and_one_radian():
    x = np.zeros((1, 1, 128))
    x[0, 0, 0] = 1.0
    assert np.array_equal(rope.rotate(x, np.array([[0, 0, 0]])), x)
    y = rope.rotate(x, np.array([[1, 0, 0]]))          # pair 0 has omega = theta**0 = 1
    assert y[0, 0, 0] == math.cos(1.0) and y[0, 0, 1] == math.sin(1.0)
    # first pair of the row axis (pair 22) and of the column axis (pair 43) also have omega 1
    x2 = np.zeros((1, 1, 128)); x2[0, 0, 44] = 1.0; x2[0, 0, 86] = 1.0
    y2 = rope.rotate(x2, np.array([[0, 1, 2]]))
    assert y2[0, 0, 44] == math.cos(1.0) and y2[0, 0, 45] == math.sin(1.0)
    assert y2[0, 0, 86] == math.cos(2.0) and y2[0, 0, 87] == math.sin(2.0)


def test_rope_frequency_ladder():
    w = rope.omegas()
    assert w.shape == (64,)
    assert w[0] == 1.0 and w[22] == 1.0 and w[43] == 1.0
    assert abs(w[1] - 1e4 ** (-1 / 22)) < 1e-15
    assert abs(w[21] - 1e4 ** (-21 / 22)) < 1e-18
    assert abs(w[42] - 1e4 ** (-20 / 21)) < 1e-18
    assert np.all(np.diff(w[:22]) < 0) and np.all(np.diff(w[22:43]) < 0) and np.all(np.diff(w[43:]) < 0)


def test_rope_preserves_pair_norms():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((50, 3, 128))
    pos = rng.integers(0, 200, size=(50, 3))
    y = rope.rotate(x, pos)
    nx = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    ny = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    assert np.max(np.abs(nx - ny)) < 1e-12


def test_rope_scores_depend_only_on_position_difference():
    rng = np.random.default_rng(11)
    q = rng.standard_normal((1, 1, 128))
    k = rng.standard_normal((1, 1, 128))
    pq = np.array([[5, 3, 9]])
    pk = np.array([[2, 7, 1]])
    base = float(np.sum(rope.rotate(q, pq) * rope.rotate(k, pk)))
    for shift in ([1, 0, 0], [13, 0, 0], [0, 4, 0], [0, 0, 30], [40, 17, 22]):
        s = np.array([shift])
        moved = float(np.sum(rope.rotate(q, pq + s) * rope.rotate(k, pk + s)))
        assert abs(moved - base) < 1e-10
    # and do depend on it
    other = float(np.sum(rope.rotate(q, pq + [[1, 0, 0]]) * rope.rotate(k, pk)))
    assert abs(other - base) > 1e-6


def test_relative_time_ids():
    # ABot shape: window 21, five reference sinks, chunks of 3 frames
    W, S, C = 21, 5, 3
    # first generated chunk (frames 5..7) after the five references: chunk's last frame -> 20
    ids = rope.time_ids_relative(list(range(0, 8)), 5, C, W)
    assert list(ids) == [13, 14, 15, 16, 17, 18, 19, 20]
    # steady state: chunk 65..67; visible history 52..64; sinks clamp to 0
    f0 = 65
    frames = list(range(S)) + list(range(f0 + C - (W - S), f0)) + list(range(f0, f0 + C))
    ids = rope.time_ids_relative(frames, f0, C, W)
    assert list(ids) == [0] * S + list(range(S, W - C)) + [18, 19, 20]
    assert ids.min() >= 0 and ids.max() <= W - 1


def test_rope_apply_relative_ids_hand_worked():
    # standalone rotation, relative mode: t = clamp(f - (window_end - W), 0, W - 1), W = 6
    H, gh, gw, W, S, D = 1, 1, 2, 6, 2, 128
    T = gh * gw
    lay = OracleLayer(H, D, T, gh, gw, W, S, OracleLayer.RELATIVE)
    rng = np.random.default_rng(6)
    cases = [
        (10, 2, 12, [4, 5]),        # the window's last two frames
        (0, 2, 12, [0, 0]),         # old sinks clamp to 0
        (6, 4, 12, [0, 1, 2, 3]),
        (0, 4, 4, [2, 3, 4, 5]),    # warm-up: the window end is frame 4
        (40, 2, 30, [5, 5]),        # beyond the window end: clamped to W - 1
    ]
    for start, n, end, ids in cases:
        x = bf16.from_f64(rng.standard_normal((n * T, H, D)))
        got = lay.rope_apply(x, n, start, end)
        want = rope.rotate(bf16.to_f64(x), rope.token_positions(ids, T, gw))
        assert np.array_equal(got, want), (start, n, end)


def test_token_positions_grid_order():
    pos = rope.token_positions([4, 9], tokens_per_frame=6, grid_w=3)
    assert pos.tolist() == [[4, 0, 0], [4, 0, 1], [4, 0, 2], [4, 1, 0], [4, 1, 1], [4, 1, 2],
                            [9, 0, 0], [9, 0, 1], [9, 0, 2], [9, 1, 0], [9, 1, 1], [9, 1, 2]]
