"""3D rotary position embedding, fp64 (oracle; test infrastructure only).

Each token carries three position ids (t, h, w): its time id, and the row and
column of its latent patch in the ``grid_h x grid_w`` grid of a frame. Tokens
are frame-major, then grid row, then grid column, so token ``i`` of a frame has
``h = i // grid_w`` and ``w = i % grid_w``.

The head dimension d is split into d/2 adjacent pairs (x[2p], x[2p+1]). The
first ``pairs[0]`` pairs belong to the time axis, the next ``pairs[1]`` to the
row axis and the last ``pairs[2]`` to the column axis (22 / 21 / 21 for d=128,
theta=1e4, as in the benchmark configurations). Pair p with local index j on an
axis with n pairs turns by ``pos_axis * omega_p`` radians, omega_p = theta**(-j/n),
the usual RoPE frequency ladder on a 2n-dimensional sub-space.

Time ids ([P1] §Attention Sink; [P2] §3 ``causal_rope_apply``; [P3] §改造③ ``rope_apply(...,
start_frame=current_start_frame)``; [P4] §机制三 ``relative_rope_apply``):

* absolute: the id is the frame's absolute index (the chunk is shifted by its start frame);
* relative: ids are re-based so that the current chunk's last frame is ``window-1`` and then
  clamped to ``[0, window-1]`` (the page's "clamp the time id to [0, 20]" for a 21-frame
  window); raw keys are cached and re-rotated with these ids on every call.
* relative, slot order: the id is the frame's position in the visible window listed in
  logical order (sinks, then the kept history, then the chunk): 0 .. n-1. This is the other
  plain reading of [P4] §机制三's "query and key share one local coordinate system over the
  current window"; it differs from the clamped re-basing only in the sink frames, which
  keep distinct ids 0 .. S-1 instead of collapsing onto 0.
"""
from __future__ import annotations

import numpy as np

DEFAULT_PAIRS = (22, 21, 21)
DEFAULT_THETA = 1.0e4


def pair_table(pairs=DEFAULT_PAIRS):
    """(axis, j, n) for every pair p: axis 0=t, 1=h, 2=w; j = index on that axis; n = pairs on it."""
    axis, loc, cnt = [], [], []
    for a, n in enumerate(pairs):
        for j in range(n):
            axis.append(a)
            loc.append(j)
            cnt.append(n)
    return np.array(axis), np.array(loc, dtype=np.float64), np.array(cnt, dtype=np.float64)


def omegas(theta=DEFAULT_THETA, pairs=DEFAULT_PAIRS) -> np.ndarray:
    """Angular frequency of each pair: theta ** (-j / n_axis)."""
    _, j, n = pair_table(pairs)
    return np.power(float(theta), -j / n)


def time_ids_absolute(frames) -> np.ndarray:
    return np.asarray(frames, dtype=np.int64)


def time_ids_slot_order(n_visible: int) -> np.ndarray:
    """Ids of the visible window's frames in their logical order: 0 .. n_visible-1."""
    return np.arange(n_visible, dtype=np.int64)


def time_ids_relative(frames, start_frame: int, n_frames: int, window: int) -> np.ndarray:
    """t = clamp(f - (start_frame + n_frames - window), 0, window - 1)."""
    base = start_frame + n_frames - window
    return np.clip(np.asarray(frames, dtype=np.int64) - base, 0, window - 1)


def token_positions(frame_time_ids, tokens_per_frame: int, grid_w: int) -> np.ndarray:
    """[n_frames * T, 3] int64 (t, h, w) for consecutive whole frames with the given time ids."""
    t_ids = np.asarray(frame_time_ids, dtype=np.int64)
    tok = np.arange(tokens_per_frame, dtype=np.int64)
    pos = np.empty((len(t_ids) * tokens_per_frame, 3), dtype=np.int64)
    pos[:, 0] = np.repeat(t_ids, tokens_per_frame)
    pos[:, 1] = np.tile(tok // grid_w, len(t_ids))
    pos[:, 2] = np.tile(tok % grid_w, len(t_ids))
    return pos


def rotate(x: np.ndarray, pos: np.ndarray, theta=DEFAULT_THETA, pairs=DEFAULT_PAIRS) -> np.ndarray:
    """Rotate x [n, H, d] (fp64) by the positions pos [n, 3]; returns a new fp64 array."""
    x = np.asarray(x, dtype=np.float64)
    axis, _, _ = pair_table(pairs)
    ang = pos[:, axis].astype(np.float64) * omegas(theta, pairs)[None, :]      # [n, d/2]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    a = x[..., 0::2]
    b = x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return out
