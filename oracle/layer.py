"""One DiT layer's rolling-cache attention, as the pages run it (oracle; test infrastructure only).

Per chunk of ``n_frames`` frames starting at ``start_frame``:

* a denoise *read* ([P2] §2-§3; [P4] §机制二) attends with the chunk's K/V placed in
  the cache as the shift-left rule would place them, but does not keep them
  (reads never change what later chunks see: only the clean write-back does);
* the t=0 *commit* ([P2] §3 "用t0再前向一次"; [P4] §机制二 干净上下文回写;
  ``context_noise: 0``) attends the same way and then keeps the chunk's K/V;
* ``write_chunk`` keeps frames without attending (e.g. the five reference views
  that become sinks, [P4] §机制一).

Keys are cached raw (un-rotated) in both RoPE modes and rotated with the ids of
the current call ([P4] §机制三 caches ``k_raw``); for absolute ids the rotation
of a key never changes, so this equals caching rotated keys.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from . import bf16, rope
from .attention import attend
from .cache import RollingCache


class StateError(RuntimeError):
    """A call that needs state not set yet (cross-attention before the text K/V)."""


class OrderError(ValueError):
    """start_frame is not the number of frames committed so far."""


@dataclass
class Frame:
    frame: int
    k: np.ndarray  # [T, H, d] uint16 bf16 bits (raw, un-rotated)
    v: np.ndarray  # [T, H, d] uint16


class OracleLayer:
    ABSOLUTE = 0
    RELATIVE = 1
    RELATIVE_SLOTS = 2  # relative RoPE with ids = position in the visible window (sinks 0..S-1)

    def __init__(self, H, d, tokens_per_frame, grid_h, grid_w, window, sink, rope_mode,
                 theta=rope.DEFAULT_THETA, pairs=rope.DEFAULT_PAIRS):
        if grid_h * grid_w != tokens_per_frame:
            raise ValueError("grid_h * grid_w must equal tokens_per_frame")
        if 2 * sum(pairs) != d:
            raise ValueError("the rotary pairs must cover the head dimension")
        self.H, self.d, self.T = H, d, tokens_per_frame
        self.grid_h, self.grid_w = grid_h, grid_w
        self.window, self.sink = window, sink
        self.rope_mode = rope_mode
        self.theta, self.pairs = theta, tuple(pairs)
        self.cache = RollingCache(window, sink)
        self.committed = 0

    # ------------------------------------------------------------ helpers
    def _split_frames(self, k_bits, v_bits, n_frames, start_frame):
        k = np.asarray(k_bits, dtype=np.uint16).reshape(n_frames, self.T, self.H, self.d)
        v = np.asarray(v_bits, dtype=np.uint16).reshape(n_frames, self.T, self.H, self.d)
        return [Frame(start_frame + i, k[i], v[i]) for i in range(n_frames)]

    def _check_order(self, start_frame):
        if start_frame != self.committed:
            raise OrderError(f"start_frame {start_frame} != frames committed {self.committed}")

    def time_ids(self, frames, start_frame, n_frames):
        if self.rope_mode == self.ABSOLUTE:
            return rope.time_ids_absolute(frames)
        return rope.time_ids_relative(frames, start_frame, n_frames, self.window)

    # ------------------------------------------------------------ API
    def write_chunk(self, k_bits, v_bits, n_frames, start_frame):
        self._check_order(start_frame)
        self.cache.append(self._split_frames(k_bits, v_bits, n_frames, start_frame))
        self.committed += n_frames

    def window_frames(self, n_frames, start_frame):
        """Frame ids the chunk [start_frame, start_frame+n_frames) attends to, in logical order."""
        ids = [Frame(start_frame + i, None, None) for i in range(n_frames)]
        return [f.frame for f in self.cache.after_append(ids)]

    def chunk_attention(self, q_bits, k_bits, v_bits, n_frames, start_frame, commit,
                        rows=None, heads=None, rope_out_bf16=False):
        """fp64 attention output [len(rows), len(heads), d] for the chunk's queries.

        rope_out_bf16: round the rotated queries and keys to bf16 (nearest even) before the
        attention, as the pages' bf16 pipeline hands them over ([P2] §3: causal_rope_apply's
        bf16 output goes into attention(roped_query, k_cache, v_cache)); off by default (the
        rotation stays exact in fp64)."""
        self._check_order(start_frame)
        chunk = self._split_frames(k_bits, v_bits, n_frames, start_frame)
        window = self.cache.after_append(chunk)
        hs = list(range(self.H)) if heads is None else list(heads)

        k = np.concatenate([f.k for f in window], axis=0)[:, hs, :]
        v = np.concatenate([f.v for f in window], axis=0)[:, hs, :]
        if self.rope_mode == self.RELATIVE_SLOTS:
            k_ids = rope.time_ids_slot_order(len(window))
        else:
            k_ids = self.time_ids([f.frame for f in window], start_frame, n_frames)
        k_pos = rope.token_positions(k_ids, self.T, self.grid_w)
        k_rot = rope.rotate(bf16.to_f64(k), k_pos, self.theta, self.pairs)

        q = np.asarray(q_bits, dtype=np.uint16).reshape(n_frames * self.T, self.H, self.d)[:, hs, :]
        if self.rope_mode == self.RELATIVE_SLOTS:
            q_ids = k_ids[len(window) - n_frames:]  # the chunk is the window's last n_frames frames
        else:
            q_ids = self.time_ids([start_frame + i for i in range(n_frames)], start_frame, n_frames)
        q_pos = rope.token_positions(q_ids, self.T, self.grid_w)
        if rows is not None:
            rows = np.asarray(rows)
            q, q_pos = q[rows], q_pos[rows]
        q_rot = rope.rotate(bf16.to_f64(q), q_pos, self.theta, self.pairs)
        if rope_out_bf16:
            q_rot = bf16.to_f64(bf16.from_f64(q_rot))
            k_rot = bf16.to_f64(bf16.from_f64(k_rot))

        out = attend(q_rot, k_rot, bf16.to_f64(v))
        if commit:
            self.cache.slots = window
            self.committed += n_frames
        return out

    # ------------------------------------------------------------ cross-attention
    def set_text_kv(self, k_bits, v_bits):
        """The text context's K and V, [n_text, H, d] bf16 bits, computed once per prompt and
        kept for every later chunk ([P1] §核心答案 CrossAttention_KVCache; [P2] §3 cross-attn
        cache; [P4] §一次流式生成的完整链路 step 1, 512 text tokens). The self-attention
        cache is not touched."""
        k = np.asarray(k_bits, dtype=np.uint16)
        v = np.asarray(v_bits, dtype=np.uint16)
        assert k.shape == v.shape and k.ndim == 3 and k.shape[1:] == (self.H, self.d) and k.shape[0] > 0
        self.text_k, self.text_v = k.copy(), v.copy()

    def cross_attention(self, q_bits, rows=None, heads=None):
        """softmax(q K_text^T / sqrt(d)) V_text per head over all text tokens: no mask, no
        positions (so no RoPE); fp64 result [len(rows), len(heads), d]."""
        if getattr(self, "text_k", None) is None:
            raise StateError("no text K/V set")
        hs = list(range(self.H)) if heads is None else list(heads)
        q = np.asarray(q_bits, dtype=np.uint16).reshape(-1, self.H, self.d)[:, hs, :]
        if rows is not None:
            q = q[np.asarray(rows)]
        return attend(bf16.to_f64(q), bf16.to_f64(self.text_k[:, hs, :]), bf16.to_f64(self.text_v[:, hs, :]))

    def rope_apply(self, x_bits, n_frames, start_frame, window_end_frame=None):
        """RoPE of x [n_frames*T, H, d] as the standalone rotation call defines it: fp64 result.

        Absolute mode: t = frame index. Relative mode: t = clamp(f - (window_end_frame - window),
        0, window - 1), where window_end_frame is one past the last frame of the window.
        Slot-order mode: the frame's position in the window ending at window_end_frame, i.e.
        t = f for a sink frame (f < sink) and otherwise f minus the number of non-sink frames
        already evicted, max(0, window_end_frame - window); the result is then clamped to
        [0, window - 1] (which only bites for frames outside that window)."""
        frames = np.arange(start_frame, start_frame + n_frames)
        if self.rope_mode == self.ABSOLUTE:
            t = rope.time_ids_absolute(frames)
        elif self.rope_mode == self.RELATIVE_SLOTS:
            evicted = max(0, window_end_frame - self.window)
            t = np.clip(np.where(frames < self.sink, frames, frames - evicted), 0, self.window - 1)
        else:
            t = np.clip(frames - (window_end_frame - self.window), 0, self.window - 1)
        pos = rope.token_positions(t, self.T, self.grid_w)
        x = np.asarray(x_bits, dtype=np.uint16).reshape(n_frames * self.T, self.H, self.d)
        return rope.rotate(bf16.to_f64(x), pos, self.theta, self.pairs)

    # ------------------------------------------------------------ state read-back
    def logical_frames(self):
        return [f.frame for f in self.cache.slots]

    def logical_kv_bits(self):
        """Cache contents in logical order: ([n*T, H, d], [n*T, H, d]) uint16."""
        if not self.cache.slots:
            z = np.zeros((0, self.H, self.d), dtype=np.uint16)
            return z, z
        return (np.concatenate([f.k for f in self.cache.slots], axis=0),
                np.concatenate([f.v for f in self.cache.slots], axis=0))
