"""Planted mistakes in the oracle, for checking that its pins catch them (CPU only).

Loaded as a pytest plugin (``-p oracle_mutants``) by ``test_oracle_mutants.py``: when the
environment names a mutant (``RKV_ORACLE_MUTANT``), the plugin replaces one oracle function
with a copy that carries one plausible mistake (a dropped term, a wrong sign, index or axis,
a transposed operand, an off-by-one), before any test module imports the oracle. The pins
(``test_oracle_*.py``) then run against the mutated oracle and at least one must fail.
Nothing here is used by the product or by the unmutated test run.
"""
from __future__ import annotations

import os

import numpy as np

import oracle
from oracle import attention, bf16, cache, flow, layer, rope


def _rebind(module_attr_pairs, new):
    for mod, name in module_attr_pairs:
        setattr(mod, name, new)


# ------------------------------------------------------------------ attention
def _attend_with(scale_fn=None, axis=1, use_k_as_v=False, normalise=True):
    def attend(q, k, v):
        q = np.asarray(q, dtype=np.float64)
        k = np.asarray(k, dtype=np.float64)
        v = np.asarray(v, dtype=np.float64)
        Lq, H, d = q.shape
        out = np.empty((Lq, H, v.shape[2]), dtype=np.float64)
        scale = 1.0 / np.sqrt(d) if scale_fn is None else scale_fn(d)
        for h in range(H):
            s = (q[:, h, :] @ k[:, h, :].T) * scale
            s = s - s.max(axis=axis, keepdims=True)
            p = np.exp(s)
            if normalise:
                p = p / p.sum(axis=axis, keepdims=True)
            out[:, h, :] = p @ (k if use_k_as_v else v)[:, h, :]
        return out
    return attend


def _patch_attend(fn):
    _rebind([(attention, "attend"), (layer, "attend")], fn)


# ------------------------------------------------------------------ rope
def _rotate_with(sign=1.0, halves=False):
    def rotate(x, pos, theta=rope.DEFAULT_THETA, pairs=rope.DEFAULT_PAIRS):
        x = np.asarray(x, dtype=np.float64)
        axis, _, _ = rope.pair_table(pairs)
        ang = pos[:, axis].astype(np.float64) * rope.omegas(theta, pairs)[None, :]
        c = np.cos(ang)[:, None, :]
        s = sign * np.sin(ang)[:, None, :]
        half = x.shape[-1] // 2
        a = x[..., :half] if halves else x[..., 0::2]
        b = x[..., half:] if halves else x[..., 1::2]
        out = np.empty_like(x)
        if halves:
            out[..., :half] = a * c - b * s
            out[..., half:] = a * s + b * c
        else:
            out[..., 0::2] = a * c - b * s
            out[..., 1::2] = a * s + b * c
        return out
    return rotate


def _pair_table_axes_shifted(pairs=rope.DEFAULT_PAIRS):
    axis, loc, cnt = [], [], []
    for a, n in enumerate(pairs):
        for j in range(n):
            axis.append((a + 1) % 3)   # h, w, t instead of t, h, w
            loc.append(j)
            cnt.append(n)
    return np.array(axis), np.array(loc, dtype=np.float64), np.array(cnt, dtype=np.float64)


def _omegas_with(two_j=False, global_ladder=False):
    def omegas(theta=rope.DEFAULT_THETA, pairs=rope.DEFAULT_PAIRS):
        _, j, n = rope.pair_table(pairs)
        if global_ladder:
            return np.power(float(theta), -np.arange(len(j), dtype=np.float64) / len(j))
        return np.power(float(theta), -(2.0 if two_j else 1.0) * j / n)
    return omegas


def _token_positions_transposed(frame_time_ids, tokens_per_frame, grid_w):
    t_ids = np.asarray(frame_time_ids, dtype=np.int64)
    tok = np.arange(tokens_per_frame, dtype=np.int64)
    grid_h = tokens_per_frame // grid_w
    pos = np.empty((len(t_ids) * tokens_per_frame, 3), dtype=np.int64)
    pos[:, 0] = np.repeat(t_ids, tokens_per_frame)
    pos[:, 1] = np.tile(tok % grid_h, len(t_ids))      # column-major walk of the grid
    pos[:, 2] = np.tile(tok // grid_h, len(t_ids))
    return pos


def _time_ids_relative_with(clamp=True, shift=0):
    def time_ids_relative(frames, start_frame, n_frames, window):
        base = start_frame + n_frames - window + shift
        t = np.asarray(frames, dtype=np.int64) - base
        return np.clip(t, 0, window - 1) if clamp else t
    return time_ids_relative


# ------------------------------------------------------------------ cache
def _after_append_with(kind):
    def after_append(self, entries):
        cur = list(self.slots)
        n = len(entries)
        if n > self.window - self.sink:
            raise cache.CapacityError("does not fit")
        if len(cur) + n <= self.window:
            return cur + list(entries)
        e = len(cur) + n - self.window
        if kind == "sinks_evicted":
            return cur[e:] + list(entries)
        if kind == "newest_evicted":
            return cur[:len(cur) - e] + list(entries)
        if kind == "one_extra":
            return cur[:self.sink] + cur[self.sink + e + 1:] + list(entries)
        raise AssertionError(kind)
    return after_append


# ------------------------------------------------------------------ layer
def _chunk_attention_with(kind):
    orig = layer.OracleLayer.chunk_attention

    def chunk_attention(self, q_bits, k_bits, v_bits, n_frames, start_frame, commit, rows=None, heads=None):
        if kind == "reads_persist":
            return orig(self, q_bits, k_bits, v_bits, n_frames, start_frame, True, rows, heads)
        if kind == "slots_as_clamped":
            saved = self.rope_mode
            if saved == self.RELATIVE_SLOTS:
                self.rope_mode = self.RELATIVE
            try:
                return orig(self, q_bits, k_bits, v_bits, n_frames, start_frame, commit, rows, heads)
            finally:
                self.rope_mode = saved
        raise AssertionError(kind)
    return chunk_attention


def _time_ids_query_from_window_start():
    orig = layer.OracleLayer.time_ids

    def time_ids(self, frames, start_frame, n_frames):
        t = orig(self, frames, start_frame, n_frames)
        if self.rope_mode == self.ABSOLUTE and len(frames) == n_frames and list(frames)[0] == start_frame:
            return t - start_frame     # the chunk's queries get ids 0.. instead of their frame ids
        return t
    return time_ids


def _rope_apply_window_end_off_by_one(modes):
    orig = layer.OracleLayer.rope_apply

    def rope_apply(self, x_bits, n_frames, start_frame, window_end_frame=None):
        if self.rope_mode not in modes:
            return orig(self, x_bits, n_frames, start_frame, window_end_frame)
        return orig(self, x_bits, n_frames, start_frame, None if window_end_frame is None else window_end_frame + 1)
    return rope_apply


def _cross_drop_last_token():
    orig = layer.OracleLayer.cross_attention

    def cross_attention(self, q_bits, rows=None, heads=None):
        if getattr(self, "text_k", None) is None:
            return orig(self, q_bits, rows, heads)
        full_k, full_v = self.text_k, self.text_v
        if full_k.shape[0] > 1:
            self.text_k, self.text_v = full_k[:-1], full_v[:-1]
        try:
            return orig(self, q_bits, rows, heads)
        finally:
            self.text_k, self.text_v = full_k, full_v
    return cross_attention


def _cross_with_positions():
    orig = layer.OracleLayer.cross_attention

    def cross_attention(self, q_bits, rows=None, heads=None):
        out = orig(self, q_bits, rows, heads)
        # as if the text keys had been rotated by their index on the time axis
        k_bits = self.text_k
        pos = np.zeros((k_bits.shape[0], 3), dtype=np.int64)
        pos[:, 0] = np.arange(k_bits.shape[0])
        hs = list(range(self.H)) if heads is None else list(heads)
        q = np.asarray(q_bits, dtype=np.uint16).reshape(-1, self.H, self.d)[:, hs, :]
        if rows is not None:
            q = q[np.asarray(rows)]
        k_rot = rope.rotate(bf16.to_f64(k_bits[:, hs, :]), pos, self.theta, self.pairs)
        out[...] = attention.attend(bf16.to_f64(q), k_rot, bf16.to_f64(self.text_v[:, hs, :]))
        return out
    return cross_attention


def _chunk_attention_rotating_v():
    """The layer's attention with V rotated by the keys' positions, like K."""
    def chunk_attention(self, q_bits, k_bits, v_bits, n_frames, start_frame, commit, rows=None, heads=None,
                        rope_out_bf16=False):
        self._check_order(start_frame)
        chunk = self._split_frames(k_bits, v_bits, n_frames, start_frame)
        window = self.cache.after_append(chunk)
        hs = list(range(self.H)) if heads is None else list(heads)
        k = np.concatenate([f.k for f in window], axis=0)[:, hs, :]
        v = np.concatenate([f.v for f in window], axis=0)[:, hs, :]
        if self.rope_mode == self.RELATIVE_SLOTS:
            k_ids = rope.time_ids_slot_order(len(window))
            q_ids = k_ids[len(window) - n_frames:]
        else:
            k_ids = self.time_ids([f.frame for f in window], start_frame, n_frames)
            q_ids = self.time_ids([start_frame + i for i in range(n_frames)], start_frame, n_frames)
        k_pos = rope.token_positions(k_ids, self.T, self.grid_w)
        k_rot = rope.rotate(bf16.to_f64(k), k_pos, self.theta, self.pairs)
        v_rot = rope.rotate(bf16.to_f64(v), k_pos, self.theta, self.pairs)
        q = np.asarray(q_bits, dtype=np.uint16).reshape(n_frames * self.T, self.H, self.d)[:, hs, :]
        q_pos = rope.token_positions(q_ids, self.T, self.grid_w)
        if rows is not None:
            q, q_pos = q[np.asarray(rows)], q_pos[np.asarray(rows)]
        out = attention.attend(rope.rotate(bf16.to_f64(q), q_pos, self.theta, self.pairs), k_rot, v_rot)
        if commit:
            self.cache.slots = window
            self.committed += n_frames
        return out
    return chunk_attention


def _chunk_attention_ignoring_rope_out_bf16():
    orig = layer.OracleLayer.chunk_attention

    def chunk_attention(self, q_bits, k_bits, v_bits, n_frames, start_frame, commit, rows=None, heads=None,
                        rope_out_bf16=False):
        return orig(self, q_bits, k_bits, v_bits, n_frames, start_frame, commit, rows, heads)
    return chunk_attention


def _slot_query_ids_from_window_start():
    orig = rope.time_ids_slot_order

    def time_ids_slot_order(n_visible):
        ids = orig(n_visible)
        return ids[::-1].copy()     # ids counted from the other end of the window
    return time_ids_slot_order


# ------------------------------------------------------------------ flow
def _x0_renoise_with(kind):
    def x0_renoise_f64(xt, v, eps, sigma, sigma_next):
        xt = np.asarray(xt, dtype=np.float64)
        v = np.asarray(v, dtype=np.float64)
        x0 = xt + sigma * v if kind == "x0_plus" else xt - sigma * v
        if sigma_next < 0:
            return x0, None
        eps = np.asarray(eps, dtype=np.float64)
        if kind == "renoise_swapped":
            return x0, sigma_next * x0 + (1.0 - sigma_next) * eps
        if kind == "renoise_from_xt":
            return x0, (1.0 - sigma_next) * xt + sigma_next * eps
        return x0, (1.0 - sigma_next) * x0 + sigma_next * eps
    return x0_renoise_f64


def _cfg_with(kind):
    def cfg_combine_f64(v_cond, v_uncond, scale):
        c = np.asarray(v_cond, dtype=np.float64)
        u = np.asarray(v_uncond, dtype=np.float64)
        if kind == "swapped":
            return c + scale * (u - c)
        if kind == "scale_on_u":
            return scale * u + (c - u)
        return scale * (c - u)
    return cfg_combine_f64


def _x0_renoise_sigma_for_next():
    def x0_renoise_f64(xt, v, eps, sigma, sigma_next):
        xt = np.asarray(xt, dtype=np.float64)
        v = np.asarray(v, dtype=np.float64)
        x0 = xt - sigma * v
        if sigma_next < 0:
            return x0, None
        eps = np.asarray(eps, dtype=np.float64)
        return x0, (1.0 - sigma) * x0 + sigma * eps     # renoised to the current sigma
    return x0_renoise_f64


# ------------------------------------------------------------------ bf16
def _from_f64_with(kind):
    orig = bf16.from_f64

    def from_f64(x):
        x = np.asarray(x, dtype=np.float64)
        if not np.all(np.isfinite(x)):
            raise ValueError("bf16 rounding of a non-finite value")
        if kind == "saturate":
            y = orig(np.clip(x, -bf16._MAX_FINITE, bf16._MAX_FINITE))
            return y
        m, e = np.frexp(x)
        r = np.ldexp(m, 8)
        if kind == "truncate":
            q = np.trunc(r)
        elif kind == "ties_away":
            q = np.sign(r) * np.floor(np.abs(r) + 0.5)
        elif kind == "no_subnormal_grid":
            q = np.rint(r)
        else:
            raise AssertionError(kind)
        y = np.ldexp(q, e - 8)
        if kind != "no_subnormal_grid":
            small = np.abs(x) < bf16._MIN_NORMAL
            if np.any(small):
                y = np.where(small, np.rint(x / bf16._SUBNORMAL_ULP) * bf16._SUBNORMAL_ULP, y)
        y = np.where(np.abs(y) > bf16._MAX_FINITE, np.copysign(np.inf, y), y)
        return (y.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    return from_f64


def _patch_from_f64(fn):
    _rebind([(bf16, "from_f64")], fn)


MUTANTS = {
    # attention
    "attend_no_scale": lambda: _patch_attend(_attend_with(scale_fn=lambda d: 1.0)),
    "attend_scale_1_over_d": lambda: _patch_attend(_attend_with(scale_fn=lambda d: 1.0 / d)),
    "attend_softmax_over_queries": lambda: _patch_attend(_attend_with(axis=0)),
    "attend_values_are_keys": lambda: _patch_attend(_attend_with(use_k_as_v=True)),
    "attend_unnormalised": lambda: _patch_attend(_attend_with(normalise=False)),
    # rope
    "rope_reverse_rotation": lambda: _rebind([(rope, "rotate")], _rotate_with(sign=-1.0)),
    "rope_half_split_pairs": lambda: _rebind([(rope, "rotate")], _rotate_with(halves=True)),
    "rope_axis_order_hwt": lambda: _rebind([(rope, "pair_table")], _pair_table_axes_shifted),
    "rope_frequency_2j": lambda: _rebind([(rope, "omegas")], _omegas_with(two_j=True)),
    "rope_single_ladder": lambda: _rebind([(rope, "omegas")], _omegas_with(global_ladder=True)),
    "rope_grid_transposed": lambda: _rebind([(rope, "token_positions")], _token_positions_transposed),
    "rope_relative_unclamped": lambda: _rebind([(rope, "time_ids_relative")], _time_ids_relative_with(clamp=False)),
    "rope_relative_base_off_by_one": lambda: _rebind([(rope, "time_ids_relative")], _time_ids_relative_with(shift=1)),
    # cache
    "cache_sinks_evicted": lambda: setattr(cache.RollingCache, "after_append", _after_append_with("sinks_evicted")),
    "cache_newest_evicted": lambda: setattr(cache.RollingCache, "after_append", _after_append_with("newest_evicted")),
    "cache_evicts_one_extra": lambda: setattr(cache.RollingCache, "after_append", _after_append_with("one_extra")),
    # layer
    "layer_reads_persist": lambda: setattr(layer.OracleLayer, "chunk_attention", _chunk_attention_with("reads_persist")),
    "layer_slots_as_clamped": lambda: setattr(layer.OracleLayer, "chunk_attention", _chunk_attention_with("slots_as_clamped")),
    "layer_query_ids_from_zero": lambda: setattr(layer.OracleLayer, "time_ids", _time_ids_query_from_window_start()),
    "layer_rope_apply_relative_window_end_off_by_one": lambda: setattr(
        layer.OracleLayer, "rope_apply", _rope_apply_window_end_off_by_one((layer.OracleLayer.RELATIVE,))),
    "layer_rope_apply_slots_window_end_off_by_one": lambda: setattr(
        layer.OracleLayer, "rope_apply", _rope_apply_window_end_off_by_one((layer.OracleLayer.RELATIVE_SLOTS,))),
    "cross_drops_last_text_token": lambda: setattr(layer.OracleLayer, "cross_attention", _cross_drop_last_token()),
    "cross_rotates_text_keys": lambda: setattr(layer.OracleLayer, "cross_attention", _cross_with_positions()),
    # flow
    "flow_x0_sign": lambda: _rebind([(flow, "x0_renoise_f64")], _x0_renoise_with("x0_plus")),
    "flow_renoise_weights_swapped": lambda: _rebind([(flow, "x0_renoise_f64")], _x0_renoise_with("renoise_swapped")),
    "flow_renoise_from_xt": lambda: _rebind([(flow, "x0_renoise_f64")], _x0_renoise_with("renoise_from_xt")),
    "cfg_branches_swapped": lambda: _rebind([(flow, "cfg_combine_f64")], _cfg_with("swapped")),
    "cfg_missing_base": lambda: _rebind([(flow, "cfg_combine_f64")], _cfg_with("no_base")),
    "cfg_scale_on_u": lambda: _rebind([(flow, "cfg_combine_f64")], _cfg_with("scale_on_u")),
    "flow_renoise_to_current_sigma": lambda: _rebind([(flow, "x0_renoise_f64")], _x0_renoise_sigma_for_next()),
    "layer_values_rotated_like_keys": lambda: setattr(layer.OracleLayer, "chunk_attention", _chunk_attention_rotating_v()),
    "layer_ignores_rope_out_bf16": lambda: setattr(layer.OracleLayer, "chunk_attention",
                                                   _chunk_attention_ignoring_rope_out_bf16()),
    "rope_slot_ids_reversed": lambda: _rebind([(rope, "time_ids_slot_order")], _slot_query_ids_from_window_start()),
    # bf16
    "bf16_truncates": lambda: _patch_from_f64(_from_f64_with("truncate")),
    "bf16_ties_away": lambda: _patch_from_f64(_from_f64_with("ties_away")),
    "bf16_no_subnormal_grid": lambda: _patch_from_f64(_from_f64_with("no_subnormal_grid")),
    "bf16_saturates": lambda: _patch_from_f64(_from_f64_with("saturate")),
}

_name = os.environ.get("RKV_ORACLE_MUTANT")
if _name:
    MUTANTS[_name]()
    assert oracle is not None
