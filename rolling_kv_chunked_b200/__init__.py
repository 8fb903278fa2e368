"""Python binding of librkv.so (rolling-window chunk attention for B200).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels. Tensors are torch CUDA tensors (bf16, contiguous); PyTorch provides
device memory and streams. The C ABI is declared in include/rkv.h; the names
here are the C names without the ``rkv_`` prefix.

The library must be built (``python rolling_kv_chunked_b200/build.py``); if it
is missing, importing this package raises.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librkv.so")

OK = 0
ERR_ARG = 1
ERR_ORDER = 2
ERR_CAPACITY = 3
ERR_UNSUPPORTED = 4
ERR_CUDA = 5
ERR_TIMEOUT = 6
ERR_STATE = 7

ROPE_ABSOLUTE = 0
ROPE_RELATIVE = 1
ROPE_RELATIVE_SLOTS = 2

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built; run `python rolling_kv_chunked_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)

_c_int, _c_ll, _c_dbl, _vp = ctypes.c_int, ctypes.c_longlong, ctypes.c_double, ctypes.c_void_p
_int_p = ctypes.POINTER(ctypes.c_int)


class FlowEpilogue(ctypes.Structure):
    """Mirror of ``rkv_flow_epilogue``."""
    _fields_ = [("xt", _vp), ("eps", _vp), ("sigma", _c_dbl), ("sigma_next", _c_dbl),
                ("x0_out", _vp), ("xt_next_out", _vp)]


class HeadCopy(ctypes.Structure):
    """Mirror of ``rkv_head_copy``: n_tok tokens x n_heads head vectors, strides in elements."""
    _fields_ = [("src", _vp), ("dst", _vp), ("src_tok_stride", _c_ll), ("src_head_stride", _c_ll),
                ("dst_tok_stride", _c_ll), ("dst_head_stride", _c_ll), ("n_tok", _c_int)]


_SIGS = {
    "rkv_create": ([_c_int] * 7 + [ctypes.POINTER(_vp)], _c_int),
    "rkv_set_rope_grid": ([_vp, _c_int, _c_int, _c_dbl, _c_int, _c_int, _c_int], _c_int),
    "rkv_write_chunk": ([_vp, _c_int, _vp, _vp, _c_int, _c_int, _vp], _c_int),
    "rkv_chunk_attention": ([_vp, _c_int, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _vp], _c_int),
    "rkv_chunk_attention_flow": ([_vp, _c_int, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int,
                                  ctypes.POINTER(FlowEpilogue), _vp], _c_int),
    "rkv_chunk_attention_cfg_flow": ([_vp, _c_int, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int,
                                      ctypes.POINTER(FlowEpilogue), _vp, _c_dbl, _vp], _c_int),
    "rkv_set_text_kv": ([_vp, _c_int, _vp, _vp, _c_int, _vp], _c_int),
    "rkv_cross_attention": ([_vp, _c_int, _vp, _vp, _c_int, _vp], _c_int),
    "rkv_rope_apply": ([_vp, _vp, _c_int, _c_int, _c_int, _vp], _c_int),
    "rkv_flow_x0_renoise": ([_vp, _vp, _vp, _c_dbl, _c_dbl, _vp, _vp, _c_ll, _vp], _c_int),
    "rkv_flow_cfg_x0_renoise": ([_vp, _vp, _vp, _vp, _c_dbl, _c_dbl, _c_dbl, _vp, _vp, _c_ll, _vp], _c_int),
    "rkv_slot_frames": ([_vp, _c_int, _int_p], _c_int),
    "rkv_frames_committed": ([_vp, _c_int, _int_p], _c_int),
    "rkv_cache_ptrs": ([_vp, _c_int, ctypes.POINTER(_vp), ctypes.POINTER(_vp)], _c_int),
    "rkv_reset": ([_vp], _c_int),
    "rkv_destroy": ([_vp], _c_int),
    "rkv_status_string": ([_c_int], ctypes.c_char_p),
    "rkv_poll_device_status": ([_vp, _vp], _c_int),
    "rkv_set_wait_limit": ([_vp, _c_ll], _c_int),
    "rkv_chunk_attention_noalloc": ([_vp, _vp, _vp, _vp] + [_c_int] * 8 + [_int_p, _c_int, _vp], _c_int),
    "rkv_timing_begin": ([_vp, _c_int], _c_int),
    "rkv_timing_end": ([_vp, ctypes.POINTER(ctypes.c_float), _c_int, _int_p], _c_int),
    "rkv_plan_window": ([_c_int, _c_int, _c_int, _c_int, _c_int, _int_p, _c_int, _int_p], _c_int),
    "rkv_copy_heads": ([ctypes.POINTER(HeadCopy), _c_int, _c_int, _vp], _c_int),
}
for _name, (_args, _res) in _SIGS.items():
    try:
        _fn = getattr(_lib, _name)
    except AttributeError as _e:
        raise ImportError(f"{LIB_PATH} does not export {_name}; rebuild it") from _e
    _fn.argtypes = _args
    _fn.restype = _res

EXPORTED = tuple(_SIGS)


class RkvError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} (code {code})")


def status_string(code: int) -> str:
    return _lib.rkv_status_string(code).decode()


def _check(code: int, where: str) -> None:
    if code != OK:
        raise RkvError(code, where)


def _ptr(t):
    """Device pointer of a torch tensor (or an int / None)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def plan_window(window_frames: int, sink_frames: int, frames_committed: int, n_frames: int, start_frame: int):
    """Host-only: the key segments chunk [start_frame, start_frame+n_frames) attends to."""
    buf = (ctypes.c_int * 16)()
    n = ctypes.c_int(0)
    _check(_lib.rkv_plan_window(window_frames, sink_frames, frames_committed, n_frames, start_frame,
                                buf, 4, ctypes.byref(n)), "rkv_plan_window")
    return [tuple(buf[4 * i:4 * i + 4]) for i in range(n.value)]


def flow_x0_renoise(xt, v, eps, sigma: float, sigma_next: float, x0_out, xt_next_out=None, stream=None) -> None:
    """x0 = xt - sigma v; xt_next = (1 - sigma') x0 + sigma' eps (sigma' < 0: last step)."""
    _check(_lib.rkv_flow_x0_renoise(_ptr(xt), _ptr(v), _ptr(eps), float(sigma), float(sigma_next),
                                    _ptr(x0_out), _ptr(xt_next_out), xt.numel(), _stream(stream)),
           "rkv_flow_x0_renoise")


def copy_heads(runs, n_heads: int, stream=None) -> None:
    """Strided head-vector copies. ``runs``: (src_ptr, dst_ptr, src_tok_stride, src_head_stride,
    dst_tok_stride, dst_head_stride, n_tok) tuples, pointers as ints, strides in elements."""
    arr = (HeadCopy * max(1, len(runs)))()
    for i, r in enumerate(runs):
        arr[i] = HeadCopy(*r)
    _check(_lib.rkv_copy_heads(arr, len(runs), int(n_heads), _stream(stream)), "rkv_copy_heads")


def flow_cfg_x0_renoise(xt, v_cond, v_uncond, eps, cfg_scale: float, sigma: float, sigma_next: float, x0_out,
                        xt_next_out=None, stream=None) -> None:
    """v = v_uncond + cfg_scale (v_cond - v_uncond), then the x0 / renoise step of flow_x0_renoise."""
    _check(_lib.rkv_flow_cfg_x0_renoise(_ptr(xt), _ptr(v_cond), _ptr(v_uncond), _ptr(eps), float(cfg_scale),
                                        float(sigma), float(sigma_next), _ptr(x0_out), _ptr(xt_next_out),
                                        xt.numel(), _stream(stream)), "rkv_flow_cfg_x0_renoise")


class RollingKV:
    """One rkv handle: per-layer rolling caches plus the RoPE configuration."""

    def __init__(self, layers: int, H: int, d: int, tokens_per_frame: int, window_frames: int,
                 sink_frames: int, rope_mode: int):
        h = _vp()
        _check(_lib.rkv_create(layers, H, d, tokens_per_frame, window_frames, sink_frames, rope_mode,
                               ctypes.byref(h)), "rkv_create")
        self._h = h
        self.layers, self.H, self.d, self.T = layers, H, d, tokens_per_frame
        self.window_frames, self.sink_frames, self.rope_mode = window_frames, sink_frames, rope_mode

    # ------------------------------------------------------------------ config
    def set_rope_grid(self, grid_h: int, grid_w: int, theta: float = 1.0e4, pairs=(22, 21, 21)) -> None:
        _check(_lib.rkv_set_rope_grid(self._h, grid_h, grid_w, float(theta), *pairs), "rkv_set_rope_grid")

    def set_wait_limit(self, nanoseconds: int) -> None:
        _check(_lib.rkv_set_wait_limit(self._h, int(nanoseconds)), "rkv_set_wait_limit")

    # ------------------------------------------------------------------ hot path
    def write_chunk(self, layer: int, k, v, n_frames: int, start_frame: int, stream=None) -> None:
        _check(_lib.rkv_write_chunk(self._h, layer, _ptr(k), _ptr(v), n_frames, start_frame, _stream(stream)),
               "rkv_write_chunk")

    def chunk_attention(self, layer: int, q, k, v, out, n_frames: int, start_frame: int, commit: bool,
                        stream=None, flow: dict | None = None) -> None:
        """out = attention of the chunk's queries; ``flow`` = dict(xt, eps, sigma, sigma_next, x0_out,
        xt_next_out) fuses the x0/renoise epilogue into the output store. With ``v_cond`` and
        ``cfg_scale`` in ``flow`` this call is the unconditional branch of a guided step: the epilogue
        uses v = out + cfg_scale (v_cond - out)."""
        if flow is None:
            rc = _lib.rkv_chunk_attention(self._h, layer, _ptr(q), _ptr(k), _ptr(v), _ptr(out), n_frames,
                                          start_frame, int(bool(commit)), _stream(stream))
            _check(rc, "rkv_chunk_attention")
            return
        epi = FlowEpilogue(_ptr(flow["xt"]), _ptr(flow.get("eps")), float(flow["sigma"]),
                           float(flow["sigma_next"]), _ptr(flow["x0_out"]), _ptr(flow.get("xt_next_out")))
        if flow.get("v_cond") is not None:
            rc = _lib.rkv_chunk_attention_cfg_flow(self._h, layer, _ptr(q), _ptr(k), _ptr(v), _ptr(out), n_frames,
                                                   start_frame, int(bool(commit)), ctypes.byref(epi),
                                                   _ptr(flow["v_cond"]), float(flow["cfg_scale"]), _stream(stream))
            _check(rc, "rkv_chunk_attention_cfg_flow")
            return
        rc = _lib.rkv_chunk_attention_flow(self._h, layer, _ptr(q), _ptr(k), _ptr(v), _ptr(out), n_frames,
                                           start_frame, int(bool(commit)), ctypes.byref(epi), _stream(stream))
        _check(rc, "rkv_chunk_attention_flow")

    def set_text_kv(self, layer: int, k_text, v_text, stream=None) -> None:
        """Cache the text context's K and V ([n_text, H, d] each) for cross-attention."""
        _check(_lib.rkv_set_text_kv(self._h, layer, _ptr(k_text), _ptr(v_text), k_text.shape[0], _stream(stream)),
               "rkv_set_text_kv")

    def cross_attention(self, layer: int, q, out, stream=None) -> None:
        """out = softmax(q K_text^T / sqrt(d)) V_text over the cached text tokens; q, out [n, H, d]."""
        _check(_lib.rkv_cross_attention(self._h, layer, _ptr(q), _ptr(out), q.shape[0], _stream(stream)),
               "rkv_cross_attention")

    def rope_apply(self, x, n_frames: int, start_frame: int, window_end_frame: int = 0, stream=None) -> None:
        _check(_lib.rkv_rope_apply(self._h, _ptr(x), n_frames, start_frame, window_end_frame, _stream(stream)),
               "rkv_rope_apply")

    # ------------------------------------------------------------------ state
    def slot_frames(self, layer: int):
        buf = (ctypes.c_int * self.window_frames)()
        _check(_lib.rkv_slot_frames(self._h, layer, buf), "rkv_slot_frames")
        return list(buf)

    def frames_committed(self, layer: int) -> int:
        n = ctypes.c_int(0)
        _check(_lib.rkv_frames_committed(self._h, layer, ctypes.byref(n)), "rkv_frames_committed")
        return n.value

    def cache_ptrs(self, layer: int):
        k, v = _vp(), _vp()
        _check(_lib.rkv_cache_ptrs(self._h, layer, ctypes.byref(k), ctypes.byref(v)), "rkv_cache_ptrs")
        return k.value, v.value

    def timing_begin(self, max_launches: int) -> None:
        """Record CUDA events around each attention kernel launch (instrumentation only)."""
        _check(_lib.rkv_timing_begin(self._h, int(max_launches)), "rkv_timing_begin")

    def timing_end(self, max_launches: int = 4096):
        """Synchronise and return the recorded attention launch durations in ms."""
        buf = (ctypes.c_float * max_launches)()
        n = ctypes.c_int(0)
        _check(_lib.rkv_timing_end(self._h, buf, max_launches, ctypes.byref(n)), "rkv_timing_end")
        return list(buf[:n.value])

    def poll_device_status(self, stream=None) -> int:
        """Synchronise the stream and return (and clear) the device status: OK or ERR_TIMEOUT."""
        return _lib.rkv_poll_device_status(self._h, _stream(stream))

    def reset(self) -> None:
        _check(_lib.rkv_reset(self._h), "rkv_reset")

    def close(self) -> None:
        if getattr(self, "_h", None):
            _lib.rkv_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
