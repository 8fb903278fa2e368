"""Seeded synthetic inputs: one counter-based generator, two implementations.

This module serves both sides of the parity tests and the benchmark. It holds
none of the attention / RoPE / cache / sampler arithmetic: only the random
source that stands in for the activations a trained DiT would produce.

Definition (both implementations follow it to the bit):

* ``mix64`` is the SplitMix64 output function (Steele, Lea & Flood, "Fast
  splittable pseudorandom number generators", OOPSLA 2014; the finaliser is
  Stafford's "Mix13"), on unsigned 64-bit integers with wrap-around.
* Element ``n`` of the stream with 64-bit key ``K`` draws three words
  ``w_r = mix64(K + (3n + r + 1) * GOLDEN)`` for ``r = 0, 1, 2``.
* The twelve 16-bit lanes of ``w_0, w_1, w_2`` are summed (Irwin-Hall):
  ``s`` in ``[0, 12 * 65535]``.
* ``x = (s - 393210) / 65536`` is exact in fp32 (mean 0, variance ~1,
  bounded by +-6), then rounded to bf16 with round-to-nearest-even on the
  fp32 bit pattern.

The CUDA twin is ``synth_fill_normal_bf16`` in ``synth.cu`` (built into
``libsynth.so`` next to this file); a GPU test checks the two bit for bit.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

MASK64 = (1 << 64) - 1
GOLDEN = 0x9E3779B97F4A7C15
MUL1 = 0xBF58476D1CE4E5B9
MUL2 = 0x94D049BB133111EB
IRWIN_HALL_CENTRE = 393210  # 12 * 65535 / 2

# Tensor tags used in stream keys.
TAG = {"q": 1, "k": 2, "v": 3, "xt": 4, "eps": 5, "x": 6}


def mix64_int(z: int) -> int:
    """SplitMix64 output function on a Python int (mod 2**64)."""
    z &= MASK64
    z = ((z ^ (z >> 30)) * MUL1) & MASK64
    z = ((z ^ (z >> 27)) * MUL2) & MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, *fields: int) -> int:
    """64-bit key of one tensor stream: seed, then any number of integer fields
    (config id, layer, chunk, call, tensor tag, ...) folded in order."""
    k = mix64_int(seed * GOLDEN + 1)
    for f in fields:
        k = mix64_int(k ^ mix64_int(int(f) + GOLDEN))
    return k


def _mix64_np(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * np.uint64(MUL1)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(MUL2)
    return z ^ (z >> np.uint64(31))


def _bits_of(k: np.uint64, n: np.ndarray) -> np.ndarray:
    """bf16 bits of the elements with (uint64) indices n of the stream with key k."""
    g = np.uint64(GOLDEN)
    s = np.zeros(n.shape, dtype=np.int64)
    for r in range(3):
        w = _mix64_np(k + (np.uint64(3) * n + np.uint64(r + 1)) * g)
        for lane in range(4):
            s += ((w >> np.uint64(16 * lane)) & np.uint64(0xFFFF)).astype(np.int64)
    x = ((s - IRWIN_HALL_CENTRE).astype(np.float32) * np.float32(1.0 / 65536.0))
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return u.astype(np.uint16)


def normal_bf16_bits(key: int, start: int, count: int, block: int = 1 << 16) -> np.ndarray:
    """bf16 bit patterns (uint16) of elements ``start .. start+count-1`` of stream ``key``."""
    out = np.empty(count, dtype=np.uint16)
    k = np.uint64(key & MASK64)
    with np.errstate(over="ignore"):
        for b0 in range(0, count, block):
            n = np.arange(start + b0, start + min(count, b0 + block), dtype=np.uint64)
            out[b0:b0 + len(n)] = _bits_of(k, n)
    return out


def normal_bf16_bits_at(key: int, index, block: int = 1 << 16) -> np.ndarray:
    """bf16 bit patterns of the elements at the given indices (any shape) of stream ``key``."""
    idx = np.asarray(index, dtype=np.uint64)
    flat = idx.reshape(-1)
    out = np.empty(flat.shape, dtype=np.uint16)
    k = np.uint64(key & MASK64)
    with np.errstate(over="ignore"):
        for b0 in range(0, flat.size, block):
            out[b0:b0 + block] = _bits_of(k, flat[b0:b0 + block])
    return out.reshape(idx.shape)


# ---------------------------------------------------------------- CUDA twin
_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsynth.so")
        if not os.path.exists(path):
            raise RuntimeError(f"synth CUDA twin not built: {path} missing (run __graft_entry__.build())")
        lib = ctypes.CDLL(path)
        lib.synth_fill_normal_bf16.argtypes = [ctypes.c_void_p, ctypes.c_longlong,
                                               ctypes.c_ulonglong, ctypes.c_longlong,
                                               ctypes.c_void_p]
        lib.synth_fill_normal_bf16.restype = ctypes.c_int
        _LIB = lib
    return _LIB


def fill_normal_bf16_cuda(dev_ptr: int, count: int, key: int, start: int = 0, stream: int = 0) -> None:
    """Fill ``count`` bf16 values at device pointer ``dev_ptr`` with elements
    ``start ..`` of stream ``key`` (same bits as ``normal_bf16_bits``)."""
    rc = _lib().synth_fill_normal_bf16(ctypes.c_void_p(dev_ptr), count, key & MASK64, start,
                                        ctypes.c_void_p(stream))
    if rc != 0:
        raise RuntimeError(f"synth_fill_normal_bf16 failed with CUDA error {rc}")
