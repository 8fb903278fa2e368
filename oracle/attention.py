"""Chunk attention over a visible key set, fp64 (oracle; test infrastructure only).

O = softmax(Q K^T / sqrt(d)) V per head, no mask inside the visible set: the
chunk's queries see every key of the window, which is the current chunk plus
the cached history and sinks ([P2] §3: the window slice
``kv_cache[:, max(0, local_end_index - max_attention_size):local_end_index]``
followed by ``attention(roped_query, k_cache, v_cache)``; [P4] §机制二: a new
block's queries see their own block and the history blocks in the window,
frames inside a block see each other). Scale 1/sqrt(d); no dropout.
"""
from __future__ import annotations

import numpy as np


def attend(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """q [Lq, H, d], k [Lk, H, d], v [Lk, H, d] (fp64) -> O [Lq, H, d] fp64."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    Lq, H, d = q.shape
    out = np.empty((Lq, H, v.shape[2]), dtype=np.float64)
    scale = 1.0 / np.sqrt(d)
    for h in range(H):
        s = (q[:, h, :] @ k[:, h, :].T) * scale            # [Lq, Lk]
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=1, keepdims=True)
        out[:, h, :] = p @ v[:, h, :]
    return out
