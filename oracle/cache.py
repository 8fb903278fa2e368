"""The rolling KV cache exactly as the pages describe it (oracle; test infrastructure only).

Physical order = logical order. The cache holds at most ``window`` frames
(``local_attn_size``); the first ``sink`` frames ever written are never evicted
(attention sink, ``sink_size``). When appending ``n`` frames would overflow,
the ``e`` oldest frames after the sinks are dropped, everything after them
shifts left by ``e`` positions, and the new frames go at the end:

* [P1] §滑动窗口 KV 缓存: overflow pushes the oldest tokens out and shifts the rest left;
  §Attention Sink: the first ``sink_size`` frames stay unchanged when rolling.
* [P2] §3 (KV 缓存 + 滚动窗口): when nearly full, the old KV after the sink is shifted
  left as a whole, overwriting the oldest part, then the new KV is appended.
* [P4] §机制一: cache size ``local_attn_size`` x tokens per frame; the oldest frame is
  popped ("roll"); the reference-view sinks at the front are never evicted.

Entries are opaque (whatever the caller stores per frame); this class only moves them.
"""
from __future__ import annotations

from typing import Any, List


class CapacityError(ValueError):
    """The appended frames cannot fit next to the sinks."""


class RollingCache:
    def __init__(self, window: int, sink: int):
        if window < 1 or sink < 0 or sink >= window:
            raise ValueError("need window >= 1 and 0 <= sink < window")
        self.window = window
        self.sink = sink
        self.slots: List[Any] = []  # physical order == logical order

    def after_append(self, entries: List[Any]) -> List[Any]:
        """The cache contents after appending ``entries`` (does not modify the cache)."""
        cur = list(self.slots)
        n = len(entries)
        if n > self.window - self.sink:
            raise CapacityError(f"{n} frames do not fit beside {self.sink} sinks in a window of {self.window}")
        if len(cur) + n <= self.window:
            return cur + list(entries)
        e = len(cur) + n - self.window           # frames to evict
        # positions [sink, sink+e) are evicted; [sink+e, filled) shift left; append at the end
        return cur[:self.sink] + cur[self.sink + e:] + list(entries)

    def append(self, entries: List[Any]) -> None:
        """Persist an append (a commit / write-back)."""
        self.slots = self.after_append(entries)

    def __len__(self) -> int:
        return len(self.slots)
