"""Plain fp64 CPU oracle of the rolling-window chunk attention path.

TEST INFRASTRUCTURE ONLY. Nothing in the product (the ``rolling_kv_chunked_b200``
package, its C-ABI library or its kernels) imports, links or calls this
package; only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline``
/ ``--impl reference`` legs of ``bench.py`` may. It shares no code with the
CUDA path: the only module both sides use is ``synth`` (seeded inputs).

What it computes, in the pages' order and notation, slow and obviously:

* ``bf16``      exact bf16 <-> fp64 conversion (round-to-nearest-even by definition).
* ``cache``     the literal shift-left rolling KV cache with never-evicted sinks.
* ``rope``      3D RoPE (t, h, w axes), absolute or relative (re-based, clamped) time ids.
* ``attention`` softmax(Q K^T / sqrt(d)) V over the visible window, per head, fp64.
* ``flow``      flow-matching x0 = xt - sigma * v and the renoise to the next sigma, fp64.
* ``layer``     one layer's state machine tying the four together (reads vs commits), and
                the cross-attention over the cached text K/V (no positions, no mask).

Pages cited (by title and section):

[P1] "LingBot-World 2.0因果预训练范式深度剖析：为什么它能持续生成视频而不“掉画质”"
     (sheratonhq.com/news/156439)
[P2] "从40步到4步：LingBot-World 2.0实时推理蒸馏（causal_fast）原理与关键代码解读"
     (hmyw.cn/news/135683)
[P3] LingBot-World 2.0 ``wan/`` source-map article (kwkr.cn/news/564388)
[P4] "ABot-World流式因果推理深度解析：KV缓存与块级注意力如何让24小时连续生成不漂移"
     (lpnh.cn/news/2488095)
[P5] "无限生成的秘密：ABot-World如何用Causal Forcing与LongForcing蒸馏实现无限世界推演"
     (nxmr.cn/news/121609)

Every function is pinned by a ``-m "not gpu"`` test against something other
than itself (closed forms, brute force, invariants, hand-worked fixtures under
``tests/golden``); none is "parity unpinned".
"""
from . import bf16, cache, rope, attention, flow, layer  # noqa: F401
