"""GPU test of rkv_chunk_attention_noalloc, the entry point for callers that may not
allocate device memory (their host framework's allocator must own every byte, or
allocation is forbidden once the process is running): it keeps its scratch in a fixed
static device array instead of allocating.

The window it attends to is built from the fp64 oracle's own cache state (the oracle
rolled through warm-up, eviction and wrap on the seeded inputs), so the inputs do not
come from the CUDA path. It is called through the C ABI twice in a row, and both results
must match the oracle within the attention tolerance of the other tests, and match the
output of the handle path (rkv_chunk_attention on a handle rolled with the same inputs)
within the same tolerance. Argument and size errors must return before anything is
launched: the output buffer keeps its sentinel bytes.
This file is named to be collected last; it depends on no other test.
"""
import ctypes

import numpy as np
import pytest

from oracle import bf16
from oracle.layer import OracleLayer
from rollout import Config, compare, host_bits, to_bits, MAX_ABS, MEAN_ABS, REL_RMS

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import rolling_kv_chunked_b200 as rkv  # noqa: E402

_lib = ctypes.CDLL(rkv.LIB_PATH)
_fn = _lib.rkv_chunk_attention_noalloc
_fn.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int] * 8 + [ctypes.POINTER(ctypes.c_int), ctypes.c_int,
                                                            ctypes.c_void_p]
_fn.restype = ctypes.c_int


def _noalloc(q, kw, vw, out, H, T, gh, gw, W, mode, C, f0, ids):
    arr = (ctypes.c_int * max(1, len(ids)))(*ids)
    return _fn(q.data_ptr(), kw.data_ptr(), vw.data_ptr(), out.data_ptr(), H, T, gh, gw, W, mode, C, f0, arr,
               len(ids), torch.cuda.current_stream().cuda_stream)


def _upload(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


CASES = [
    # relative RoPE, two reference sinks, through eviction and wrap; 480-key window (ragged tile)
    Config("noalloc-rel", 31, H=2, grid_h=8, grid_w=10, C=3, W=7, S=2, rope_mode=OracleLayer.RELATIVE, refs=2,
           chunks=5),
    # absolute RoPE, 400 tokens per frame (3200 keys: whole tiles)
    Config("noalloc-abs", 32, H=4, grid_h=20, grid_w=20, C=2, W=8, S=2, rope_mode=OracleLayer.ABSOLUTE, chunks=6),
    # absolute RoPE with a ragged key tile: 63 tokens per frame, 315 keys
    Config("noalloc-abs-ragged", 34, H=3, grid_h=7, grid_w=9, C=2, W=5, S=1, rope_mode=OracleLayer.ABSOLUTE,
           chunks=4),
]


@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_noalloc_matches_oracle_and_handle_path_twice(cfg):
    T = cfg.T
    orc = OracleLayer(cfg.H, 128, T, cfg.grid_h, cfg.grid_w, cfg.W, cfg.S, cfg.rope_mode)
    h = rkv.RollingKV(1, cfg.H, 128, T, cfg.W, cfg.S, cfg.rope_mode)
    h.set_rope_grid(cfg.grid_h, cfg.grid_w)
    f0 = 0
    if cfg.refs:
        kb, vb = host_bits(cfg, 0, -1, 0, "k", cfg.refs * T), host_bits(cfg, 0, -1, 0, "v", cfg.refs * T)
        orc.write_chunk(kb, vb, cfg.refs, 0)
        h.write_chunk(0, _upload(kb), _upload(vb), cfg.refs, 0)
        f0 = cfg.refs
    out = torch.empty((cfg.Lq, cfg.H, 128), dtype=torch.bfloat16, device="cuda")
    for chunk in range(cfg.chunks):           # roll past the first eviction and the ring wrap
        q, k, v = (host_bits(cfg, 0, chunk, 4, t, cfg.Lq) for t in ("q", "k", "v"))
        orc.write_chunk(k, v, cfg.C, f0)
        h.chunk_attention(0, _upload(q), _upload(k), _upload(v), out, cfg.C, f0, True)
        f0 += cfg.C
    # the read: the frames it attends to in logical order (the sinks and the history frames
    # the chunk does not evict, from the oracle's cache), then the chunk itself
    qb, kb, vb = (host_bits(cfg, 0, 99, 0, t, cfg.Lq) for t in ("q", "k", "v"))
    ids = orc.window_frames(cfg.C, f0)
    held = orc.logical_frames()
    assert ids[-cfg.C:] == list(range(f0, f0 + cfg.C)) and set(ids[:-cfg.C]) <= set(held)
    ck, cv = orc.logical_kv_bits()
    rows = [np.arange(held.index(f) * T, (held.index(f) + 1) * T) for f in ids[:-cfg.C]]
    sel = np.concatenate(rows) if rows else np.zeros(0, dtype=np.int64)
    kw, vw = _upload(np.concatenate([ck[sel], kb])), _upload(np.concatenate([cv[sel], vb]))
    ref = orc.chunk_attention(qb, kb, vb, cfg.C, f0, False)
    q = _upload(qb)
    handle_out = torch.empty((cfg.Lq, cfg.H, 128), dtype=torch.bfloat16, device="cuda")
    h.chunk_attention(0, q, _upload(kb), _upload(vb), handle_out, cfg.C, f0, False)
    torch.cuda.synchronize()
    handle_f64 = bf16.to_f64(to_bits(handle_out))
    for call in range(2):
        got = torch.full((cfg.Lq, cfg.H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _noalloc(q, kw, vw, got, cfg.H, T, cfg.grid_h, cfg.grid_w, cfg.W, cfg.rope_mode, cfg.C, f0,
                        ids) == rkv.OK
        torch.cuda.synchronize()
        bits = to_bits(got)
        for name, want in (("oracle", ref), ("handle path", handle_f64)):
            mx, mean, rel = compare(bits, want)
            assert mx <= MAX_ABS and mean <= MEAN_ABS and rel <= REL_RMS, (call, name, mx, mean, rel)
    h.close()


def _sentinel(n):
    return torch.full((n,), -7.0, dtype=torch.bfloat16, device="cuda")


def _untouched(t):
    torch.cuda.synchronize()
    return bool((t == -7.0).all())


def test_noalloc_rejects_before_launching():
    """Every argument and size error returns before any launch (the output keeps its sentinel)."""
    H, gh, gw = 2, 4, 4
    T = gh * gw
    big = torch.zeros(64 * T * H * 128, dtype=torch.bfloat16, device="cuda")
    out = _sentinel(4 * T * H * 128)
    rel, ab = rkv.ROPE_RELATIVE, rkv.ROPE_ABSOLUTE
    cases = {
        # the window and the queries need more than the fixed array (ABot-size window)
        "capacity": (rkv.ERR_CAPACITY, (24, 880, 22, 40, 21, rel, 3, 18, list(range(21)))),
        # the chunk must be the window's last frames
        "chunk not last": (rkv.ERR_ARG, (H, T, gh, gw, 6, rel, 2, 2, [0, 1, 2, 3, 4])),
        # ids must be strictly increasing
        "repeated id": (rkv.ERR_ARG, (H, T, gh, gw, 6, rel, 1, 2, [0, 1, 1, 2])),
        "decreasing ids": (rkv.ERR_ARG, (H, T, gh, gw, 6, ab, 1, 5, [3, 1, 4, 5])),
        # relative mode: no more frames than the window holds
        "window overfull": (rkv.ERR_ARG, (H, T, gh, gw, 2, rel, 1, 2, [0, 1, 2])),
        # absolute ids are limited to the fixed time table
        "absolute id 4096": (rkv.ERR_UNSUPPORTED, (H, T, gh, gw, 6, ab, 2, 4095, [4094, 4095, 4096])),
        # the relative time table has window_frames rows, limited to 4096
        "relative window 5000": (rkv.ERR_UNSUPPORTED, (H, T, gh, gw, 5000, rel, 1, 2, [0, 1, 2])),
        # at most seven runs of consecutive frames (one launch of the rotation kernel)
        "eight runs": (rkv.ERR_UNSUPPORTED, (H, T, gh, gw, 64, ab, 1, 14, [0, 2, 4, 6, 8, 10, 12, 14])),
        # grid and tokens per frame disagree
        "grid": (rkv.ERR_ARG, (H, T, gh, gw + 1, 6, rel, 1, 1, [0, 1])),
    }
    for name, (want, (h_, t_, gh_, gw_, w_, mode, c_, f0, ids)) in cases.items():
        rc = _noalloc(big, big, big, out, h_, t_, gh_, gw_, w_, mode, c_, f0, ids)
        assert rc == want, (name, rc)
        assert _untouched(out), name
    # a misaligned pointer
    assert _noalloc(big, big, big[1:], out, H, T, gh, gw, 6, rel, 1, 1, [0, 1]) == rkv.ERR_ARG
    assert _untouched(out)
