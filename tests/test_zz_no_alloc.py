"""GPU test of rkv_chunk_attention_noalloc, the entry point for callers that may
not allocate device memory (their host framework's allocator must own every
byte, or allocation is forbidden after start-up): it keeps its scratch in a
fixed static device array instead of allocating.

It is called through the C ABI (ctypes) twice in a row on the window the
handle path attends to, and both results must agree with the handle path's
rkv_chunk_attention output within the attention tolerance of the other tests.
This file is named to be collected last; it depends on no other test.
"""
import ctypes

import numpy as np
import pytest

from oracle import bf16
from oracle.layer import OracleLayer
from rollout import Config, _wrap, compare, dev_tensor, to_bits, MAX_ABS, MEAN_ABS, REL_RMS

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


def _noalloc(q, kw, vw, out, cfg, f0, ids):
    arr = (ctypes.c_int * len(ids))(*ids)
    return _fn(q.data_ptr(), kw.data_ptr(), vw.data_ptr(), out.data_ptr(), cfg.H, cfg.T, cfg.grid_h, cfg.grid_w,
               cfg.W, cfg.rope_mode, cfg.C, f0, arr, len(ids), torch.cuda.current_stream().cuda_stream)


def _window(h, cfg, f0, k_chunk, v_chunk):
    """The frames the handle path attends to, gathered in logical order from its raw ring."""
    T = cfg.T
    kp, vp = h.cache_ptrs(0)
    n_el = cfg.H * cfg.W * T * 128
    k_all = _wrap(torch, kp, n_el).view(cfg.H, cfg.W * T, 128)
    v_all = _wrap(torch, vp, n_el).view(cfg.H, cfg.W * T, 128)
    ks, vs, ids = [], [], []
    for src, first, n, fr0 in rkv.plan_window(cfg.W, cfg.S, h.frames_committed(0), cfg.C, f0):
        if src == 0:
            ks.append(k_all[:, first * T:(first + n) * T].permute(1, 0, 2))
            vs.append(v_all[:, first * T:(first + n) * T].permute(1, 0, 2))
        else:
            ks.append(k_chunk)
            vs.append(v_chunk)
        ids += list(range(fr0, fr0 + n))
    return torch.cat(ks).contiguous(), torch.cat(vs).contiguous(), ids


CASES = [
    Config("noalloc-rel", 31, H=2, grid_h=8, grid_w=10, C=3, W=7, S=2, rope_mode=OracleLayer.RELATIVE, refs=2,
           chunks=5),
    Config("noalloc-abs", 32, H=4, grid_h=20, grid_w=20, C=2, W=8, S=2, rope_mode=OracleLayer.ABSOLUTE, chunks=6),
]


@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_noalloc_matches_handle_path_twice(cfg):
    h = rkv.RollingKV(1, cfg.H, 128, cfg.T, cfg.W, cfg.S, cfg.rope_mode)
    h.set_rope_grid(cfg.grid_h, cfg.grid_w)
    f0 = 0
    if cfg.refs:
        h.write_chunk(0, dev_tensor(torch, cfg, 0, -1, 0, "k", cfg.refs * cfg.T),
                      dev_tensor(torch, cfg, 0, -1, 0, "v", cfg.refs * cfg.T), cfg.refs, 0)
        f0 = cfg.refs
    for chunk in range(cfg.chunks):           # roll past the first eviction and the ring wrap
        q, k, v = (dev_tensor(torch, cfg, 0, chunk, 4, t, cfg.Lq) for t in ("q", "k", "v"))
        out = torch.empty((cfg.Lq, cfg.H, 128), dtype=torch.bfloat16, device="cuda")
        h.chunk_attention(0, q, k, v, out, cfg.C, f0, True)
        f0 += cfg.C
    q, k, v = (dev_tensor(torch, cfg, 0, 99, 0, t, cfg.Lq) for t in ("q", "k", "v"))
    ref = torch.empty((cfg.Lq, cfg.H, 128), dtype=torch.bfloat16, device="cuda")
    h.chunk_attention(0, q, k, v, ref, cfg.C, f0, False)
    kw, vw, ids = _window(h, cfg, f0, k, v)
    torch.cuda.synchronize()
    ref_f64 = bf16.to_f64(to_bits(ref))
    for call in range(2):
        out = torch.full((cfg.Lq, cfg.H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _noalloc(q, kw, vw, out, cfg, f0, ids) == rkv.OK
        torch.cuda.synchronize()
        mx, mean, rel = compare(to_bits(out), ref_f64)
        assert mx <= MAX_ABS and mean <= MEAN_ABS and rel <= REL_RMS, (call, mx, mean, rel)
    h.close()


def test_noalloc_rejects_oversize_window():
    cfg = Config("big", 33, H=24, grid_h=22, grid_w=40, C=3, W=21, S=5, rope_mode=OracleLayer.RELATIVE)
    t = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    ids = list(range(21))
    assert _noalloc(t, t, t, t, cfg, 18, ids) == rkv.ERR_CAPACITY
    assert _noalloc(t, t, t, t, cfg, 17, ids) == rkv.ERR_ARG          # chunk must end the window
