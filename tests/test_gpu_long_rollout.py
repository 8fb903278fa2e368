"""Long-rollout stress: the ABot shape (H=24, 880 tokens/frame, chunks of 3 frames,
window 21 frames, 5 reference sinks, relative RoPE) stacked 30 layers deep with
independent seeded inputs per layer, 1200 chunks x (4 denoise reads + 1 commit).

The oracle follows every layer's literal shift-left cache by frame id. After chunks
1, 7, 100 and 1200 every layer's slot map must equal the ring placement of exactly the
frames the oracle holds, and sampled cache bytes (all held frames, 2 heads, 16 tokens
per frame, K and V) must equal the generator's bits of the commits that wrote them.
After the last chunk one more read is checked on sampled rows of two layers against
the fp64 oracle. About three minutes of GPU time.
"""
import numpy as np
import pytest

import synth
from oracle.cache import RollingCache
from oracle.layer import Frame, OracleLayer
from rollout import Config, _wrap, assert_close, dev_tensor, host_bits_heads, key, sample_rows, to_bits

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import rolling_kv_chunked_b200 as rkv  # noqa: E402

CFG = Config("long", 40, H=24, grid_h=22, grid_w=40, C=3, W=21, S=5, rope_mode=OracleLayer.RELATIVE, refs=5,
             chunks=1200, reads=4, layers=30)
CHECK_AFTER = (1, 7, 100, 1200)


def _origin(frame, cfg):
    """(chunk, call, token offset) of the commit that wrote `frame` (chunk -1 = the references)."""
    if frame < cfg.refs:
        return -1, 0, frame * cfg.T
    c = (frame - cfg.refs) // cfg.C
    return c, cfg.reads, (frame - cfg.refs - c * cfg.C) * cfg.T


def _check_layer_cache(h, cfg, layer, cache, heads, toks):
    S, R, T = cfg.S, cfg.W - cfg.S, cfg.T
    frames = h.slot_frames(layer)
    held = sorted(f for f in frames if f >= 0)
    assert held == cache.slots, layer
    for s, f in enumerate(frames):
        if f >= 0:
            assert s == (f if f < S else S + (f - S) % R)
    kp, vp = h.cache_ptrs(layer)
    n_el = cfg.H * cfg.W * T * 128
    k_all = _wrap(torch, kp, n_el).view(cfg.H, cfg.W * T, 128)
    v_all = _wrap(torch, vp, n_el).view(cfg.H, cfg.W * T, 128)
    hs = torch.tensor(heads, device="cuda")
    for s, f in enumerate(frames):
        if f < 0:
            continue
        rows = torch.tensor([s * T + t for t in toks], device="cuda")
        kg = to_bits(k_all.index_select(0, hs).index_select(1, rows))     # [heads, toks, 128]
        vg = to_bits(v_all.index_select(0, hs).index_select(1, rows))
        c, call, off = _origin(f, cfg)
        tok = (off + np.asarray(toks))[None, :, None]
        idx = (tok * cfg.H + np.asarray(heads)[:, None, None]) * 128 + np.arange(128)[None, None, :]
        assert np.array_equal(kg, synth.normal_bf16_bits_at(key(cfg, layer, c, call, "k"), idx)), (layer, f)
        assert np.array_equal(vg, synth.normal_bf16_bits_at(key(cfg, layer, c, call, "v"), idx)), (layer, f)


def test_long_rollout_30_layers_1200_chunks():
    cfg = CFG
    T, C = cfg.T, cfg.C
    h = rkv.RollingKV(cfg.layers, cfg.H, 128, T, cfg.W, cfg.S, cfg.rope_mode)
    h.set_rope_grid(cfg.grid_h, cfg.grid_w)
    caches = [RollingCache(cfg.W, cfg.S) for _ in range(cfg.layers)]
    for layer in range(cfg.layers):
        k = dev_tensor(torch, cfg, layer, -1, 0, "k", cfg.refs * T)
        v = dev_tensor(torch, cfg, layer, -1, 0, "v", cfg.refs * T)
        h.write_chunk(layer, k, v, cfg.refs, 0)
        caches[layer].append(list(range(cfg.refs)))
    q = torch.empty((cfg.Lq, cfg.H, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.empty_like(q)
    v = torch.empty_like(q)
    out = torch.empty_like(q)
    heads, toks = [0, cfg.H - 1], [0, 1, 39, 40, 127, 128, 300, 439, 440, 511, 512, 700, 799, 800, 878, 879]
    for c in range(cfg.chunks):
        f0 = cfg.refs + c * C
        for layer in range(cfg.layers):
            for call in range(cfg.reads + 1):
                dev_tensor(torch, cfg, layer, c, call, "q", cfg.Lq, out=q)
                dev_tensor(torch, cfg, layer, c, call, "k", cfg.Lq, out=k)
                dev_tensor(torch, cfg, layer, c, call, "v", cfg.Lq, out=v)
                h.chunk_attention(layer, q, k, v, out, C, f0, call == cfg.reads)
            caches[layer].append(list(range(f0, f0 + C)))
        if c + 1 in CHECK_AFTER:
            torch.cuda.synchronize()
            assert h.poll_device_status() == rkv.OK
            for layer in range(cfg.layers):
                assert h.frames_committed(layer) == f0 + C
                _check_layer_cache(h, cfg, layer, caches[layer], heads, toks)

    # one more read after the last chunk, checked on sampled rows of two layers
    f0 = cfg.refs + cfg.chunks * C
    rows = sample_rows(cfg.Lq, n=48, seed=5)
    for layer in (0, cfg.layers - 1):
        for t_, buf in (("q", q), ("k", k), ("v", v)):
            dev_tensor(torch, cfg, layer, cfg.chunks, 0, t_, cfg.Lq, out=buf)
        h.chunk_attention(layer, q, k, v, out, C, f0, False)
        orc = OracleLayer(len(heads), 128, T, cfg.grid_h, cfg.grid_w, cfg.W, cfg.S, cfg.rope_mode)
        slots = []
        for f in caches[layer].slots:
            cc, call, off = _origin(f, cfg)
            tok = (off + np.arange(T))[:, None, None]
            idx = (tok * cfg.H + np.asarray(heads)[None, :, None]) * 128 + np.arange(128)[None, None, :]
            slots.append(Frame(f, synth.normal_bf16_bits_at(key(cfg, layer, cc, call, "k"), idx),
                               synth.normal_bf16_bits_at(key(cfg, layer, cc, call, "v"), idx)))
        orc.cache.slots = slots
        orc.committed = f0
        ref = orc.chunk_attention(*(host_bits_heads(cfg, layer, cfg.chunks, 0, t_, cfg.Lq, heads) for t_ in "qkv"),
                                  C, f0, False, rows=rows)
        assert_close(to_bits(out)[rows][:, heads], ref, f"long layer {layer}")
    assert h.poll_device_status() == rkv.OK
    h.close()
