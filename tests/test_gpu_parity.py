"""GPU parity: the C-ABI kernels against the fp64 oracle on the same seeded inputs.

* the CUDA twin of the input generator reproduces the numpy generator bit for bit;
* flow x0 / renoise: bit-exact (fp64 arithmetic, no FMA, RNE) incl. a ragged tail;
* RoPE: every output within one bf16 ulp of the fp64 rotation;
* chunk attention: every call of small rollouts compared element by element
  (max |err| <= 1.5e-2, mean |err| <= 1e-3, relative RMS <= 1e-2), cache bytes
  and slot -> frame map bit-exact after every commit, through warm-up, sink
  straddling, eviction and ring wrap, several tiles and ragged tails;
* the fused epilogue equals the standalone epilogue applied to the stored output.
"""
import numpy as np
import pytest

import synth
from oracle import bf16, flow as oflow
from oracle.layer import OracleLayer
from rollout import Config, Rollout, assert_close, cache_logical_bits, dev_tensor, host_bits, sample_rows, to_bits

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import rolling_kv_chunked_b200 as rkv  # noqa: E402

ABS, REL, SLOTS = OracleLayer.ABSOLUTE, OracleLayer.RELATIVE, OracleLayer.RELATIVE_SLOTS


def _dev_bits(key, n):
    t = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    synth.fill_normal_bf16_cuda(t.data_ptr(), n, key, 0, torch.cuda.current_stream().cuda_stream)
    return t


def test_generator_twin_bit_exact():
    for n, k in [(1, 5), (1000003, 11), (4096, synth.stream_key(3, 1, 2))]:
        got = to_bits(_dev_bits(k, n))
        assert np.array_equal(got, synth.normal_bf16_bits(k, 0, n))
    t = torch.empty(777, dtype=torch.bfloat16, device="cuda")
    synth.fill_normal_bf16_cuda(t.data_ptr(), 777, 9, 12345, torch.cuda.current_stream().cuda_stream)
    assert np.array_equal(to_bits(t), synth.normal_bf16_bits(9, 12345, 777))


@pytest.mark.parametrize("n", [8, 1000003, 2640 * 3072])
def test_flow_x0_renoise_bit_exact(n):
    xt, v, eps = (_dev_bits(synth.stream_key(0, 50, i, n % 1000), n) for i in range(3))
    sig = oflow.sigmas() + [-1.0]
    for s, sn in zip(sig[:-1], sig[1:]):
        x0 = torch.empty_like(xt)
        xn = torch.empty_like(xt)
        rkv.flow_x0_renoise(xt, v, eps, s, sn, x0, xn if sn >= 0 else None)
        torch.cuda.synchronize()
        rx0, rxn = oflow.x0_renoise_bf16(to_bits(xt), to_bits(v), to_bits(eps), s, sn)
        assert np.array_equal(to_bits(x0), rx0), (n, s)
        if sn >= 0:
            assert np.array_equal(to_bits(xn), rxn), (n, s)


@pytest.mark.parametrize("mode", [ABS, REL, SLOTS])
def test_rope_apply_within_one_ulp(mode):
    H, gh, gw, W, n_frames = 3, 6, 7, 9, 4
    T = gh * gw
    h = rkv.RollingKV(1, H, 128, T, W, 2, mode)
    h.set_rope_grid(gh, gw)
    orc = OracleLayer(H, 128, T, gh, gw, W, 2, mode)
    # (0, 4) and (1, 4) start among the two sinks (split runs in slot-order mode)
    for start, wend in [(0, 4), (1, 4), (5, 9), (37, 41), (200, 300)]:
        x = _dev_bits(synth.stream_key(1, start), n_frames * T * H * 128).view(n_frames * T, H, 128)
        xb = to_bits(x)
        h.rope_apply(x, n_frames, start, wend)
        torch.cuda.synchronize()
        ref = orc.rope_apply(xb, n_frames, start, wend)
        got = bf16.to_f64(to_bits(x))
        # one bf16 ulp at the reference's magnitude: 2**(floor(log2|ref|) - 7)
        ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -126))) - 7)
        assert np.all(np.abs(got - ref) <= ulp), (start, wend)
    h.close()


def test_rope_apply_top_of_time_table():
    """Absolute ids at the top of the library's time table (65534, 65535: angles of tens of
    thousands of radians, the (cos, sin) rows built in fp64 on the host) within one bf16 ulp
    of the oracle; a chunk reaching id 65536 is refused before anything is launched."""
    H, gh, gw, W = 2, 4, 5, 6
    T = gh * gw
    h = rkv.RollingKV(1, H, 128, T, W, 2, ABS)
    h.set_rope_grid(gh, gw)
    orc = OracleLayer(H, 128, T, gh, gw, W, 2, ABS)
    x = _dev_bits(synth.stream_key(1, 65534), 2 * T * H * 128).view(2 * T, H, 128)
    xb = to_bits(x)
    h.rope_apply(x, 2, 65534, 0)
    torch.cuda.synchronize()
    ref = orc.rope_apply(xb, 2, 65534)
    after = to_bits(x)
    got = bf16.to_f64(after)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -126))) - 7)
    assert np.all(np.abs(got - ref) <= ulp)
    with pytest.raises(rkv.RkvError):
        h.rope_apply(x, 2, 65535, 0)
    torch.cuda.synchronize()
    assert np.array_equal(to_bits(x), after)   # the refused call launched nothing
    h.close()


SMALL = [
    Config("tiny-abs", 1, H=2, grid_h=4, grid_w=4, C=2, W=6, S=2, rope_mode=ABS, chunks=10),
    Config("tiny-rel-refs", 2, H=2, grid_h=4, grid_w=4, C=2, W=6, S=2, rope_mode=REL, refs=2, chunks=10),
    Config("ragged-abs", 3, H=3, grid_h=8, grid_w=10, C=3, W=7, S=2, rope_mode=ABS, chunks=8, reads=2),
    Config("ragged-rel", 4, H=3, grid_h=8, grid_w=10, C=3, W=7, S=2, rope_mode=REL, refs=1, chunks=8, reads=2),
    Config("two-cta", 5, H=2, grid_h=10, grid_w=20, C=2, W=5, S=1, rope_mode=ABS, chunks=6, reads=1),
    Config("straddle", 6, H=2, grid_h=4, grid_w=6, C=4, W=18, S=6, rope_mode=ABS, chunks=8, reads=1),
    Config("no-sink", 7, H=1, grid_h=3, grid_w=5, C=1, W=4, S=0, rope_mode=REL, chunks=9, reads=1),
    Config("tiny-slots-refs", 8, H=2, grid_h=4, grid_w=4, C=2, W=6, S=2, rope_mode=SLOTS, refs=2, chunks=10),
    Config("ragged-slots", 9, H=3, grid_h=8, grid_w=10, C=3, W=7, S=2, rope_mode=SLOTS, refs=1, chunks=8, reads=2),
    Config("straddle-slots", 10, H=2, grid_h=4, grid_w=6, C=4, W=18, S=6, rope_mode=SLOTS, chunks=8, reads=1),
    # the chunk fills the whole ring (W - S == C): no history frame is ever visible
    Config("no-history", 11, H=2, grid_h=4, grid_w=6, C=3, W=4, S=1, rope_mode=ABS, chunks=6, reads=1),
    # the largest window the library takes (256 frames), filled and then evicting
    Config("max-window", 12, H=1, grid_h=2, grid_w=8, C=4, W=256, S=3, rope_mode=REL, chunks=70, reads=1),
    # one-token frames: one query row per chunk, every key segment a one-key ragged tile; with
    # 1-5 visible keys the outputs are of order one, so they are compared with the oracle's
    # output rounded to bf16
    Config("single-token", 13, H=2, grid_h=1, grid_w=1, C=1, W=4, S=1, rope_mode=REL, chunks=8, reads=1,
           ref_bf16=True),
    Config("single-token-abs", 14, H=3, grid_h=1, grid_w=1, C=2, W=5, S=2, rope_mode=ABS, chunks=8, reads=2,
           ref_bf16=True),
    # a peaked softmax: queries x 4 (scores x 4), through warm-up, eviction and wrap
    Config("peaked-rel", 15, H=2, grid_h=8, grid_w=10, C=3, W=7, S=2, rope_mode=REL, refs=1, chunks=8, reads=1,
           q_scale=4.0),
    Config("peaked-abs", 16, H=2, grid_h=10, grid_w=20, C=2, W=5, S=1, rope_mode=ABS, chunks=6, reads=1,
           q_scale=4.0),
]


@pytest.mark.parametrize("cfg", SMALL, ids=[c.name for c in SMALL])
def test_rollout_small_every_call(cfg):
    ro = Rollout(cfg, rkv, torch)
    if cfg.refs:
        ro.check_cache(0)
    for chunk in range(cfg.chunks):
        ro.run_chunk(0, chunk)
        torch.cuda.synchronize()
        ro.check_cache(0)
    assert ro.h.poll_device_status() == rkv.OK
    ro.h.close()


def test_fused_flow_epilogue_matches_standalone():
    cfg = Config("fused", 8, H=2, grid_h=8, grid_w=10, C=3, W=7, S=2, rope_mode=ABS, chunks=1)
    h = rkv.RollingKV(1, cfg.H, 128, cfg.T, cfg.W, cfg.S, cfg.rope_mode)
    h.set_rope_grid(cfg.grid_h, cfg.grid_w)
    Lq, n = cfg.Lq, cfg.Lq * cfg.H * 128
    q, k, v = (dev_tensor(torch, cfg, 0, 0, 0, t, Lq) for t in ("q", "k", "v"))
    xt = _dev_bits(synth.stream_key(0, 8, 1), n)
    eps = _dev_bits(synth.stream_key(0, 8, 2), n)
    for s, sn in [(1.0, 0.75), (0.25, -1.0)]:
        out = torch.empty((Lq, cfg.H, 128), dtype=torch.bfloat16, device="cuda")
        x0 = torch.empty(n, dtype=torch.bfloat16, device="cuda")
        xn = torch.empty(n, dtype=torch.bfloat16, device="cuda")
        h.chunk_attention(0, q, k, v, out, cfg.C, 0, False,
                          flow=dict(xt=xt, eps=eps, sigma=s, sigma_next=sn, x0_out=x0,
                                    xt_next_out=xn if sn >= 0 else None))
        torch.cuda.synchronize()
        rx0, rxn = oflow.x0_renoise_bf16(to_bits(xt), to_bits(out).reshape(-1), to_bits(eps), s, sn)
        assert np.array_equal(to_bits(x0), rx0)
        if sn >= 0:
            assert np.array_equal(to_bits(xn), rxn)
        # and the attention output itself against the oracle
        orc = OracleLayer(cfg.H, 128, cfg.T, cfg.grid_h, cfg.grid_w, cfg.W, cfg.S, cfg.rope_mode)
        ref = orc.chunk_attention(to_bits(q), to_bits(k), to_bits(v), cfg.C, 0, False)
        assert_close(to_bits(out), ref, "fused")
    h.close()


def test_outputs_are_deterministic():
    cfg = Config("det", 9, H=2, grid_h=8, grid_w=10, C=3, W=7, S=2, rope_mode=REL, chunks=1)
    h = rkv.RollingKV(1, cfg.H, 128, cfg.T, cfg.W, cfg.S, cfg.rope_mode)
    h.set_rope_grid(cfg.grid_h, cfg.grid_w)
    q, k, v = (dev_tensor(torch, cfg, 0, 0, 0, t, cfg.Lq) for t in ("q", "k", "v"))
    outs = []
    for _ in range(3):
        o = torch.empty((cfg.Lq, cfg.H, 128), dtype=torch.bfloat16, device="cuda")
        h.chunk_attention(0, q, k, v, o, cfg.C, 0, False)
        outs.append(to_bits(o))
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[0], outs[2])
    h.close()


@pytest.mark.parametrize("mode", [ABS, REL, SLOTS])
def test_mixed_chunk_sizes(mode):
    """Chunks of 1 to 4 frames in an irregular order after two reference frames, through
    eviction and ring wrap, with one group of frames written mid-rollout without attention
    (rkv_write_chunk: in absolute mode its rotated keys come from the caller's k, not from a
    call's rotated chunk): every read and commit element by element, the cache bit for bit
    after every chunk."""
    H, gh, gw, W, S = 2, 4, 5, 9, 2
    T = gh * gw
    sizes = [1, 3, 2, 4, 1, 1, 3, 2, 4, 2, 1, 3, 4, 1, 2]
    h = rkv.RollingKV(1, H, 128, T, W, S, mode)
    h.set_rope_grid(gh, gw)
    orc = OracleLayer(H, 128, T, gh, gw, W, S, mode)
    cfg = Config("mixed", 40 + mode, H=H, grid_h=gh, grid_w=gw, C=1, W=W, S=S, rope_mode=mode)
    kr, vr = (dev_tensor(torch, cfg, 0, -1, 0, t, S * T) for t in ("k", "v"))
    h.write_chunk(0, kr, vr, S, 0)
    orc.write_chunk(host_bits(cfg, 0, -1, 0, "k", S * T), host_bits(cfg, 0, -1, 0, "v", S * T), S, 0)
    f0 = S
    for i, C in enumerate(sizes):
        n = C * T
        if i == 6:   # frames kept without attention, mid-rollout
            kw, vw = (dev_tensor(torch, cfg, 0, i, 9, t, n) for t in ("k", "v"))
            h.write_chunk(0, kw, vw, C, f0)
            orc.write_chunk(host_bits(cfg, 0, i, 9, "k", n), host_bits(cfg, 0, i, 9, "v", n), C, f0)
            f0 += C
            continue
        for call in range(2):
            commit = call == 1
            q, k, v = (dev_tensor(torch, cfg, 0, i, call, t, n) for t in ("q", "k", "v"))
            out = torch.empty((n, H, 128), dtype=torch.bfloat16, device="cuda")
            h.chunk_attention(0, q, k, v, out, C, f0, commit)
            ref = orc.chunk_attention(*(host_bits(cfg, 0, i, call, t, n) for t in ("q", "k", "v")), C, f0, commit)
            torch.cuda.synchronize()
            assert_close(to_bits(out), ref, f"mixed mode {mode} chunk {i} (C={C}) call {call}")
        f0 += C
        frames, kb, vb = cache_logical_bits(h, torch, cfg, 0)
        assert frames == orc.logical_frames()
        ok_, ov = orc.logical_kv_bits()
        assert np.array_equal(kb, ok_) and np.array_equal(vb, ov)
    assert h.poll_device_status() == rkv.OK
    h.close()


@pytest.mark.parametrize("mode", [ABS, REL])
def test_reset_replays_bit_for_bit(mode):
    """rkv_reset returns a handle to its just-created state: the same rollout (reference
    frames, then reads and commits through eviction and wrap) run again after a reset gives
    bit for bit the same outputs, slot map and cache bytes; in relative mode this includes
    the rotated ring, whose validity is keyed on the chunk's position."""
    cfg = Config("reset", 45 + mode, H=2, grid_h=4, grid_w=5, C=2, W=6, S=2, rope_mode=mode, refs=1, chunks=7,
                 reads=2)
    h = rkv.RollingKV(1, cfg.H, 128, cfg.T, cfg.W, cfg.S, mode)
    h.set_rope_grid(cfg.grid_h, cfg.grid_w)

    def rollout():
        outs = []
        kr, vr = (dev_tensor(torch, cfg, 0, -1, 0, t, cfg.refs * cfg.T) for t in ("k", "v"))
        h.write_chunk(0, kr, vr, cfg.refs, 0)
        f0 = cfg.refs
        for chunk in range(cfg.chunks):
            for call in range(cfg.reads + 1):
                q, k, v = (dev_tensor(torch, cfg, 0, chunk, call, t, cfg.Lq) for t in ("q", "k", "v"))
                out = torch.empty((cfg.Lq, cfg.H, 128), dtype=torch.bfloat16, device="cuda")
                h.chunk_attention(0, q, k, v, out, cfg.C, f0, call == cfg.reads)
                outs.append(to_bits(out))
            f0 += cfg.C
        frames, kb, vb = cache_logical_bits(h, torch, cfg, 0)
        return outs, list(h.slot_frames(0)), frames, kb, vb

    first = rollout()
    h.reset()
    assert h.frames_committed(0) == 0 and all(f < 0 for f in h.slot_frames(0))
    second = rollout()
    assert len(first[0]) == len(second[0]) and all(np.array_equal(a, b) for a, b in zip(first[0], second[0]))
    assert first[1] == second[1] and first[2] == second[2]
    assert np.array_equal(first[3], second[3]) and np.array_equal(first[4], second[4])
    assert h.poll_device_status() == rkv.OK
    h.close()


def test_two_handles_on_two_streams_match_sequential():
    """Handles share no device state: two handles driven concurrently on two streams (reads
    and commits interleaved, no ordering between the streams) give bit for bit the outputs
    and caches of the same calls run one after another on one stream."""
    cfgs = [Config("conc-a", 30, H=2, grid_h=8, grid_w=10, C=3, W=7, S=2, rope_mode=REL, chunks=5, reads=2),
            Config("conc-b", 31, H=3, grid_h=10, grid_w=20, C=2, W=5, S=1, rope_mode=ABS, chunks=5, reads=2)]

    def run(streams):
        hs, outs = [], []
        for c in cfgs:
            h = rkv.RollingKV(1, c.H, 128, c.T, c.W, c.S, c.rope_mode)
            h.set_rope_grid(c.grid_h, c.grid_w)
            hs.append(h)
        inputs = [[[[dev_tensor(torch, c, 0, chunk, call, t, c.Lq) for t in ("q", "k", "v")]
                    for call in range(c.reads + 1)] for chunk in range(c.chunks)] for c in cfgs]
        res = [[torch.empty((c.Lq, c.H, 128), dtype=torch.bfloat16, device="cuda")
                for _ in range(c.chunks * (c.reads + 1))] for c in cfgs]
        torch.cuda.synchronize()
        for chunk in range(5):
            for i, (c, h) in enumerate(zip(cfgs, hs)):
                st = streams[i]
                with torch.cuda.stream(st):
                    for call in range(c.reads + 1):
                        q, k, v = inputs[i][chunk][call]
                        h.chunk_attention(0, q, k, v, res[i][chunk * (c.reads + 1) + call], c.C, chunk * c.C,
                                          call == c.reads, stream=st.cuda_stream)
        torch.cuda.synchronize()
        for i, (c, h) in enumerate(zip(cfgs, hs)):
            outs.append([to_bits(o) for o in res[i]] + [to_bits(_cache_view(h, c, w)) for w in (0, 1)])
            assert h.poll_device_status() == rkv.OK
            h.close()
        return outs

    one = torch.cuda.Stream()
    seq = run([one, one])
    par = run([torch.cuda.Stream(), torch.cuda.Stream()])
    for a, b in zip(seq, par):
        assert len(a) == len(b) and all(np.array_equal(x, y) for x, y in zip(a, b))


def _cache_view(h, c, which):
    ptr = h.cache_ptrs(0)[which]
    n = c.H * c.W * c.T * 128

    class _A:
        __cuda_array_interface__ = {"shape": (n,), "typestr": "<i2", "data": (ptr, False), "version": 3}
    return torch.as_tensor(_A(), device="cuda").view(torch.bfloat16)


@pytest.mark.parametrize("sink_score", [-2000.0, -150.0, 400.0])
@pytest.mark.parametrize("mode", [ABS, REL])
def test_score_jumps_between_key_tiles(sink_score, mode):
    """The sink frame fills the first key tile with scores far below (or above) the rest.
    -2000: the later tiles' numerators overflow against the first tile's reference, so the
    exact path (maximum first) must take over; -150: the reference moves lazily (tile sums
    near 2^19); +400: the first tile dominates and the later ones underflow. Queries share
    one direction u on the lowest-frequency rotary pairs (near-zero rotation at these
    positions), so q.k_sink stays close to the chosen score whatever the positions."""
    H, gh, gw, W, S, C = 2, 8, 16, 4, 1, 1
    T = gh * gw
    rng = np.random.default_rng(int(abs(sink_score)) + 7 * mode)
    low = [p for p in range(64) if 17 <= p < 22 or 38 <= p < 43 or 59 <= p < 64]
    dims = np.array([2 * p + e for p in low for e in (0, 1)])
    u = np.zeros((H, 128))
    u[:, dims] = rng.standard_normal((H, len(dims)))
    qf = np.broadcast_to(u, (C * T, H, 128)).copy()
    ksink = np.broadcast_to(sink_score * u / np.sum(u * u, axis=1, keepdims=True), (T, H, 128))

    def bits(x):
        return bf16.from_f64(np.asarray(x, dtype=np.float64))

    def dev(b):
        return torch.from_numpy(b.view(np.int16)).cuda().view(torch.bfloat16)

    h = rkv.RollingKV(1, H, 128, T, W, S, mode)
    h.set_rope_grid(gh, gw)
    orc = OracleLayer(H, 128, T, gh, gw, W, S, mode)
    kb, vb = bits(ksink), bits(rng.standard_normal((T, H, 128)))
    h.write_chunk(0, dev(kb), dev(vb), 1, 0)
    orc.write_chunk(kb, vb, 1, 0)
    qb = bits(qf)
    for f0 in range(1, 6):
        kb, vb = bits(rng.standard_normal((T, H, 128))), bits(rng.standard_normal((T, H, 128)))
        out = torch.empty((C * T, H, 128), dtype=torch.bfloat16, device="cuda")
        for commit in (False, True):
            h.chunk_attention(0, dev(qb), dev(kb), dev(vb), out, C, f0, commit)
            torch.cuda.synchronize()
            ref = orc.chunk_attention(qb, kb, vb, C, f0, commit)
            got = to_bits(out)
            assert np.all(np.isfinite(bf16.to_f64(got)))
            assert_close(got, ref, f"sink score {sink_score} frame {f0} commit {commit}")
    assert h.poll_device_status() == rkv.OK
    h.close()


@pytest.mark.parametrize("half", [0, 1])
@pytest.mark.parametrize("jump", [900.0, 2000.0])
@pytest.mark.parametrize("mode", [REL, ABS])
def test_score_jump_inside_a_later_key_tile(half, jump, mode):
    """One frame (128 tokens = one key tile) of the window has keys 64*half .. 64*half+63 with
    scores `jump` above the rest, the tile not being the first of the key stream, so the
    one-pass softmax against the running reference meets numerators far above its bound (900:
    near 2^115, finite; 2000: beyond fp32) in one half of a later tile and must take the exact
    path (maximum first) for that tile, with O and the row sum rescaled. The jump keys share one
    value vector: their weights then decide nothing (the output is that vector up to the
    other keys' vanishing weights), so the comparison is not swamped by the bf16 rounding of
    operands this large, which moves each of their scores by several units."""
    H, gh, gw, W, S, C = 2, 8, 16, 4, 1, 1
    T = gh * gw
    rng = np.random.default_rng(int(jump) + 10 * half + 100 * mode)
    low = [p for p in range(64) if 17 <= p < 22 or 38 <= p < 43 or 59 <= p < 64]
    dims = np.array([2 * p + e for p in low for e in (0, 1)])
    u = np.zeros((H, 128))
    u[:, dims] = rng.standard_normal((H, len(dims)))
    qf = np.broadcast_to(u, (C * T, H, 128)).copy()

    def bits(x):
        return bf16.from_f64(np.asarray(x, dtype=np.float64))

    def dev(b):
        return torch.from_numpy(b.view(np.int16)).cuda().view(torch.bfloat16)

    h = rkv.RollingKV(1, H, 128, T, W, S, mode)
    h.set_rope_grid(gh, gw)
    orc = OracleLayer(H, 128, T, gh, gw, W, S, mode)
    qb = bits(qf)
    for f0 in range(0, 6):
        k = rng.standard_normal((T, H, 128))
        v = rng.standard_normal((T, H, 128))
        if f0 == 2:  # the frame whose half carries the jump (a later tile of the next windows)
            k[64 * half:64 * half + 64] = jump * u / np.sum(u * u, axis=1, keepdims=True)
            v[64 * half:64 * half + 64] = rng.standard_normal((H, 128))
        kb, vb = bits(k), bits(v)
        out = torch.empty((C * T, H, 128), dtype=torch.bfloat16, device="cuda")
        for commit in (False, True):
            h.chunk_attention(0, dev(qb), dev(kb), dev(vb), out, C, f0, commit)
            torch.cuda.synchronize()
            ref = orc.chunk_attention(qb, kb, vb, C, f0, commit)
            got = to_bits(out)
            assert np.all(np.isfinite(bf16.to_f64(got)))
            assert_close(got, ref, f"jump {jump} half {half} frame {f0} commit {commit}")
    assert h.poll_device_status() == rkv.OK
    h.close()


@pytest.mark.parametrize("mode", [REL, SLOTS, ABS])
def test_relative_translation_invariance_bitwise(mode):
    """Identical raw window contents at two chunks whose ring layout is the same (chunks 6 and
    6 + R, contents repeating every R chunks) give bit-identical GPU outputs in both relative
    modes (the ids depend only on a frame's place in the window); absolute ids make them differ."""
    H, gh, gw, C, W, S = 2, 8, 10, 2, 6, 2
    T = gh * gw
    R = W - S
    h = rkv.RollingKV(1, H, 128, T, W, S, mode)
    h.set_rope_grid(gh, gw)
    stream = torch.cuda.current_stream().cuda_stream

    def fill(*key):
        t = torch.empty((C * T, H, 128), dtype=torch.bfloat16, device="cuda")
        synth.fill_normal_bf16_cuda(t.data_ptr(), t.numel(), synth.stream_key(8, *key), 0, stream)
        return t

    sink_k = torch.empty((S * T, H, 128), dtype=torch.bfloat16, device="cuda")
    sink_v = torch.empty_like(sink_k)
    synth.fill_normal_bf16_cuda(sink_k.data_ptr(), sink_k.numel(), synth.stream_key(8, 99, 1), 0, stream)
    synth.fill_normal_bf16_cuda(sink_v.data_ptr(), sink_v.numel(), synth.stream_key(8, 99, 2), 0, stream)
    h.write_chunk(0, sink_k, sink_v, S, 0)
    outs = {}
    f0 = S
    for c in range(6 + R + 1):
        key = c % R
        out = torch.empty((C * T, H, 128), dtype=torch.bfloat16, device="cuda")
        h.chunk_attention(0, fill(key, 0), fill(key, 1), fill(key, 2), out, C, f0, False)
        outs[c] = to_bits(out)
        h.chunk_attention(0, fill(key, 3), fill(key, 4), fill(key, 5), out, C, f0, True)
        f0 += C
    torch.cuda.synchronize()
    same = np.array_equal(outs[6], outs[6 + R])
    assert same == (mode != ABS), mode
    h.close()


def test_host_errors_launch_nothing():
    cfg = Config("err", 10, H=2, grid_h=4, grid_w=4, C=2, W=6, S=2, rope_mode=ABS)
    h = rkv.RollingKV(1, cfg.H, 128, cfg.T, cfg.W, cfg.S, cfg.rope_mode)
    q, k, v = (dev_tensor(torch, cfg, 0, 0, 0, t, cfg.Lq) for t in ("q", "k", "v"))
    out = torch.zeros((cfg.Lq, cfg.H, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rkv.RkvError) as e:
        h.chunk_attention(0, q, k, v, out, cfg.C, 0, True)          # grid not set yet
    assert e.value.code == rkv.ERR_STATE
    h.set_rope_grid(cfg.grid_h, cfg.grid_w)
    for args, code in [((0, q, k, v, out, cfg.C, 2, False), rkv.ERR_ORDER),
                       ((0, q, k, v, out, 5, 0, False), rkv.ERR_CAPACITY),
                       ((1, q, k, v, out, cfg.C, 0, False), rkv.ERR_ARG),
                       ((0, q, k, v, out, 0, 0, False), rkv.ERR_ARG)]:
        with pytest.raises(rkv.RkvError) as e:
            h.chunk_attention(*args)
        assert e.value.code == code
    with pytest.raises(rkv.RkvError) as e:
        h.chunk_attention(0, q.data_ptr() + 2, k, v, out, cfg.C, 0, False)   # misaligned pointer
    assert e.value.code == rkv.ERR_ARG
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0
    assert h.frames_committed(0) == 0 and h.slot_frames(0) == [-1] * cfg.W
    h.close()


def test_expired_wait_reports_timeout_and_context_survives():
    """A 1 ns cap makes the kernel's first unsatisfied wait expire: the call must come back
    (no hang, no trap) with RKV_ERR_TIMEOUT from the status word, and the next call with the
    normal cap must be correct."""
    cfg = Config("timeout", 11, H=2, grid_h=4, grid_w=4, C=2, W=6, S=2, rope_mode=ABS)
    h = rkv.RollingKV(1, cfg.H, 128, cfg.T, cfg.W, cfg.S, cfg.rope_mode)
    h.set_rope_grid(cfg.grid_h, cfg.grid_w)
    q, k, v = (dev_tensor(torch, cfg, 0, 0, 0, t, cfg.Lq) for t in ("q", "k", "v"))
    out = torch.zeros((cfg.Lq, cfg.H, 128), dtype=torch.bfloat16, device="cuda")
    h.set_wait_limit(1)
    h.chunk_attention(0, q, k, v, out, cfg.C, 0, False)
    assert h.poll_device_status() == rkv.ERR_TIMEOUT
    assert h.poll_device_status() == rkv.OK          # the word is cleared by the poll
    h.set_wait_limit(2_000_000_000)
    h.chunk_attention(0, q, k, v, out, cfg.C, 0, False)
    assert h.poll_device_status() == rkv.OK
    orc = OracleLayer(cfg.H, 128, cfg.T, cfg.grid_h, cfg.grid_w, cfg.W, cfg.S, cfg.rope_mode)
    ref = orc.chunk_attention(to_bits(q), to_bits(k), to_bits(v), cfg.C, 0, False)
    assert_close(to_bits(out), ref, "after timeout")
    h.close()


def test_flow_epilogue_all_finite_bit_patterns():
    """Inputs drawn uniformly over every finite bf16 bit pattern (zeros, subnormals, the
    largest magnitudes): x0 and xt' must equal the oracle's fp64 result rounded to nearest
    even bit for bit, including rounding ties, subnormal results and overflow to infinity."""
    rng = np.random.default_rng(123)
    n = 1 << 20
    def finite_bits():
        b = rng.integers(0, 1 << 16, size=n, dtype=np.uint32).astype(np.uint16)
        exp = (b.astype(np.uint32) >> 7) & 0xFF
        b[exp == 0xFF] &= 0x807F          # map inf / nan patterns to finite ones
        return b
    xb, vb, eb = finite_bits(), finite_bits(), finite_bits()
    dev = lambda b: torch.from_numpy(b.view(np.int16).copy()).cuda().view(torch.bfloat16)
    xt, v, eps = dev(xb), dev(vb), dev(eb)
    for s, sn in [(1.0, 0.75), (0.75, 0.5), (0.5, 0.25), (0.25, -1.0), (0.5, 0.0)]:
        x0 = torch.empty_like(xt)
        xn = torch.empty_like(xt)
        rkv.flow_x0_renoise(xt, v, eps, s, sn, x0, xn if sn >= 0 else None)
        torch.cuda.synchronize()
        rx0, rxn = oflow.x0_renoise_bf16(xb, vb, eb, s, sn)
        assert np.array_equal(to_bits(x0), rx0), s
        if sn >= 0:
            assert np.array_equal(to_bits(xn), rxn), s


def test_chained_calls_see_their_predecessors_writes():
    """Calls are asynchronous on the caller's stream. Chains of calls where each launch reads
    what the previous one wrote, issued back to back without a host synchronisation, must give
    bit for bit what the same calls give with a synchronisation after each: RoPE applied in
    place three times (ABot chunk size), and four x0 / renoise steps each feeding the next."""
    H, gh, gw, n_frames = 24, 22, 40, 3
    T = gh * gw
    h = rkv.RollingKV(1, H, 128, T, 21, 5, ABS)
    h.set_rope_grid(gh, gw)
    x0 = _dev_bits(synth.stream_key(11, 1), n_frames * T * H * 128).view(n_frames * T, H, 128)
    chained, synced = x0.clone(), x0.clone()
    for k in range(3):
        h.rope_apply(chained, n_frames, 5 + k, 0)
    for k in range(3):
        h.rope_apply(synced, n_frames, 5 + k, 0)
        torch.cuda.synchronize()
    torch.cuda.synchronize()
    assert np.array_equal(to_bits(chained), to_bits(synced))
    assert not np.array_equal(to_bits(chained), to_bits(x0))
    h.close()

    n = n_frames * T * H * 128
    v, eps = (_dev_bits(synth.stream_key(11, 2 + i), n) for i in range(2))
    xt = _dev_bits(synth.stream_key(11, 4), n)
    sig = [1.0, 0.75, 0.5, 0.25, -1.0]
    outs = {}
    for mode in ("chained", "synced"):
        cur = xt.clone()
        for s in range(4):
            x0b, xn = torch.empty_like(cur), torch.empty_like(cur)
            rkv.flow_x0_renoise(cur, v, eps, sig[s], sig[s + 1], x0b, xn if sig[s + 1] >= 0 else None)
            if mode == "synced":
                torch.cuda.synchronize()
            cur = xn if sig[s + 1] >= 0 else x0b
        torch.cuda.synchronize()
        outs[mode] = to_bits(cur)
    assert np.array_equal(outs["chained"], outs["synced"])


@pytest.mark.parametrize("gh, gw, C, W", [(8, 10, 3, 7), (10, 20, 2, 12)])
def test_outputs_stay_in_bounds_and_feed_the_next_call(gh, gw, C, W):
    """Each call's output is the next call's queries, issued without a host synchronisation,
    and the output is a view followed by guard rows. The chunk (240 / 400 queries) ends inside
    the second 128-row tile of its last query block; the windows cover short key streams (a
    few tiles, output written through shared memory by TMA stores) and, in the second shape,
    long ones (up to 19 tiles, one row per thread). Outputs equal bit for bit those of the same
    chain with a synchronisation after each call, and no guard row changes."""
    H, S = 2, 2
    T = gh * gw
    Lq = C * T
    outs = {}
    for mode in ("chained", "synced"):
        h = rkv.RollingKV(1, H, 128, T, W, S, ABS)
        h.set_rope_grid(gh, gw)
        full = torch.full((Lq + 80, H, 128), -7.0, dtype=torch.bfloat16, device="cuda")
        q = _dev_bits(synth.stream_key(12, 1), Lq * H * 128).view(Lq, H, 128)
        seq = []
        for c in range(6):
            k = _dev_bits(synth.stream_key(12, 2, c), Lq * H * 128).view(Lq, H, 128)
            v = _dev_bits(synth.stream_key(12, 3, c), Lq * H * 128).view(Lq, H, 128)
            out = full[:Lq]
            h.chunk_attention(0, q, k, v, out, C, c * C, True)
            if mode == "synced":
                torch.cuda.synchronize()
            q = out.clone() if mode == "synced" else _copy_on_stream(out)
            seq.append(q)
        torch.cuda.synchronize()
        assert bool((full[Lq:] == -7.0).all()), f"{mode}: rows past the output written"
        assert h.poll_device_status() == rkv.OK
        outs[mode] = [to_bits(t) for t in seq]
        h.close()
    for a, b in zip(outs["chained"], outs["synced"]):
        assert np.array_equal(a, b)


def _copy_on_stream(t):
    """A device copy queued on the current stream (no host synchronisation)."""
    c = torch.empty_like(t)
    c.copy_(t, non_blocking=True)
    return c


def test_fused_flow_with_more_units_than_sms():
    """A short key stream (1560 keys = 13 tiles: the persistent short-stream kernel) with 40
    heads x 7 query blocks = 280 units, so CTAs walk two units each, with the fused x0 /
    renoise epilogue: x0 and xt' bit-exact against the oracle's step on the stored output, the
    output on sampled rows of sampled heads within the attention tolerance, through three
    chunks (the window rolls)."""
    cfg = Config("units", 17, H=40, grid_h=30, grid_w=52, C=1, W=1, S=0, rope_mode=ABS, chunks=1)
    h = rkv.RollingKV(1, cfg.H, 128, cfg.T, cfg.W, cfg.S, cfg.rope_mode)
    h.set_rope_grid(cfg.grid_h, cfg.grid_w)
    orc = OracleLayer(cfg.H, 128, cfg.T, cfg.grid_h, cfg.grid_w, cfg.W, cfg.S, cfg.rope_mode)
    Lq, n = cfg.Lq, cfg.Lq * cfg.H * 128
    rows = sample_rows(Lq, n=48, seed=5)
    heads = [0, 17, 39]
    for chunk in range(3):
        q, k, v = (dev_tensor(torch, cfg, 0, chunk, 0, t, Lq) for t in ("q", "k", "v"))
        xt = _dev_bits(synth.stream_key(0, 17, chunk, 1), n)
        eps = _dev_bits(synth.stream_key(0, 17, chunk, 2), n)
        out = torch.empty((Lq, cfg.H, 128), dtype=torch.bfloat16, device="cuda")
        x0 = torch.empty(n, dtype=torch.bfloat16, device="cuda")
        xn = torch.empty(n, dtype=torch.bfloat16, device="cuda")
        h.chunk_attention(0, q, k, v, out, cfg.C, chunk, True,
                          flow=dict(xt=xt, eps=eps, sigma=0.75, sigma_next=0.5, x0_out=x0, xt_next_out=xn))
        torch.cuda.synchronize()
        assert h.poll_device_status() == rkv.OK
        rx0, rxn = oflow.x0_renoise_bf16(to_bits(xt), to_bits(out).reshape(-1), to_bits(eps), 0.75, 0.5)
        assert np.array_equal(to_bits(x0), rx0) and np.array_equal(to_bits(xn), rxn)
        qb, kb, vb = (to_bits(t) for t in (q, k, v))
        ref = orc.chunk_attention(qb, kb, vb, cfg.C, chunk, True, rows=rows, heads=heads)
        assert_close(to_bits(out)[rows][:, heads], ref, f"chunk {chunk}")
    h.close()


def test_split_last_wave_with_fused_flow():
    """16 heads x 10 query blocks = 160 units of a 50-tile key stream: 148 run whole, the last
    12 (heads 14 and 15) as two CTAs over half the keys each plus a combine launch. The fused
    x0 / renoise step must equal the oracle's step on the stored output bit for bit (also on
    the split units), and the output of a split head and of a whole one must match the oracle
    on sampled rows."""
    cfg = Config("split", 18, H=16, grid_h=32, grid_w=40, C=2, W=5, S=1, rope_mode=ABS, chunks=1)
    h = rkv.RollingKV(1, cfg.H, 128, cfg.T, cfg.W, cfg.S, cfg.rope_mode)
    h.set_rope_grid(cfg.grid_h, cfg.grid_w)
    orc = OracleLayer(cfg.H, 128, cfg.T, cfg.grid_h, cfg.grid_w, cfg.W, cfg.S, cfg.rope_mode)
    kw, vw = (dev_tensor(torch, cfg, 0, -1, 0, t, 3 * cfg.T) for t in ("k", "v"))
    h.write_chunk(0, kw, vw, 3, 0)
    orc.write_chunk(to_bits(kw), to_bits(vw), 3, 0)
    Lq, n = cfg.Lq, cfg.Lq * cfg.H * 128
    q, k, v = (dev_tensor(torch, cfg, 0, 0, 0, t, Lq) for t in ("q", "k", "v"))
    xt = _dev_bits(synth.stream_key(0, 18, 1), n)
    eps = _dev_bits(synth.stream_key(0, 18, 2), n)
    for s, sn in [(1.0, 0.75), (0.25, -1.0)]:
        out = torch.empty((Lq, cfg.H, 128), dtype=torch.bfloat16, device="cuda")
        x0 = torch.empty(n, dtype=torch.bfloat16, device="cuda")
        xn = torch.empty(n, dtype=torch.bfloat16, device="cuda")
        h.chunk_attention(0, q, k, v, out, cfg.C, 3, False,
                          flow=dict(xt=xt, eps=eps, sigma=s, sigma_next=sn, x0_out=x0,
                                    xt_next_out=xn if sn >= 0 else None))
        torch.cuda.synchronize()
        assert h.poll_device_status() == rkv.OK
        rx0, rxn = oflow.x0_renoise_bf16(to_bits(xt), to_bits(out).reshape(-1), to_bits(eps), s, sn)
        assert np.array_equal(to_bits(x0), rx0)
        if sn >= 0:
            assert np.array_equal(to_bits(xn), rxn)
    rows = sample_rows(Lq, n=64, seed=18)
    heads = [0, 15]
    ref = orc.chunk_attention(to_bits(q), to_bits(k), to_bits(v), cfg.C, 3, False, rows=rows, heads=heads)
    assert_close(to_bits(out)[rows][:, heads], ref, "split last wave")
    h.close()
