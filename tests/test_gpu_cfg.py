"""GPU parity of classifier-free guidance, the causal pre-training mode: two branches
(conditional, unconditional), one rolling cache each, guidance scale 5.0 and 40 steps
per chunk, then the clean commit of each branch.

* the standalone guided epilogue is bit-exact against the oracle: N(0,1) inputs with a
  ragged tail, every finite bf16 bit pattern, scales 5, 1, 0 and -2.5;
* fused: in a two-handle rollout every attention output is within tolerance of the fp64
  oracle; the guided x0 / xt' of the unconditional call is bit-exact against the oracle
  applied to the two branches' stored outputs, chained from step to step; each branch's
  cache bytes and slot map are bit-exact after every commit;
* argument errors (missing epilogue, aliasing out, non-finite scale) launch nothing.
"""
from dataclasses import replace

import numpy as np
import pytest

import synth
from oracle import flow as oflow
from oracle.layer import OracleLayer
from rollout import Config, Rollout, assert_close, dev_tensor, host_bits, sample_rows, to_bits

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import rolling_kv_chunked_b200 as rkv  # noqa: E402

ABS, REL = OracleLayer.ABSOLUTE, OracleLayer.RELATIVE
CFG_SCALE = 5.0
STEPS = 40


def _dev_bits(key, n):
    t = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    synth.fill_normal_bf16_cuda(t.data_ptr(), n, key, 0, torch.cuda.current_stream().cuda_stream)
    return t


def _schedule(steps):
    """sigma_k = 1 - k / steps, then -1 for "no next step"."""
    return [1.0 - k / steps for k in range(steps)] + [-1.0]


@pytest.mark.parametrize("n", [13, 1000003])
def test_cfg_flow_bit_exact(n):
    xt, c, u, eps = (_dev_bits(synth.stream_key(0, 60, i, n % 1000), n) for i in range(4))
    bits = [to_bits(t) for t in (xt, c, u, eps)]
    for scale in (CFG_SCALE, 1.0, 0.0, -2.5):
        for s, sn in [(1.0, 0.975), (0.5, 0.25), (0.025, -1.0), (0.5, 0.0)]:
            x0 = torch.empty_like(xt)
            xn = torch.empty_like(xt)
            rkv.flow_cfg_x0_renoise(xt, c, u, eps, scale, s, sn, x0, xn if sn >= 0 else None)
            torch.cuda.synchronize()
            rx0, rxn = oflow.cfg_x0_renoise_bf16(bits[0], bits[1], bits[2], bits[3], scale, s, sn)
            assert np.array_equal(to_bits(x0), rx0), (n, scale, s)
            if sn >= 0:
                assert np.array_equal(to_bits(xn), rxn), (n, scale, s)


def test_cfg_flow_all_finite_bit_patterns():
    rng = np.random.default_rng(321)
    n = 1 << 20

    def finite_bits():
        b = rng.integers(0, 1 << 16, size=n, dtype=np.uint32).astype(np.uint16)
        b[((b.astype(np.uint32) >> 7) & 0xFF) == 0xFF] &= 0x807F
        return b
    xb, cb, ub, eb = (finite_bits() for _ in range(4))
    dev = lambda b: torch.from_numpy(b.view(np.int16).copy()).cuda().view(torch.bfloat16)
    xt, c, u, eps = dev(xb), dev(cb), dev(ub), dev(eb)
    for scale, s, sn in [(CFG_SCALE, 1.0, 0.975), (CFG_SCALE, 0.025, -1.0), (-2.5, 0.5, 0.25)]:
        x0 = torch.empty_like(xt)
        xn = torch.empty_like(xt)
        rkv.flow_cfg_x0_renoise(xt, c, u, eps, scale, s, sn, x0, xn if sn >= 0 else None)
        torch.cuda.synchronize()
        rx0, rxn = oflow.cfg_x0_renoise_bf16(xb, cb, ub, eb, scale, s, sn)
        assert np.array_equal(to_bits(x0), rx0), (scale, s)
        if sn >= 0:
            assert np.array_equal(to_bits(xn), rxn), (scale, s)


CFG_ROLLOUTS = [
    # evictions from chunk 3 on, one query tile, absolute RoPE
    Config("cfg-tiny", 20, H=2, grid_h=4, grid_w=4, C=2, W=6, S=2, rope_mode=ABS, chunks=4, reads=STEPS),
    # relative RoPE, a reference sink, two query tiles with a ragged tail, ring wrap
    Config("cfg-rel", 21, H=2, grid_h=8, grid_w=10, C=3, W=7, S=2, rope_mode=REL, refs=1, chunks=3, reads=STEPS),
]


@pytest.mark.parametrize("cfg", CFG_ROLLOUTS, ids=[c.name for c in CFG_ROLLOUTS])
def test_cfg_two_cache_rollout(cfg):
    branches = [Rollout(cfg, rkv, torch), Rollout(replace(cfg, seed=cfg.seed + 1), rkv, torch)]
    Lq, n = cfg.Lq, cfg.Lq * cfg.H * 128
    sig = _schedule(STEPS)
    check_steps = set(range(STEPS)) if cfg.T * cfg.W <= 128 else {0, 1, STEPS // 2, STEPS - 1}
    outs = [torch.empty((Lq, cfg.H, 128), dtype=torch.bfloat16, device="cuda") for _ in branches]
    for chunk in range(cfg.chunks):
        f0 = branches[0].f0[0]
        xt = _dev_bits(synth.stream_key(cfg.seed, cfg.cfg_id, 99, chunk), n)
        xt_ref = to_bits(xt)
        for step in range(STEPS):
            s, sn = sig[step], sig[step + 1]
            eps = _dev_bits(synth.stream_key(cfg.seed, cfg.cfg_id, 98, chunk, step), n)
            x0 = torch.empty(n, dtype=torch.bfloat16, device="cuda")
            xn = torch.empty(n, dtype=torch.bfloat16, device="cuda")
            qkv = [[dev_tensor(torch, b.cfg, 0, chunk, step, t, Lq) for t in "qkv"] for b in branches]
            branches[0].h.chunk_attention(0, *qkv[0], outs[0], cfg.C, f0, False)
            branches[1].h.chunk_attention(0, *qkv[1], outs[1], cfg.C, f0, False,
                                          flow=dict(xt=xt, eps=eps, sigma=s, sigma_next=sn, x0_out=x0,
                                                    xt_next_out=xn if sn >= 0 else None,
                                                    v_cond=outs[0], cfg_scale=CFG_SCALE))
            torch.cuda.synchronize()
            c_bits, u_bits = to_bits(outs[0]), to_bits(outs[1])
            rx0, rxn = oflow.cfg_x0_renoise_bf16(xt_ref, c_bits.reshape(-1), u_bits.reshape(-1), to_bits(eps),
                                                 CFG_SCALE, s, sn)
            assert np.array_equal(to_bits(x0), rx0), (cfg.name, chunk, step)
            if sn >= 0:
                assert np.array_equal(to_bits(xn), rxn), (cfg.name, chunk, step)
                xt, xt_ref = xn, rxn
            if step in check_steps:
                for b, got in zip(branches, (c_bits, u_bits)):
                    ref = b.oracles[0].chunk_attention(*(host_bits(b.cfg, 0, chunk, step, t, Lq) for t in "qkv"),
                                                       cfg.C, f0, False)
                    assert_close(got, ref, f"{b.cfg.name} seed {b.cfg.seed} chunk {chunk} step {step}")
        # the clean pass of each branch writes its own cache
        for b, out in zip(branches, outs):
            q, k, v = (dev_tensor(torch, b.cfg, 0, chunk, STEPS, t, Lq) for t in "qkv")
            b.h.chunk_attention(0, q, k, v, out, cfg.C, f0, True)
            ref = b.oracles[0].chunk_attention(*(host_bits(b.cfg, 0, chunk, STEPS, t, Lq) for t in "qkv"),
                                               cfg.C, f0, True)
            torch.cuda.synchronize()
            assert_close(to_bits(out), ref, f"{b.cfg.name} seed {b.cfg.seed} chunk {chunk} commit")
            b.f0[0] = f0 + cfg.C
            b.check_cache(0)
    for b in branches:
        assert b.h.poll_device_status() == rkv.OK
        b.h.close()


def test_cfg_argument_errors_launch_nothing():
    cfg = Config("cfg-err", 22, H=2, grid_h=4, grid_w=4, C=2, W=6, S=2, rope_mode=ABS, chunks=1)
    h = rkv.RollingKV(1, cfg.H, 128, cfg.T, cfg.W, cfg.S, cfg.rope_mode)
    h.set_rope_grid(cfg.grid_h, cfg.grid_w)
    Lq, n = cfg.Lq, cfg.Lq * cfg.H * 128
    q, k, v = (dev_tensor(torch, cfg, 0, 0, 0, t, Lq) for t in "qkv")
    out = torch.empty((Lq, cfg.H, 128), dtype=torch.bfloat16, device="cuda")
    c = torch.empty_like(out)
    xt, eps, x0, xn = (torch.zeros(n, dtype=torch.bfloat16, device="cuda") for _ in range(4))
    good = dict(xt=xt, eps=eps, sigma=1.0, sigma_next=0.975, x0_out=x0, xt_next_out=xn, v_cond=c,
                cfg_scale=CFG_SCALE)
    for bad in (dict(v_cond=out), dict(cfg_scale=float("nan")), dict(cfg_scale=float("inf")),
                dict(v_cond=torch.empty(n + 8, dtype=torch.bfloat16, device="cuda")[1:])):
        with pytest.raises(rkv.RkvError) as e:
            h.chunk_attention(0, q, k, v, out, cfg.C, 0, False, flow={**good, **bad})
        assert e.value.code == rkv.ERR_ARG
    with pytest.raises(rkv.RkvError):
        rkv.flow_cfg_x0_renoise(xt, c, out, eps, float("nan"), 1.0, 0.975, x0, xn)
    assert h.frames_committed(0) == 0
    h.chunk_attention(0, q, k, v, out, cfg.C, 0, True, flow=good)
    torch.cuda.synchronize()
    assert h.frames_committed(0) == cfg.C and h.poll_device_status() == rkv.OK
    h.close()


def test_cfg_fused_epilogue_abot_size():
    """The guided mode at the ABot shape (24 heads, 2640 queries, 18480 keys, relative RoPE,
    five reference sinks): two caches, 7 chunks of 4 guided steps, through the first evictions.
    On the chunks after evictions start: the fused guided x0 / renoise outputs bit for bit
    against the oracle's epilogue on the stored bf16 c and u, and both branches' attention on
    sampled rows of the first and last head; both caches bit for bit at the end."""
    cfg = Config("cfg-abot", 25, H=24, grid_h=22, grid_w=40, C=3, W=21, S=5, rope_mode=REL, refs=5, chunks=7,
                 reads=4)
    steps = 4
    branches = [Rollout(cfg, rkv, torch), Rollout(replace(cfg, seed=cfg.seed + 1), rkv, torch)]
    Lq, n = cfg.Lq, cfg.Lq * cfg.H * 128
    sig = _schedule(steps)
    rows, heads = sample_rows(Lq, n=64, seed=25), [0, cfg.H - 1]
    checked = {5, 6}
    outs = [torch.empty((Lq, cfg.H, 128), dtype=torch.bfloat16, device="cuda") for _ in branches]
    for chunk in range(cfg.chunks):
        f0 = branches[0].f0[0]
        xt = _dev_bits(synth.stream_key(cfg.seed, cfg.cfg_id, 99, chunk), n)
        xt_ref = to_bits(xt) if chunk in checked else None
        for step in range(steps):
            s, sn = sig[step], sig[step + 1]
            eps = _dev_bits(synth.stream_key(cfg.seed, cfg.cfg_id, 98, chunk, step), n)
            x0 = torch.empty(n, dtype=torch.bfloat16, device="cuda")
            xn = torch.empty(n, dtype=torch.bfloat16, device="cuda")
            qkv = [[dev_tensor(torch, b.cfg, 0, chunk, step, t, Lq) for t in "qkv"] for b in branches]
            branches[0].h.chunk_attention(0, *qkv[0], outs[0], cfg.C, f0, False)
            branches[1].h.chunk_attention(0, *qkv[1], outs[1], cfg.C, f0, False,
                                          flow=dict(xt=xt, eps=eps, sigma=s, sigma_next=sn, x0_out=x0,
                                                    xt_next_out=xn if sn >= 0 else None,
                                                    v_cond=outs[0], cfg_scale=CFG_SCALE))
            torch.cuda.synchronize()
            if chunk not in checked:
                if sn >= 0:
                    xt = xn
                continue
            c_bits, u_bits = to_bits(outs[0]), to_bits(outs[1])
            rx0, rxn = oflow.cfg_x0_renoise_bf16(xt_ref, c_bits.reshape(-1), u_bits.reshape(-1), to_bits(eps),
                                                 CFG_SCALE, s, sn)
            assert np.array_equal(to_bits(x0), rx0), (chunk, step)
            if sn >= 0:
                assert np.array_equal(to_bits(xn), rxn), (chunk, step)
                xt, xt_ref = xn, rxn
            if step == 0:
                for b, got in zip(branches, (c_bits, u_bits)):
                    ref = b.oracles[0].chunk_attention(*(host_bits(b.cfg, 0, chunk, step, t, Lq) for t in "qkv"),
                                                       cfg.C, f0, False, rows=rows, heads=heads)
                    assert_close(got[rows][:, heads], ref, f"{b.cfg.name} seed {b.cfg.seed} chunk {chunk}")
        for b, out in zip(branches, outs):
            q, k, v = (dev_tensor(torch, b.cfg, 0, chunk, steps, t, Lq) for t in "qkv")
            b.h.chunk_attention(0, q, k, v, out, cfg.C, f0, True)
            b.oracles[0].write_chunk(host_bits(b.cfg, 0, chunk, steps, "k", Lq), host_bits(b.cfg, 0, chunk, steps, "v", Lq),
                                     cfg.C, f0)
            b.f0[0] = f0 + cfg.C
    torch.cuda.synchronize()
    for b in branches:
        b.check_cache(0)
        assert b.h.poll_device_status() == rkv.OK
        b.h.close()
