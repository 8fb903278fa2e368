"""Head-sharded attention for sequence-sharded callers, the multi-rank host path on CPU:
two gloo ranks run HeadShardedRollingKV.chunk_attention / write_chunk with the real
all-to-all (torch.distributed over gloo) around a per-rank oracle cache of H/2 heads.

The head-block copies that pack and unpack the exchange run on the CPU: the exact run
descriptors (pointers, strides, token counts) that HeadShardedRollingKV hands to
rkv_copy_heads are executed by a host interpreter of that call's definition (head vector
(t, h) of 128 bf16 moves from src + t * src_tok_stride + h * src_head_stride to the same
offsets in dst), a test double for the CUDA copy kernel; the per-rank attention is the fp64
oracle of that rank's heads. Checked: every rank's output block equals the oracle of all heads on that token
block (to bf16 rounding), through sinks written with write_chunk, warm-up, eviction and
wrap, in both RoPE modes; a head count the ranks do not divide is refused.
"""
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
H, GH, GW, C, W, S = 4, 4, 4, 2, 6, 2
T = GH * GW


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(chunk, call, tag, n_tok):
    """Seeded bf16 bits [n_tok, H, 128] of the whole chunk (all tokens, all heads)."""
    sys.path.insert(0, ROOT)
    import synth
    return synth.normal_bf16_bits(synth.stream_key(5, 40, chunk, call, tag), 0, n_tok * H * 128).reshape(n_tok, H, 128)


def _worker(rank, world, port, mode, q):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from oracle import bf16
    from oracle.layer import OracleLayer
    from rolling_kv_chunked_b200.sharded import HeadShardedRollingKV

    def to_bits(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    def from_bits(b):
        return torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16)

    class OracleLocal:
        """This rank's H/2 heads, fp64, rounded to bf16 on output."""
        def __init__(self, hl):
            self.orc = OracleLayer(hl, 128, T, GH, GW, W, S, mode)

        def write_chunk(self, layer, k, v, n_frames, start_frame, stream=None):
            self.orc.write_chunk(to_bits(k), to_bits(v), n_frames, start_frame)

        def chunk_attention(self, layer, q, k, v, out, n_frames, start_frame, commit, stream=None):
            ref = self.orc.chunk_attention(to_bits(q), to_bits(k), to_bits(v), n_frames, start_frame, commit)
            out.copy_(from_bits(bf16.from_f64(ref)))

    def host_copy_heads(runs, n_heads, stream=None):
        """rkv_copy_heads' definition on host memory: (src, dst, src_tok_stride, src_head_stride,
        dst_tok_stride, dst_head_stride, n_tok), strides in bf16 elements, 128-element vectors."""
        import ctypes
        for src, dst, sts, shs, dts, dhs, n_tok in runs:
            for t in range(n_tok):
                for h in range(n_heads):
                    ctypes.memmove(dst + 2 * (t * dts + h * dhs), src + 2 * (t * sts + h * shs), 2 * 128)

    hs = HeadShardedRollingKV(1, H, 128, T, W, S, mode, local=OracleLocal(H // world), copy_fn=host_copy_heads)
    full = OracleLayer(H, 128, T, GH, GW, W, S, mode)
    Lq = C * T
    Lb = Lq // world
    blk = slice(rank * Lb, (rank + 1) * Lb)
    # two reference frames become the sinks
    kr, vr = _inputs(-1, 0, 1, S * T), _inputs(-1, 0, 2, S * T)
    rb = slice(rank * (S * T // world), (rank + 1) * (S * T // world))
    hs.write_chunk(0, from_bits(kr[rb]), from_bits(vr[rb]), S, 0)
    full.write_chunk(kr, vr, S, 0)
    worst = 0.0
    f0 = S
    for chunk in range(5):
        for call in range(2):
            commit = call == 1
            qb, kb, vb = (_inputs(chunk, call, t, Lq) for t in (3, 4, 5))
            out = torch.empty((Lb, H, 128), dtype=torch.bfloat16)
            hs.chunk_attention(0, from_bits(qb[blk]), from_bits(kb[blk]), from_bits(vb[blk]), out, C, f0, commit)
            ref = full.chunk_attention(qb, kb, vb, C, f0, commit)[blk]
            got = bf16.to_f64(to_bits(out))
            err = np.abs(got - ref) - (2.0 ** -8) * np.abs(ref)
            worst = max(worst, float(err.max()))
        f0 += C
    q.put((rank, worst))
    dist.destroy_process_group()


@pytest.mark.parametrize("mode", [0, 1])
def test_head_sharded_attention_over_two_gloo_ranks(mode):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, mode, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=300) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert set(got) == {0, 1}
    assert all(w <= 1e-12 for w in got.values()), got


def test_head_count_must_split_over_ranks():
    sys.path.insert(0, ROOT)
    from rolling_kv_chunked_b200.sharded import HeadShardedRollingKV
    with pytest.raises(ValueError):
        HeadShardedRollingKV(1, 6, 128, T, W, S, 0, world_size=4, rank=0, local=object())
    hs = HeadShardedRollingKV(1, 8, 128, 15, W, S, 0, world_size=4, rank=1, local=object())
    assert hs.Hl == 2 and hs.block_tokens(4) == 15
    with pytest.raises(ValueError):
        hs.block_tokens(1)  # 15 tokens over 4 ranks
