"""Head-sharded attention on the GPU kernels: two ranks emulated in one process on one GPU.

Each emulated rank is a HeadShardedRollingKV (its own caches of H/2 heads); the phases run
with this library's kernels (rkv_copy_heads packs / unpacks the head blocks, the chunk
attention runs per rank) and the all-to-all between the ranks is done in-process by the
test (copies of the ranks' send slices; no collective, nothing waits on another rank).
At a small shape and at the ABot shape (24 heads, 880 tokens per frame, window 21 with 5
sinks), through sinks, warm-up, eviction and wrap, in both RoPE modes:

* every rank's output block is compared element by element with the fp64 oracle at the
  attention tolerance (the small shape on all heads and rows, the ABot shape on sampled
  heads of both ranks and sampled rows of every block), and the x0 / renoise step on each
  rank's latent block is bit-exact against the oracle's step on the same values;
* every output block and epilogue is also bit-identical to one unsharded RollingKV of all
  heads on the same inputs, and each rank's cache equals the unsharded cache's heads.

rkv_copy_heads against numpy slicing and its argument errors are checked as well.
"""
import numpy as np
import pytest

import synth
from oracle import flow as oflow
from oracle.layer import OracleLayer
from rollout import assert_close, sample_rows, to_bits

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import rolling_kv_chunked_b200 as rkv  # noqa: E402
from rolling_kv_chunked_b200.sharded import HeadShardedRollingKV  # noqa: E402

G = 2
# (H, grid_h, grid_w, C, W, S, chunks): a small shape, and the ABot shape through its first
# evictions (window 21 frames with 5 sinks, chunks of 3 frames of 22 x 40 tokens)
SHAPES = {"small": (4, 8, 10, 2, 6, 2, 5), "abot": (24, 22, 40, 3, 21, 5, 7)}


# heads the oracle follows at each shape (both ranks' head ranges), and rows sampled per call
ORACLE_HEADS = {"small": None, "abot": [0, 5, 11, 12, 17, 23]}


def _dev(key, shape):
    t = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    synth.fill_normal_bf16_cuda(t.data_ptr(), t.numel(), key, 0, torch.cuda.current_stream().cuda_stream)
    return t


def _host(key, n_tok, H, heads):
    """The same seeded bits on the host, [n_tok, len(heads), 128] (all heads if heads is None)."""
    if heads is None:
        return synth.normal_bf16_bits(key, 0, n_tok * H * 128).reshape(n_tok, H, 128)
    t = np.arange(n_tok, dtype=np.int64)[:, None, None]
    h = np.asarray(heads, dtype=np.int64)[None, :, None]
    c = np.arange(128, dtype=np.int64)[None, None, :]
    return synth.normal_bf16_bits_at(key, (t * H + h) * 128 + c)


def _exchange(sends):
    """All-to-all among the emulated ranks: rank j receives slice j of every rank's send."""
    return [torch.stack([sends[i][j] for i in range(G)]) for j in range(G)]


def _sharded_call(ranks, H, *tensors, n_frames):
    """Pack each rank's token blocks, exchange, and return every rank's [Lq, H/G, d] inputs."""
    per_rank = []
    for x in tensors:
        sends = [ranks[r].pack(x[r], n_frames) for r in range(G)]
        per_rank.append([t.view(-1, H // G, 128) for t in _exchange(sends)])
    return per_rank


@pytest.mark.parametrize("shape", sorted(SHAPES))
@pytest.mark.parametrize("mode", [rkv.ROPE_ABSOLUTE, rkv.ROPE_RELATIVE])
def test_two_emulated_ranks_match_oracle_and_unsharded(mode, shape):
    H, GH, GW, C, W, S, n_chunks = SHAPES[shape]
    T = GH * GW
    ranks = [HeadShardedRollingKV(1, H, 128, T, W, S, mode, world_size=G, rank=r) for r in range(G)]
    full = rkv.RollingKV(1, H, 128, T, W, S, mode)
    for h in ranks + [full]:
        h.set_rope_grid(GH, GW)
    Lq = C * T
    Lb = Lq // G
    oh = ORACLE_HEADS[shape]
    orc = OracleLayer(H if oh is None else len(oh), 128, T, GH, GW, W, S, mode)
    hsel = list(range(H)) if oh is None else oh

    def blocks(x, n_tok):
        b = n_tok // G
        return [x[r * b:(r + 1) * b].contiguous() for r in range(G)]

    # sinks written without attention
    kr, vr = _dev(synth.stream_key(6, 1), (S * T, H, 128)), _dev(synth.stream_key(6, 2), (S * T, H, 128))
    (k_in, v_in) = _sharded_call(ranks, H, blocks(kr, S * T), blocks(vr, S * T), n_frames=S)
    for r in range(G):
        ranks[r].local.write_chunk(0, k_in[r], v_in[r], S, 0)
    full.write_chunk(0, kr, vr, S, 0)
    orc.write_chunk(_host(synth.stream_key(6, 1), S * T, H, oh), _host(synth.stream_key(6, 2), S * T, H, oh), S, 0)
    f0 = S
    sig = [1.0, 0.75]
    for chunk in range(n_chunks):
        xt = _dev(synth.stream_key(6, 3, chunk), (Lq, H * 128))
        for call in range(2):
            commit = call == 1
            q, k, v = (_dev(synth.stream_key(6, 4, chunk, call, t), (Lq, H, 128)) for t in range(3))
            eps = _dev(synth.stream_key(6, 5, chunk, call), (Lq, H * 128))
            out_full = torch.empty((Lq, H, 128), dtype=torch.bfloat16, device="cuda")
            x0_full, xn_full = torch.empty_like(xt), torch.empty_like(xt)
            if commit:
                full.chunk_attention(0, q, k, v, out_full, C, f0, True)
            else:
                full.chunk_attention(0, q, k, v, out_full, C, f0, False,
                                     flow=dict(xt=xt, eps=eps, sigma=sig[0], sigma_next=sig[1],
                                               x0_out=x0_full, xt_next_out=xn_full))
            qs, ks, vs = _sharded_call(ranks, H, blocks(q, Lq), blocks(k, Lq), blocks(v, Lq), n_frames=C)
            outs_h = [ranks[r].attend(0, qs[r], ks[r], vs[r], C, f0, commit) for r in range(G)]
            back = _exchange([o.view(G, Lb, H // G, 128) for o in outs_h])
            # the oracle on the same seeded inputs (sampled rows at the ABot shape)
            rows = None if oh is None else sample_rows(Lq, n=64, seed=chunk * 2 + call)
            ref = orc.chunk_attention(*(_host(synth.stream_key(6, 4, chunk, call, t), Lq, H, oh) for t in range(3)),
                                      C, f0, commit, rows=rows)
            rows_all = np.arange(Lq) if rows is None else rows
            for r in range(G):
                out_r = torch.empty((Lb, H, 128), dtype=torch.bfloat16, device="cuda")
                ranks[r].unpack(back[r], out_r, C)
                torch.cuda.synchronize()
                got_r = to_bits(out_r)
                assert np.array_equal(got_r, to_bits(out_full[r * Lb:(r + 1) * Lb])), (mode, chunk, call, r)
                mine = (rows_all >= r * Lb) & (rows_all < (r + 1) * Lb)
                assert_close(got_r[rows_all[mine] - r * Lb][:, hsel], ref[mine],
                             f"{shape} mode {mode} chunk {chunk} call {call} rank {r} vs oracle")
                if not commit:
                    xb = xt[r * Lb:(r + 1) * Lb].contiguous()
                    eb = eps[r * Lb:(r + 1) * Lb].contiguous()
                    x0_r, xn_r = torch.empty_like(xb), torch.empty_like(xb)
                    rkv.flow_x0_renoise(xb, out_r.view(Lb, H * 128), eb, sig[0], sig[1], x0_r, xn_r)
                    torch.cuda.synchronize()
                    rx0, rxn = oflow.x0_renoise_bf16(to_bits(xb), got_r.reshape(Lb, H * 128), to_bits(eb),
                                                     sig[0], sig[1])
                    assert np.array_equal(to_bits(x0_r), rx0) and np.array_equal(to_bits(xn_r), rxn)
                    assert np.array_equal(to_bits(x0_r), to_bits(x0_full[r * Lb:(r + 1) * Lb]))
                    assert np.array_equal(to_bits(xn_r), to_bits(xn_full[r * Lb:(r + 1) * Lb]))
        f0 += C
    # each rank's cache holds exactly the unsharded cache's heads
    n_el = W * T * 128
    for which in range(2):
        fp = full.cache_ptrs(0)[which]
        full_c = torch.as_tensor(_Arr(fp, H * n_el), device="cuda").view(torch.bfloat16).view(H, W * T, 128)
        for r in range(G):
            rp = ranks[r].local.cache_ptrs(0)[which]
            rc = torch.as_tensor(_Arr(rp, (H // G) * n_el), device="cuda").view(torch.bfloat16).view(H // G, W * T, 128)
            assert np.array_equal(to_bits(rc), to_bits(full_c[r * (H // G):(r + 1) * (H // G)]))
        assert ranks[0].local.slot_frames(0) == full.slot_frames(0) == ranks[1].local.slot_frames(0)
    for h in ranks:
        h.close()
    full.close()


class _Arr:
    def __init__(self, ptr, n):
        self.__cuda_array_interface__ = {"shape": (n,), "typestr": "<i2", "data": (ptr, False), "version": 3}


def test_copy_heads_strided_blocks_and_errors():
    n_tok, Hs, Hd = 37, 6, 3   # 3 of 6 heads, ragged token count
    x = _dev(synth.stream_key(6, 9), (n_tok, Hs, 128))
    y = torch.zeros((2, n_tok, Hd, 128), dtype=torch.bfloat16, device="cuda")
    runs = [(x.data_ptr() + r * Hd * 128 * 2, y[r].data_ptr(), Hs * 128, 128, Hd * 128, 128, n_tok) for r in range(2)]
    rkv.copy_heads(runs, Hd)
    torch.cuda.synchronize()
    xb = to_bits(x)
    for r in range(2):
        assert np.array_equal(to_bits(y[r]), xb[:, r * Hd:(r + 1) * Hd, :])
    # more runs than one launch takes (nine), zero-token runs skipped
    many = [(x.data_ptr(), y[0].data_ptr(), Hs * 128, 128, Hd * 128, 128, n_tok if i % 3 else 0) for i in range(9)]
    rkv.copy_heads(many, Hd)
    torch.cuda.synchronize()
    assert np.array_equal(to_bits(y[0]), xb[:, :Hd, :])
    for bad in [(x.data_ptr() + 2, y[0].data_ptr(), Hs * 128, 128, Hd * 128, 128, 4),   # misaligned
                (x.data_ptr(), y[0].data_ptr(), Hs * 128 + 4, 128, Hd * 128, 128, 4),   # stride not a multiple of 8
                (x.data_ptr(), y[0].data_ptr(), Hs * 128, 128, Hd * 128, 128, -1)]:     # negative count
        with pytest.raises(rkv.RkvError):
            rkv.copy_heads([bad], Hd)
    with pytest.raises(rkv.RkvError):
        rkv.copy_heads(runs, 0)
