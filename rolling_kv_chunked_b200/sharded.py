"""Head-sharded rolling-window attention over several GPUs, for callers that hold the chunk's
tokens split by rank (sequence parallelism).

The pages run the distilled model on several GPUs with Ulysses sequence parallelism: the
attention forward is wrapped so that an all-to-all turns token shards into head shards
before attention and back after it, which needs the GPU count to divide the head count
(LingBot-World 2.0 `wan/` source-map article, §多卡加速; "从40步到4步…", §并行加速,
``--ulysses_size 8``). Here each of the g ranks keeps the rolling caches of its own H/g heads
(heads [r H/g, (r + 1) H/g) on rank r), so the attention itself exchanges nothing; only the
chunk's q / k / v and the output cross the interconnect:

1. rank r holds tokens [r Lq/g, (r + 1) Lq/g) of every head of q, k, v ([Lq/g, H, d]);
   ``rkv_copy_heads`` packs them by destination rank, [g, Lq/g, H/g, d];
2. one all-to-all per tensor (NCCL over NVLink) gives every rank all Lq tokens of its heads,
   token-major [Lq, H/g, d], which is the layout the single-GPU path takes;
3. the rank's own kernels run the chunk attention (and the commit) for its heads;
4. one all-to-all returns to every rank its token block of every head, and
   ``rkv_copy_heads`` unpacks it to [Lq/g, H, d];
5. the x0 / renoise epilogue, elementwise, runs on each rank's token block of the latent.

The phases are separate methods so that the exchange can be driven by a caller that owns
the ranks itself; ``chunk_attention`` composes them with ``torch.distributed`` collectives.
Every step that touches the data runs in this library's kernels or in NCCL; there is no
host or CPU path.
"""
from __future__ import annotations

import torch

from . import RollingKV, copy_heads, flow_x0_renoise

HEAD_DIM = 128


class HeadShardedRollingKV:
    def __init__(self, layers: int, H: int, d: int, tokens_per_frame: int, window_frames: int,
                 sink_frames: int, rope_mode: int, group=None, world_size: int | None = None,
                 rank: int | None = None, local=None, copy_fn=None):
        """One rank of g. ``world_size`` / ``rank`` default to the process group's; ``local`` is
        the per-rank cache of H/g heads (by default a RollingKV with this library's kernels);
        ``copy_fn(runs, n_heads, stream)`` executes the strided head-block copies that ``pack``
        and ``unpack`` describe (by default ``rkv_copy_heads``)."""
        import torch.distributed as dist
        if d != HEAD_DIM:
            raise ValueError("head dimension must be 128")
        self.group = group
        self.g = world_size if world_size is not None else dist.get_world_size(group)
        self.rank = rank if rank is not None else dist.get_rank(group)
        if H % self.g != 0:
            raise ValueError(f"the rank count {self.g} must divide the head count {H}")
        self.H, self.Hl, self.d, self.T = H, H // self.g, d, tokens_per_frame
        self.local = local if local is not None else RollingKV(layers, self.Hl, d, tokens_per_frame,
                                                               window_frames, sink_frames, rope_mode)
        self.copy_fn = copy_fn if copy_fn is not None else copy_heads

    # ------------------------------------------------------------------ setup
    def set_rope_grid(self, grid_h: int, grid_w: int, theta: float = 1.0e4, pairs=(22, 21, 21)) -> None:
        self.local.set_rope_grid(grid_h, grid_w, theta, pairs)

    def close(self) -> None:
        self.local.close()

    # ------------------------------------------------------------------ phases
    def block_tokens(self, n_frames: int) -> int:
        n = n_frames * self.T
        if n % self.g != 0:
            raise ValueError(f"the chunk's {n} tokens do not split evenly over {self.g} ranks")
        return n // self.g

    def pack(self, x: torch.Tensor, n_frames: int, stream=None) -> torch.Tensor:
        """[Lq/g, H, d] token block of all heads -> [g, Lq/g, H/g, d], slice r = rank r's heads."""
        Lb = self.block_tokens(n_frames)
        if tuple(x.shape) != (Lb, self.H, self.d) or not x.is_contiguous():
            raise ValueError(f"expected a contiguous [{Lb}, {self.H}, {self.d}] token block")
        send = torch.empty((self.g, Lb, self.Hl, self.d), dtype=x.dtype, device=x.device)
        es = x.element_size()
        runs = [(x.data_ptr() + r * self.Hl * self.d * es, send[r].data_ptr(), self.H * self.d, self.d,
                 self.Hl * self.d, self.d, Lb) for r in range(self.g)]
        self.copy_fn(runs, self.Hl, stream)
        return send

    def unpack(self, recv: torch.Tensor, out: torch.Tensor, n_frames: int, stream=None) -> None:
        """[g, Lq/g, H/g, d] (slice r = rank r's heads of this token block) -> out [Lq/g, H, d]."""
        Lb = self.block_tokens(n_frames)
        if tuple(out.shape) != (Lb, self.H, self.d) or not out.is_contiguous():
            raise ValueError(f"expected a contiguous [{Lb}, {self.H}, {self.d}] output block")
        es = out.element_size()
        runs = [(recv[r].data_ptr(), out.data_ptr() + r * self.Hl * self.d * es, self.Hl * self.d, self.d,
                 self.H * self.d, self.d, Lb) for r in range(self.g)]
        self.copy_fn(runs, self.Hl, stream)

    def attend(self, layer: int, q_heads, k_heads, v_heads, n_frames: int, start_frame: int, commit: bool,
               stream=None) -> torch.Tensor:
        """The chunk attention (and commit) of this rank's heads on all Lq tokens, [Lq, H/g, d]."""
        out = torch.empty_like(q_heads)
        self.local.chunk_attention(layer, q_heads, k_heads, v_heads, out, n_frames, start_frame, commit, stream)
        return out

    # ------------------------------------------------------------------ collectives
    def _all_to_all(self, send: torch.Tensor) -> torch.Tensor:
        """[g, ...] slices to ranks 0..g-1 -> [g, ...] slices from ranks 0..g-1."""
        import torch.distributed as dist
        recv = torch.empty_like(send)
        dist.all_to_all_single(recv, send, group=self.group)
        return recv

    def write_chunk(self, layer: int, k, v, n_frames: int, start_frame: int, stream=None) -> None:
        """Frames written without attention (e.g. the reference views that become sinks), given
        as this rank's token block of all heads."""
        kh = self._all_to_all(self.pack(k, n_frames, stream)).view(-1, self.Hl, self.d)
        vh = self._all_to_all(self.pack(v, n_frames, stream)).view(-1, self.Hl, self.d)
        self.local.write_chunk(layer, kh, vh, n_frames, start_frame, stream)

    def chunk_attention(self, layer: int, q, k, v, out, n_frames: int, start_frame: int, commit: bool,
                        stream=None, flow: dict | None = None) -> None:
        """out (this rank's [Lq/g, H, d] token block) = the chunk attention of that block; ``flow``
        (xt, eps, sigma, sigma_next, x0_out, xt_next_out on this rank's [Lq/g, H * d] latent block)
        adds the x0 / renoise step on it."""
        qh, kh, vh = (self._all_to_all(self.pack(t, n_frames, stream)).view(-1, self.Hl, self.d)
                      for t in (q, k, v))
        oh = self.attend(layer, qh, kh, vh, n_frames, start_frame, commit, stream)
        recv = self._all_to_all(oh.view(self.g, -1, self.Hl, self.d))
        self.unpack(recv, out, n_frames, stream)
        if flow is not None:
            flow_x0_renoise(flow["xt"], out.view(flow["xt"].shape), flow.get("eps"), flow["sigma"],
                            flow["sigma_next"], flow["x0_out"], flow.get("xt_next_out"), stream)
