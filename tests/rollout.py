"""Side-by-side rollout driver for the GPU parity tests: the library (through the
C ABI) and the oracle run the same chunk schedule on the same seeded inputs.

Inputs: every tensor of every call comes from the ``synth`` generator keyed by
(seed, config id, layer, chunk, call, tensor tag); the GPU side fills device
buffers with the CUDA twin, the oracle side draws the same bits with numpy.
Per chunk: ``reads`` denoise reads (commit=0), then one commit (the t=0 pass).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

import synth
from oracle import bf16
from oracle.layer import OracleLayer

# tolerance of the attention output against the fp64 oracle (bf16 output, N(0,1) inputs)
MAX_ABS = 1.5e-2
MEAN_ABS = 1.0e-3
REL_RMS = 1.0e-2


@dataclass
class Config:
    name: str
    cfg_id: int
    H: int
    grid_h: int
    grid_w: int
    C: int
    W: int
    S: int
    rope_mode: int
    refs: int = 0          # reference frames written with write_chunk before the chunks (become sinks)
    # compare with the oracle's output rounded to bf16 (shapes with a handful of visible keys,
    # whose O(1) outputs put bf16's own rounding at the size of the mean bound)
    ref_bf16: bool = False
    # queries multiplied by this power of two (exact in bf16): a peaked softmax, checked by the
    # relative bounds (the absolute ones are stated for N(0,1) inputs)
    q_scale: float = 1.0
    chunks: int = 4
    reads: int = 4
    layers: int = 1
    seed: int = 0

    @property
    def T(self):
        return self.grid_h * self.grid_w

    @property
    def Lq(self):
        return self.C * self.T


def key(cfg: Config, layer: int, chunk: int, call: int, tag: str) -> int:
    return synth.stream_key(cfg.seed, cfg.cfg_id, layer, chunk, call, synth.TAG[tag])


def host_bits(cfg, layer, chunk, call, tag, n_tok):
    return synth.normal_bf16_bits(key(cfg, layer, chunk, call, tag), 0, n_tok * cfg.H * 128).reshape(
        n_tok, cfg.H, 128)


def dev_tensor(torch, cfg, layer, chunk, call, tag, n_tok, out=None):
    t = out if out is not None else torch.empty((n_tok, cfg.H, 128), dtype=torch.bfloat16, device="cuda")
    synth.fill_normal_bf16_cuda(t.data_ptr(), t.numel(), key(cfg, layer, chunk, call, tag), 0,
                                torch.cuda.current_stream().cuda_stream)
    return t


def to_bits(t) -> np.ndarray:
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def compare(out_bits: np.ndarray, ref: np.ndarray):
    """Error statistics of a bf16 GPU result against the fp64 oracle."""
    got = bf16.to_f64(out_bits)
    err = np.abs(got - ref)
    rms_ref = float(np.sqrt(np.mean(ref ** 2)))
    rel = float(np.sqrt(np.mean(err ** 2)) / rms_ref) if rms_ref > 0 else 0.0
    return float(err.max()), float(err.mean()), rel


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of the bf16 values at |x| (normal range): 2^(floor(log2 |x|) - 7)."""
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -126)))
    return np.ldexp(1.0, (e - 7).astype(np.int64))


def assert_close_peaked(out_bits, ref, ref_q, ref_q_abs, what=""):
    """A peaked softmax (queries scaled up). Against the exact oracle (ref): relative RMS error
    <= 1e-2 of its RMS, the relative check the absolute bounds give way to outside N(0,1)
    inputs. Against the oracle fed the rotated queries and keys rounded to bf16, as the tensor
    core receives them (ref_q; ref_q_abs the same read with |V|): mean error <= 1e-3 and every
    element within max(1.5e-2, 2^-5 sum_j p_j |v_j|). That covers rounding each weight (P) and
    the output to bf16 (2^-8 together) and the rare rotated element that the kernel's fp32
    rotation rounds to the neighbouring bf16 value of the oracle's fp64 one (at queries x 4 a
    score moves by up to ~0.01, a weight by ~1 %). With scores this large the bf16 rounding
    of the rotated operands alone moves the exact result by ~2.5e-2."""
    got = bf16.to_f64(out_bits)
    _, _, rel = compare(out_bits, ref)
    e = np.abs(got - ref_q)
    bad = e > np.maximum(MAX_ABS, 2.0 ** -5 * ref_q_abs)
    assert rel <= REL_RMS and not bad.any() and e.mean() <= MEAN_ABS, (
        f"{what}: rel {rel:.3e} vs exact; vs bf16 operands: {int(bad.sum())} elements beyond the bound, "
        f"max {e.max():.3e} mean {e.mean():.3e}")
    return float(e.max()), float(e.mean()), rel


def assert_close(out_bits, ref, what="", ref_bf16=False):
    """The tolerance of the attention outputs. With ref_bf16 (shapes where a query sees only a
    few keys, so the outputs are of order one) the oracle's value is first rounded to bf16
    (nearest even), since the format's own rounding of the exact value averages about 2^-9 of
    it, the size of the mean bound; and an element may then differ from that rounded value by
    one bf16 step at its magnitude when that step exceeds the absolute bound (outputs of 2 and
    more)."""
    if ref_bf16:
        ref = bf16.to_f64(bf16.from_f64(ref))
        got = bf16.to_f64(out_bits)
        allowed = np.maximum(MAX_ABS, bf16_ulp(ref))
        bad = np.abs(got - ref) > allowed
        assert not bad.any(), f"{what}: {int(bad.sum())} elements beyond max(1.5e-2, one bf16 step)"
        mx, mean, rel = compare(out_bits, ref)
        assert mean <= MEAN_ABS and rel <= REL_RMS, f"{what}: max {mx:.3e} mean {mean:.3e} rel {rel:.3e}"
        return mx, mean, rel
    mx, mean, rel = compare(out_bits, ref)
    assert mx <= MAX_ABS and mean <= MEAN_ABS and rel <= REL_RMS, f"{what}: max {mx:.3e} mean {mean:.3e} rel {rel:.3e}"
    return mx, mean, rel


def cache_logical_bits(lib_h, torch, cfg: Config, layer: int):
    """The library's raw K/V ring read back in logical (frame) order, token-major [n*T, H, d]."""
    frames = lib_h.slot_frames(layer)
    kp, vp = lib_h.cache_ptrs(layer)
    n_el = cfg.H * cfg.W * cfg.T * 128
    k_all = _wrap(torch, kp, n_el).view(cfg.H, cfg.W * cfg.T, 128)
    v_all = _wrap(torch, vp, n_el).view(cfg.H, cfg.W * cfg.T, 128)
    held = sorted((f, s) for s, f in enumerate(frames) if f >= 0)
    ks, vs = [], []
    for f, s in held:
        ks.append(k_all[:, s * cfg.T:(s + 1) * cfg.T, :].permute(1, 0, 2))
        vs.append(v_all[:, s * cfg.T:(s + 1) * cfg.T, :].permute(1, 0, 2))
    if not held:
        z = np.zeros((0, cfg.H, 128), dtype=np.uint16)
        return [], z, z
    return [f for f, _ in held], to_bits(torch.cat(ks)), to_bits(torch.cat(vs))


class _CudaArray:
    def __init__(self, ptr, n):
        self.__cuda_array_interface__ = {"shape": (n,), "typestr": "<i2", "data": (ptr, False), "version": 3}


def _wrap(torch, ptr, n):
    return torch.as_tensor(_CudaArray(ptr, n), device="cuda").view(torch.bfloat16)


@dataclass
class Rollout:
    """Drives one config on both sides. ``check(chunk, call)`` decides which calls are compared
    (returns None to skip, or (rows, heads) to compare those; rows/heads None = all)."""
    cfg: Config
    lib: object
    torch: object
    oracles: list = field(default_factory=list)

    def __post_init__(self):
        import rolling_kv_chunked_b200 as rkv
        c = self.cfg
        self.h = rkv.RollingKV(c.layers, c.H, 128, c.T, c.W, c.S, c.rope_mode)
        self.h.set_rope_grid(c.grid_h, c.grid_w, 1.0e4, (22, 21, 21))
        self.oracles = [OracleLayer(c.H, 128, c.T, c.grid_h, c.grid_w, c.W, c.S, c.rope_mode)
                        for _ in range(c.layers)]
        # peaked configs: a shadow oracle holding |V| (sign bits cleared) for sum_j p_j |v_j|
        self.abs_oracles = ([OracleLayer(c.H, 128, c.T, c.grid_h, c.grid_w, c.W, c.S, c.rope_mode)
                             for _ in range(c.layers)] if c.q_scale != 1.0 else None)
        self.f0 = [0] * c.layers
        if c.refs:
            for layer in range(c.layers):
                k = dev_tensor(self.torch, c, layer, -1, 0, "k", c.refs * c.T)
                v = dev_tensor(self.torch, c, layer, -1, 0, "v", c.refs * c.T)
                self.h.write_chunk(layer, k, v, c.refs, 0)
                kb, vb = host_bits(c, layer, -1, 0, "k", c.refs * c.T), host_bits(c, layer, -1, 0, "v", c.refs * c.T)
                self.oracles[layer].write_chunk(kb, vb, c.refs, 0)
                if self.abs_oracles is not None:
                    self.abs_oracles[layer].write_chunk(kb, vb & np.uint16(0x7FFF), c.refs, 0)
                self.f0[layer] = c.refs

    def run_chunk(self, layer, chunk, check=lambda chunk, call: (None, None), stats=None):
        c, torch = self.cfg, self.torch
        f0 = self.f0[layer]
        out = torch.empty((c.Lq, c.H, 128), dtype=torch.bfloat16, device="cuda")
        for call in range(c.reads + 1):
            commit = call == c.reads
            q = dev_tensor(torch, c, layer, chunk, call, "q", c.Lq)
            if c.q_scale != 1.0:
                q.mul_(c.q_scale)
            k = dev_tensor(torch, c, layer, chunk, call, "k", c.Lq)
            v = dev_tensor(torch, c, layer, chunk, call, "v", c.Lq)
            self.h.chunk_attention(layer, q, k, v, out, c.C, f0, commit)
            sel = check(chunk, call)
            orc = self.oracles[layer]
            if sel is None:
                if commit:
                    kb_, vb_ = host_bits(c, layer, chunk, call, "k", c.Lq), host_bits(c, layer, chunk, call, "v", c.Lq)
                    orc.write_chunk(kb_, vb_, c.C, f0)
                    if self.abs_oracles is not None:
                        self.abs_oracles[layer].write_chunk(kb_, vb_ & np.uint16(0x7FFF), c.C, f0)
                continue
            rows, heads = sel
            qb = host_bits(c, layer, chunk, call, "q", c.Lq)
            ref_q = ref_q_abs = None
            if c.q_scale != 1.0:
                qb = bf16.from_f64(bf16.to_f64(qb) * c.q_scale)
                kb_, vb_ = host_bits(c, layer, chunk, call, "k", c.Lq), host_bits(c, layer, chunk, call, "v", c.Lq)
                # a read (no state change) with bf16 rotated operands, and the same call on the
                # |V| shadow (which commits along with the main oracle)
                ref_q = orc.chunk_attention(qb, kb_, vb_, c.C, f0, False, rows=rows, heads=heads,
                                            rope_out_bf16=True)
                ref_q_abs = self.abs_oracles[layer].chunk_attention(qb, kb_, vb_ & np.uint16(0x7FFF), c.C, f0,
                                                                    commit, rows=rows, heads=heads,
                                                                    rope_out_bf16=True)
            ref = orc.chunk_attention(qb,
                                      host_bits(c, layer, chunk, call, "k", c.Lq),
                                      host_bits(c, layer, chunk, call, "v", c.Lq), c.C, f0, commit,
                                      rows=rows, heads=heads)
            got = to_bits(out)
            if rows is not None:
                got = got[np.asarray(rows)]
            if heads is not None:
                got = got[:, np.asarray(heads)]
            what = f"{c.name} layer {layer} chunk {chunk} call {call}"
            r = (assert_close_peaked(got, ref, ref_q, ref_q_abs, what) if c.q_scale != 1.0
                 else assert_close(got, ref, what, c.ref_bf16))
            if stats is not None:
                stats.append(r)
        self.f0[layer] = f0 + c.C

    def check_cache(self, layer):
        c = self.cfg
        frames, kb, vb = cache_logical_bits(self.h, self.torch, c, layer)
        orc = self.oracles[layer]
        assert frames == orc.logical_frames()
        ok, ov = orc.logical_kv_bits()
        assert np.array_equal(kb, ok) and np.array_equal(vb, ov)
        S, R = c.S, c.W - c.S
        for s, f in enumerate(self.h.slot_frames(layer)):
            if f >= 0:
                assert s == (f if f < S else S + (f - S) % R)
        assert self.h.frames_committed(layer) == self.f0[layer]


def host_bits_heads(cfg: Config, layer, chunk, call, tag, n_tok, heads):
    """bits of the selected heads only, [n_tok, len(heads), 128] (element (t, h, c) of the
    full [n_tok, H, 128] tensor sits at index (t * H + h) * 128 + c of its stream)."""
    t = np.arange(n_tok, dtype=np.int64)[:, None, None]
    h = np.asarray(heads, dtype=np.int64)[None, :, None]
    c = np.arange(128, dtype=np.int64)[None, None, :]
    return synth.normal_bf16_bits_at(key(cfg, layer, chunk, call, tag), (t * cfg.H + h) * 128 + c)


class SampledRollout:
    """Full-size rollout: the library runs every head, the oracle the sampled heads only
    (heads never interact), so the oracle's cost stays in seconds at the real sizes."""

    def __init__(self, cfg: Config, torch, heads, layer=0):
        import rolling_kv_chunked_b200 as rkv
        self.cfg, self.torch, self.heads, self.layer = cfg, torch, list(heads), layer
        c = cfg
        self.h = rkv.RollingKV(c.layers, c.H, 128, c.T, c.W, c.S, c.rope_mode)
        self.h.set_rope_grid(c.grid_h, c.grid_w, 1.0e4, (22, 21, 21))
        self.orc = OracleLayer(len(self.heads), 128, c.T, c.grid_h, c.grid_w, c.W, c.S, c.rope_mode)
        self.f0 = 0
        if c.refs:
            k = dev_tensor(torch, c, layer, -1, 0, "k", c.refs * c.T)
            v = dev_tensor(torch, c, layer, -1, 0, "v", c.refs * c.T)
            self.h.write_chunk(layer, k, v, c.refs, 0)
            self.orc.write_chunk(host_bits_heads(c, layer, -1, 0, "k", c.refs * c.T, self.heads),
                                 host_bits_heads(c, layer, -1, 0, "v", c.refs * c.T, self.heads), c.refs, 0)
            self.f0 = c.refs

    def run_chunk(self, chunk, rows=None, stats=None):
        """All calls of one chunk; with ``rows`` the first read and the commit are compared
        on those query rows of the sampled heads."""
        c, torch = self.cfg, self.torch
        out = torch.empty((c.Lq, c.H, 128), dtype=torch.bfloat16, device="cuda")
        for call in range(c.reads + 1):
            commit = call == c.reads
            q, k, v = (dev_tensor(torch, c, self.layer, chunk, call, t, c.Lq) for t in ("q", "k", "v"))
            self.h.chunk_attention(self.layer, q, k, v, out, c.C, self.f0, commit)
            if rows is not None and call in (0, c.reads):
                qb, kb, vb = (host_bits_heads(c, self.layer, chunk, call, t, c.Lq, self.heads) for t in ("q", "k", "v"))
                ref = self.orc.chunk_attention(qb, kb, vb, c.C, self.f0, commit, rows=rows)
                got = to_bits(out)[np.asarray(rows)][:, self.heads]
                r = assert_close(got, ref, f"{c.name} chunk {chunk} call {call}")
                if stats is not None:
                    stats.append(r)
            elif commit:
                self.orc.write_chunk(host_bits_heads(c, self.layer, chunk, call, "k", c.Lq, self.heads),
                                     host_bits_heads(c, self.layer, chunk, call, "v", c.Lq, self.heads), c.C, self.f0)
        self.f0 += c.C

    def check_cache(self):
        c, torch = self.cfg, self.torch
        frames = self.h.slot_frames(self.layer)
        kp, vp = self.h.cache_ptrs(self.layer)
        n_el = c.H * c.W * c.T * 128
        hs = torch.tensor(self.heads, device="cuda")
        k_all = _wrap(torch, kp, n_el).view(c.H, c.W * c.T, 128).index_select(0, hs)
        v_all = _wrap(torch, vp, n_el).view(c.H, c.W * c.T, 128).index_select(0, hs)
        held = sorted((f, s) for s, f in enumerate(frames) if f >= 0)
        assert [f for f, _ in held] == self.orc.logical_frames()
        ok, ov = self.orc.logical_kv_bits()
        kb = to_bits(torch.cat([k_all[:, s * c.T:(s + 1) * c.T].permute(1, 0, 2) for _, s in held]))
        vb = to_bits(torch.cat([v_all[:, s * c.T:(s + 1) * c.T].permute(1, 0, 2) for _, s in held]))
        assert np.array_equal(kb, ok) and np.array_equal(vb, ov)
        S, R = c.S, c.W - c.S
        for s, f in enumerate(frames):
            if f >= 0:
                assert s == (f if f < S else S + (f - S) % R)
        assert self.h.frames_committed(self.layer) == self.f0


def sample_rows(Lq, n=96, seed=0):
    """Random query rows plus the edges of every 128-row tile and of the chunk."""
    rng = np.random.default_rng(seed)
    edges = {0, 1, Lq - 2, Lq - 1}
    for b in range(128, Lq, 128):
        edges.update({b - 1, b})
    rows = set(rng.choice(Lq, size=min(n, Lq), replace=False).tolist()) | {e for e in edges if 0 <= e < Lq}
    return np.array(sorted(rows))
