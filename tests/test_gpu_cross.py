"""GPU parity of the cross-attention over the cached text K/V (through the C ABI).

* ragged and tile-aligned text lengths (1, 77, 128, 512, 600) and query counts (1 .. 3 CTAs
  with ragged tails, the second 128-row tile of a CTA absent, partial or full): every element
  within the attention tolerance of the fp64 oracle, plus a peaked-softmax case (queries x 4);
  guard rows after the output stay untouched;
* the ABot shape (H = 24, 2640 queries, 512 text tokens): all elements; the 720p shape
  (H = 40, 14400 queries): sampled rows of all heads;
* interleaved with a self-attention rollout: cross calls leave the rolling cache bit-exact,
  a new (shorter, then longer, reallocating) prompt replaces only the text K/V;
* errors: no text K/V -> RKV_ERR_STATE; oversize / misaligned -> nothing launched.
"""
import numpy as np
import pytest

import synth
from oracle.layer import OracleLayer
from rollout import Config, Rollout, assert_close, sample_rows, to_bits

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import rolling_kv_chunked_b200 as rkv  # noqa: E402


def _pair(H, n, key, scale=1.0):
    """The same seeded N(0,1) bf16 tensor [n, H, 128] on the device and as host bits."""
    bits = synth.normal_bf16_bits(key, 0, n * H * 128).reshape(n, H, 128)
    if scale != 1.0:
        from oracle import bf16
        bits = bf16.from_f64(bf16.to_f64(bits) * scale)
    dev = torch.from_numpy(bits.view(np.int16).copy()).cuda().view(torch.bfloat16)
    return dev, bits


def _oracle(H):
    return OracleLayer(H, 128, 4, 2, 2, 6, 2, OracleLayer.ABSOLUTE)


@pytest.mark.parametrize("n_text", [1, 77, 128, 512, 600])
def test_cross_small_every_element(n_text):
    H = 2
    h = rkv.RollingKV(1, H, 128, 4, 6, 2, OracleLayer.ABSOLUTE)
    kt, ktb = _pair(H, n_text, synth.stream_key(0, 70, n_text, 1))
    vt, vtb = _pair(H, n_text, synth.stream_key(0, 70, n_text, 2))
    h.set_text_kv(0, kt, vt)
    orc = _oracle(H)
    orc.set_text_kv(ktb, vtb)
    for n_q, scale in [(1, 1.0), (33, 1.0), (200, 1.0), (256, 1.0), (300, 1.0), (400, 1.0), (513, 1.0),
                       (300, 4.0)]:
        q, qb = _pair(H, n_q, synth.stream_key(0, 71, n_text, n_q), scale)
        # the output is a view followed by 80 guard rows that no store may reach
        full = torch.full((n_q + 80, H, 128), -7.0, dtype=torch.bfloat16, device="cuda")
        out = full[:n_q]
        h.cross_attention(0, q, out)
        torch.cuda.synchronize()
        assert_close(to_bits(out), orc.cross_attention(qb), f"cross n_text {n_text} n_q {n_q} x{scale}")
        assert bool((full[n_q:] == -7.0).all()), f"rows past the output written (n_text {n_text}, n_q {n_q})"
    assert h.poll_device_status() == rkv.OK
    h.close()


@pytest.mark.parametrize("shape", [("abot", 24, 2640, None), ("720p", 40, 14400, 96)])
def test_cross_full_size(shape):
    name, H, n_q, n_rows = shape
    h = rkv.RollingKV(1, H, 128, 880, 21, 5, OracleLayer.RELATIVE)
    kt, ktb = _pair(H, 512, synth.stream_key(1, 72, H, 1))
    vt, vtb = _pair(H, 512, synth.stream_key(1, 72, H, 2))
    h.set_text_kv(0, kt, vt)
    q, qb = _pair(H, n_q, synth.stream_key(1, 73, H))
    out = torch.empty_like(q)
    h.cross_attention(0, q, out)
    torch.cuda.synchronize()
    orc = OracleLayer(H, 128, 880, 22, 40, 21, 5, OracleLayer.RELATIVE)
    orc.set_text_kv(ktb, vtb)
    rows = None if n_rows is None else sample_rows(n_q, n=n_rows, seed=3)
    got = to_bits(out) if rows is None else to_bits(out)[rows]
    assert_close(got, orc.cross_attention(qb, rows=rows), f"cross {name}")
    assert h.poll_device_status() == rkv.OK
    h.close()


def test_cross_interleaved_with_rollout_and_prompt_swap():
    cfg = Config("cross-roll", 30, H=3, grid_h=8, grid_w=10, C=3, W=7, S=2, rope_mode=OracleLayer.RELATIVE,
                 refs=1, chunks=4, reads=1)
    ro = Rollout(cfg, rkv, torch)
    orc = ro.oracles[0]
    for chunk in range(cfg.chunks):
        n_text = [512, 40, 700, 700][chunk]            # shorter, then longer (reallocates)
        if chunk in (0, 1, 2):
            kt, ktb = _pair(cfg.H, n_text, synth.stream_key(2, 74, chunk, 1))
            vt, vtb = _pair(cfg.H, n_text, synth.stream_key(2, 74, chunk, 2))
            ro.h.set_text_kv(0, kt, vt)
            orc.set_text_kv(ktb, vtb)
        ro.run_chunk(0, chunk)
        q, qb = _pair(cfg.H, cfg.Lq, synth.stream_key(2, 75, chunk))
        out = torch.empty_like(q)
        ro.h.cross_attention(0, q, out)
        torch.cuda.synchronize()
        assert_close(to_bits(out), orc.cross_attention(qb), f"cross in rollout, chunk {chunk}")
        ro.check_cache(0)
    assert ro.h.poll_device_status() == rkv.OK
    ro.h.reset()
    with pytest.raises(rkv.RkvError) as e:
        ro.h.cross_attention(0, q, out)
    assert e.value.code == rkv.ERR_STATE
    ro.h.close()


def test_cross_errors_launch_nothing():
    H = 2
    h = rkv.RollingKV(2, H, 128, 4, 6, 2, OracleLayer.ABSOLUTE)
    q = torch.zeros((16, H, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.full_like(q, 7.0)
    with pytest.raises(rkv.RkvError) as e:
        h.cross_attention(0, q, out)
    assert e.value.code == rkv.ERR_STATE
    kt = torch.zeros((8, H, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rkv.RkvError) as e:
        h.set_text_kv(2, kt, kt)
    assert e.value.code == rkv.ERR_ARG
    flat = torch.zeros(8 * H * 128 + 8, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rkv.RkvError) as e:
        h.set_text_kv(0, flat[1:1 + 8 * H * 128].view(8, H, 128), kt)
    assert e.value.code == rkv.ERR_ARG
    big = torch.zeros(((1 << 16) + 1, 1, 1), dtype=torch.bfloat16, device="cuda")   # shape only is read
    with pytest.raises(rkv.RkvError) as e:
        h.set_text_kv(0, big, big)
    assert e.value.code == rkv.ERR_UNSUPPORTED
    h.set_text_kv(1, kt, kt)                           # layer 1 only: layer 0 still has none
    with pytest.raises(rkv.RkvError) as e:
        h.cross_attention(0, q, out)
    assert e.value.code == rkv.ERR_STATE
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())
    h.cross_attention(1, q, out)                       # zero keys: uniform weights, zero values
    torch.cuda.synchronize()
    assert bool((out == 0).all())
    h.close()


def test_cross_longest_text_context():
    """The largest text context the library takes (65536 tokens, 512 key tiles in one
    segment) element by element against the oracle, with a ragged query count; one more
    token is refused before anything is launched."""
    H, n_text, n_q = 1, 65536, 300
    h = rkv.RollingKV(1, H, 128, 4, 6, 2, OracleLayer.ABSOLUTE)
    kt, ktb = _pair(H, n_text, synth.stream_key(0, 74, 1))
    vt, vtb = _pair(H, n_text, synth.stream_key(0, 74, 2))
    h.set_text_kv(0, kt, vt)
    orc = _oracle(H)
    orc.set_text_kv(ktb, vtb)
    q, qb = _pair(H, n_q, synth.stream_key(0, 75))
    out = torch.empty_like(q)
    h.cross_attention(0, q, out)
    torch.cuda.synchronize()
    assert_close(to_bits(out), orc.cross_attention(qb), "cross n_text 65536")
    k2 = torch.zeros((n_text + 1, H, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rkv.RkvError):
        h.set_text_kv(0, k2, k2)
    assert h.poll_device_status() == rkv.OK
    h.close()


def test_cross_timeout_with_several_units_per_cta():
    """More query blocks than SMs (4 heads x 40 blocks of 256 queries = 160 units), so CTAs of
    the persistent short-stream kernel run two units each. A 1 ns wait cap makes waits expire
    at arbitrary points of that walk, possibly in some warps of a warpgroup and not in others:
    the call must come back with RKV_ERR_TIMEOUT, and the next call with the normal cap must
    match the oracle."""
    H, n_text, n_q = 4, 512, 40 * 256
    h = rkv.RollingKV(1, H, 128, 4, 6, 2, OracleLayer.ABSOLUTE)
    kt, ktb = _pair(H, n_text, synth.stream_key(0, 76, 1))
    vt, vtb = _pair(H, n_text, synth.stream_key(0, 76, 2))
    h.set_text_kv(0, kt, vt)
    q, qb = _pair(H, n_q, synth.stream_key(0, 76, 3))
    out = torch.zeros_like(q)
    h.set_wait_limit(1)
    for _ in range(3):
        h.cross_attention(0, q, out)
        assert h.poll_device_status() == rkv.ERR_TIMEOUT
    h.set_wait_limit(2_000_000_000)
    h.cross_attention(0, q, out)
    assert h.poll_device_status() == rkv.OK
    orc = _oracle(H)
    orc.set_text_kv(ktb, vtb)
    rows = np.arange(0, n_q, 37)
    got = to_bits(out)[rows]
    want = orc.cross_attention(qb[rows])
    assert_close(got, want, "after timeouts")
    h.close()
