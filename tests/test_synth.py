"""The seeded input generator (CPU side): SplitMix64 test vector, scalar == vectorised,
sub-range consistency, and the moments of the Irwin-Hall normal stand-in."""
import numpy as np

import synth


def test_splitmix64_published_vector():
    # SplitMix64 with state seeded to 1234567: the first five outputs of the reference generator
    seed = 1234567
    got = [synth.mix64_int(seed + i * synth.GOLDEN) for i in range(1, 6)]
    assert got == [6457827717110365317, 3203168211198807973, 9817491932198370423,
                   4593380528125082431, 16408922859458223821]


def _scalar(key, n):
    s = 0
    for r in range(3):
        w = synth.mix64_int(key + (3 * n + r + 1) * synth.GOLDEN)
        s += sum((w >> (16 * lane)) & 0xFFFF for lane in range(4))
    x = np.float32((s - 393210) / 65536.0)
    u = int(np.array([x], dtype=np.float32).view(np.uint32)[0])
    return (u + 0x7FFF + ((u >> 16) & 1)) >> 16


def test_vectorised_equals_scalar_definition():
    key = synth.stream_key(3, 1, 2, 3)
    v = synth.normal_bf16_bits(key, 1000, 64)
    assert [int(b) for b in v] == [_scalar(key, 1000 + i) for i in range(64)]


def test_subranges_are_consistent_and_keys_differ():
    key = synth.stream_key(0, 7)
    full = synth.normal_bf16_bits(key, 0, 5000, block=1024)
    assert np.array_equal(full[1234:2345], synth.normal_bf16_bits(key, 1234, 1111))
    other = synth.normal_bf16_bits(synth.stream_key(0, 8), 0, 5000)
    assert np.mean(full == other) < 0.05


def test_moments():
    b = synth.normal_bf16_bits(synth.stream_key(1), 0, 200000).astype(np.uint32) << 16
    x = b.view(np.float32).astype(np.float64)
    assert abs(x.mean()) < 0.01
    assert abs(x.var() - 1.0) < 0.02
    assert np.all(np.abs(x) <= 6.0)


def test_indexed_form_matches_contiguous():
    key = synth.stream_key(4, 2)
    full = synth.normal_bf16_bits(key, 0, 30000)
    idx = np.array([[0, 7, 29999], [12345, 3, 3]])
    assert np.array_equal(synth.normal_bf16_bits_at(key, idx), full[idx])
