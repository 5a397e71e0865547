"""The seeded input generators (no GPU): the values depend on the seed only, never on
the number of threads that draw a large matrix, and bf16 rounding is to nearest even."""
import numpy as np

from reduced_cross_entropy_b200 import synth


def test_block_parallel_draws_do_not_depend_on_the_thread_count(monkeypatch):
    shape = (70_000, 256)  # 17.9 M elements: past the single-stream limit of 2^24
    rng = np.random.Generator(np.random.PCG64(0))
    monkeypatch.setattr(synth.os, "cpu_count", lambda: 1)
    one = synth._standard_normal(rng, 3, 1, shape)
    monkeypatch.setattr(synth.os, "cpu_count", lambda: 7)
    many = synth._standard_normal(rng, 3, 1, shape)
    assert one.dtype == np.float32 and one.shape == shape
    np.testing.assert_array_equal(one, many)
    # another seed or tag gives other values; the moments are those of N(0, 1)
    assert not np.array_equal(one[:4], synth._standard_normal(rng, 3, 0, shape)[:4])
    assert abs(float(one.mean())) < 1e-3 and abs(float(one.std()) - 1.0) < 1e-3


def test_small_matrices_come_from_the_single_stream():
    rng = np.random.Generator(np.random.PCG64(5))
    a = synth._standard_normal(rng, 5, 0, (100, 64))
    b = np.random.Generator(np.random.PCG64(5)).standard_normal((100, 64), dtype=np.float32)
    np.testing.assert_array_equal(a, b)


def test_bf16_rounding_matches_the_wide_integer_formula():
    rng = np.random.default_rng(2)
    a = np.concatenate([rng.standard_normal(100_000).astype(np.float32) * 10.0 ** e
                        for e in (-30, -3, 0, 3, 30)])
    a = np.concatenate([a, np.float32([0.0, -0.0, 3.4e38, -3.4e38, 1.0 + 2.0 ** -8,
                                       1.0 + 3 * 2.0 ** -8])])
    u = a.view(np.uint32).astype(np.uint64)
    want = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    np.testing.assert_array_equal(synth.bf16_bits(a), want)
    np.testing.assert_array_equal(synth.round_bf16(a).view(np.uint32),
                                  want.astype(np.uint32) << 16)
