"""The seeded input generator: reproducible, right shapes and distributions."""
import numpy as np

import synth


def test_reproducible_and_seed_dependent():
    a = synth.gaussian_bf16(64, 128, seed=1)
    assert (a == synth.gaussian_bf16(64, 128, seed=1)).all()
    assert (a != synth.gaussian_bf16(64, 128, seed=2)).any()
    # chunked (threaded) generation equals one-shot generation
    n = (1 << 22) + 1000
    z = synth.normal(n, 3)
    assert np.array_equal(z[-1000:], synth._normal_chunk(synth._key(3, 0), n - 1000, 1000))


def test_distributions():
    z = synth.normal(1 << 20, 5)
    assert abs(z.mean()) < 5e-3 and abs(z.std() - 1) < 5e-3
    x = synth.bf16_bits_to_f32(synth.cfg2_X(256, 4096))
    cols = synth.outlier_columns(4096, 40, 1002)
    assert len(set(cols.tolist())) == 40
    big = np.abs(x[:, cols]).mean() / np.abs(np.delete(x, cols, axis=1)).mean()
    assert 15 < big < 25                                     # x20 channels
    g = synth.bf16_bits_to_f32(synth.cfg4_G(512, 512))
    assert 0.0005 < (np.abs(g) > 0.02).mean() < 0.0015       # ~0.1% entries x100


def test_bf16_rounding_is_nearest_even():
    v = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5], np.float32)
    assert synth.f32_to_bf16_bits(v).tolist() == [0x3F80, 0x3F80, 0x3F82, 0xC020]
