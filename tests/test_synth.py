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


def test_config_recipes():
    """Shapes, scales and structure of every workload recipe."""
    f = synth.bf16_bits_to_f32
    w1, x1 = synth.cfg1_W(), synth.cfg1_X()
    assert w1.shape == (256, 784) and w1.dtype == np.float32 and abs(w1.std() - 0.04) < 0.002
    assert x1.shape == (64, 784) and abs(x1.std() - 1) < 0.02
    x3 = f(synth.cfg3_X(1024, 1024)).astype(np.float64)
    assert abs(np.median(np.abs(x3)) - 0.5 * 0.765) < 0.03           # 0.5 * median |t3| (0.765)
    assert ((x3 - x3.mean()) ** 4).mean() / x3.var() ** 2 > 8        # heavy tails (t3 has no finite kurtosis)
    assert abs(f(synth.cfg3_W(512, 1024)).std() - 0.02) < 0.001
    assert abs(f(synth.cfg4_W(512, 1024)).std() - 0.02) < 0.001
    for K, count in ((4096, 20), (14336, 72)):
        a = f(synth.cfg5_A(64, K))
        cols = synth.outlier_columns(K, count, 1005)
        assert len(set(cols.tolist())) == count == int(round(0.005 * K))
        ratio = np.abs(a[:, cols]).mean() / np.abs(np.delete(a, cols, axis=1)).mean()
        assert 25 < ratio < 35                                       # x30 channels
    b = f(synth.cfg5_B(256, 1024))
    assert abs(b.std() - 1) < 0.02
    r = f(synth.relu_activation(256, 1024))
    assert r.min() == 0 and (r == 0).mean() > 0.3 and r.max() > 6 * np.median(r[r > 0])
    u = synth.uniform(1 << 16, 9)
    assert u.min() > 0 and u.max() < 1 and abs(u.mean() - 0.5) < 0.01
