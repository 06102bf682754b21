"""Pins of the oracle's KL-divergence clip calibration (low-bit blog §5, the
TensorRT method: candidate clip T, P = the histogram cut at T with the tail
folded into the last kept bin, Q = P's kept mass quantized to the levels and
spread back, the T of least D_KL(P || Q) wins)."""
from fractions import Fraction

import numpy as np
import pytest

import oracle

GRID = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3), Fraction(4), Fraction(6)]


def relu_tail(n=200_000, seed=1):
    """ReLU of a Gaussian plus a Student-t(3) component: most mass near 0 and
    a long thin tail, the shape the page describes for a ReLU activation."""
    rng = np.random.default_rng(seed)
    z = rng.standard_normal(n)
    return np.maximum(0.0, z + 0.3 * rng.standard_t(3, n)).astype(np.float32)


def test_histogram_counts_every_element_into_its_bin():
    x = relu_tail(50_000, seed=2)
    x[::97] *= -1                                           # |x| is what is counted
    amax = float(np.abs(x).max())
    bins = 512
    h = oracle.abs_histogram(x, bins, amax)
    assert int(h.sum()) == x.size
    w = amax / bins
    a = np.abs(x).astype(np.float64)
    # every element lies in its bin up to the binary32 rounding of |x| * bins / amax
    b = np.minimum(bins - 1, np.floor(a / w * (1 + 1e-6)).astype(np.int64))
    lo = np.minimum(bins - 1, np.floor(a / w * (1 - 1e-6)).astype(np.int64))
    assert (np.bincount(lo, minlength=bins).cumsum() >= h.astype(np.int64).cumsum()).all()
    assert (np.bincount(b, minlength=bins).cumsum() <= h.astype(np.int64).cumsum()).all()
    assert h[bins - 1] >= 1                                 # the maximum sits in the last bin


def test_all_zero_tensor_fills_bin_zero():
    h = oracle.abs_histogram(np.zeros(100, np.float32), 64, 0.0)
    assert h[0] == 100 and h[1:].sum() == 0


def test_e2m1_level_map_is_the_nearest_magnitude_with_even_ties():
    """Brute force in exact rationals: bin b's centre maps to 6 (b + 1/2) / i;
    the level is the nearest E2M1 magnitude, ties to the even code."""
    for i in list(range(8, 130)) + [2048, 2047, 1000]:
        for b in range(i):
            v = Fraction(6 * (2 * b + 1), 2 * i)
            d = [abs(v - g) for g in GRID]
            m = min(d)
            cands = [c for c in range(8) if d[c] == m]
            want = cands[0] if len(cands) == 1 else min(c for c in cands if c % 2 == 0)
            assert oracle.e2m1_level_of_bin(b, i) == want, (b, i)


@pytest.mark.parametrize("grid,levels", [(0, 8), (0, 4), (0, 128), (1, 8)])
def test_kl_is_non_negative_and_scale_invariant(grid, levels):
    x = relu_tail(100_000, seed=3)
    h = oracle.abs_histogram(x, 2048, float(x.max()))
    best, kl = oracle.kl_calibrate(h, levels, grid)
    finite = kl[np.isfinite(kl)]
    assert (finite >= -1e-12).all() and finite.size > 0.1 * kl.size
    best7, kl7 = oracle.kl_calibrate(h * np.uint64(7), levels, grid)
    assert best7 == best
    f = np.isfinite(kl)
    assert np.allclose(kl7[f], kl[f], rtol=1e-12, atol=1e-15)


def test_kl_vanishes_when_each_level_is_already_flat():
    """A histogram constant inside every uniform level group (no tail beyond
    the last bin) is reproduced exactly by Q at i = bins: D_KL = 0 there and
    nowhere lower; moving any group boundary would break the equality."""
    levels, per = 8, 32
    h = np.repeat(np.array([50, 9, 40, 3, 11, 6, 2, 7], np.uint64), per)
    best, kl = oracle.kl_calibrate(h, levels, 0)
    assert kl[-1] == 0.0 and best == h.size
    h2 = h.copy()
    h2[per] += 1                                           # one more count at the start of level 1
    assert oracle.kl_calibrate(h2, levels, 0)[1][-1] > 0


def test_tail_mass_folds_into_the_last_kept_bin():
    """Mass beyond T lands in P's last kept bin; if that bin's level has no
    kept mass, Q is zero where P is not and the candidate is rejected."""
    h = np.zeros(64, np.uint64)
    h[:8] = 100
    h[63] = 5                                              # an outlier far out
    best, kl = oracle.kl_calibrate(h, 4, 0)
    # i = 16: levels of 4 bins; the last kept level (bins 12..15) holds no
    # kept mass but receives the outlier -> +inf
    assert np.isinf(kl[16 - 4])
    assert 0 < kl[8 - 4] < np.inf                          # i = 8: the outlier inflates P's bin 7 only
    # i = 64 keeps the outlier in a level of its own (bins 48..63): P exactly
    assert kl[-1] == 0.0 and best == 64


def test_ties_keep_the_smallest_candidate():
    h = np.zeros(256, np.uint64)
    h[0] = 1000                                             # every candidate reproduces P exactly
    best, kl = oracle.kl_calibrate(h, 8, 0)
    assert (kl == 0).all() and best == 8


@pytest.mark.parametrize("grid", [0, 1])
def test_kl_clips_inside_the_tail_of_a_relu_activation(grid):
    """[LB] §5: on a long-tailed ReLU activation the KL-optimal clip lies well
    inside the observed maximum (the page: T = 12.8 against a maximum of 19.7)
    and the KL curve rises again toward T = max (U shape)."""
    x = relu_tail()
    amax = float(x.max())
    h = oracle.abs_histogram(x, 2048, amax)
    best, kl = oracle.kl_calibrate(h, 8, grid)
    T = oracle.kl_threshold(amax, 2048, best)
    assert T < 0.5 * amax
    assert kl[-1] > 1.5 * kl.min()
    assert T == np.float32(np.float32(best) * np.float32(np.float32(amax) / np.float32(2048)))
