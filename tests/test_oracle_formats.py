"""Pins of the oracle's element formats, scale rule, Philox and FWHT.

Each test checks the oracle against something other than itself: values the
pages print (tests/golden), published known-answer vectors, a library
conversion (torch float8 / scipy Hadamard), closed forms and brute force.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [l.split() for l in f if l.strip() and not l.startswith("#")]


# --------------------------------------------------------------------- E2M1
def test_e2m1_grid_is_the_pages_15_values():
    rows = {r[0].rstrip(":"): r[1:] for r in _golden_lines("e2m1_grid.txt")}
    page = sorted(float(v) for v in rows["values"])
    decoded = [oracle.e2m1_value(c) for c in range(16)]
    assert len(set(decoded)) == 15                      # +0 and -0 coincide
    assert sorted(set(decoded)) == page
    pos = sorted(v for v in set(decoded) if v >= 0)
    assert pos[1] - pos[0] == float(rows["spacing_near_zero"][0])
    assert pos[-1] - pos[-2] == float(rows["spacing_at_top"][0])
    assert (min(decoded), max(decoded)) == tuple(float(v) for v in rows["range"])
    # sign bit is bit 3 and flips the value
    for c in range(8):
        assert oracle.e2m1_value(c | 8) == -oracle.e2m1_value(c)


def test_e2m1_rne_tie_table():
    # midpoints between neighbours go to the code with mantissa bit 0
    ties = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for v, want in ties.items():
        assert oracle.e2m1_value(oracle.e2m1_rne(v)) == want
        assert oracle.e2m1_value(oracle.e2m1_rne(-v)) == -want
    assert oracle.e2m1_rne(7.0) == 7 and oracle.e2m1_rne(-1e30) == 15       # saturate to +-6
    assert oracle.e2m1_rne(-0.0) == 8 and oracle.e2m1_rne(-0.1) == 8        # sign copied


def test_e2m1_rne_is_nearest_bruteforce():
    rng = np.random.default_rng(0)
    grid = np.array([oracle.e2m1_value(c) for c in range(8)], np.float64)
    vals = list(rng.uniform(-8, 8, 4000).astype(np.float32))
    for g in grid:                                       # neighbours of every midpoint
        for d in (-1e-6, 0.0, 1e-6):
            vals.append(np.float32(g + 0.25 + d))
    for v in vals:
        c = oracle.e2m1_rne(float(v))
        a = abs(float(v))
        d = np.abs(grid - a)
        assert abs(abs(oracle.e2m1_value(c)) - a) == d.min()
        assert (c >> 3) == (1 if math.copysign(1, v) < 0 else 0)


def test_e2m1_sr_rule():
    grid = [oracle.e2m1_value(c) for c in range(8)]
    for c, g in enumerate(grid):                         # grid values are exact for any word
        for r in (0, 0x12345678, 0xFFFFFFFF):
            assert oracle.e2m1_sr(g, r) == c
    # v = 2.5 lies halfway between 2 and 3: p = 1/2, u = (r>>8)*2^-24
    half = 1 << 31                                       # u = 0.5 exactly -> not up
    assert oracle.e2m1_value(oracle.e2m1_sr(2.5, half)) == 2.0
    assert oracle.e2m1_value(oracle.e2m1_sr(2.5, half - 256)) == 3.0
    assert oracle.e2m1_value(oracle.e2m1_sr(7.0, 0)) == 6.0
    # the fraction of words that round up equals p on a fine sweep of u
    for v in (0.1, 0.6, 1.3, 2.2, 3.9, 5.5):
        lo = max(g for g in grid if g <= v)
        hi = min(g for g in grid if g > v)
        p = (np.float32(v) - lo) / (hi - lo)
        words = np.arange(0, 1 << 32, 1 << 16, dtype=np.uint64)
        ups = sum(abs(oracle.e2m1_value(oracle.e2m1_sr(v, int(w)))) == hi for w in words)
        assert abs(ups / len(words) - p) <= 1.0 / len(words) + 1e-12


# --------------------------------------------------------------------- E4M3
def _torch_e4m3_bits(v):
    t = torch.tensor(np.asarray(v, np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


def test_e4m3_decode_matches_torch_float8():
    b = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(b).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    ours = np.array([oracle.e4m3_value(int(x)) for x in b], np.float32)
    nan = np.isnan(ref)
    assert (np.isnan(ours) == nan).all() and nan.sum() == 2
    assert (ours[~nan] == ref[~nan]).all()
    assert oracle.e4m3_value(0x7E) == 448.0 and oracle.e4m3_value(0x01) == 2.0 ** -9
    assert oracle.e4m3_value(0x08) == 2.0 ** -6


def test_e4m3_rne_matches_torch_float8_in_range():
    rng = np.random.default_rng(1)
    pos = np.array([oracle.e4m3_value(b) for b in range(127)], np.float64)
    mids = (pos[:-1] + pos[1:]) / 2
    vals = np.concatenate([
        rng.uniform(-448, 448, 3000), np.exp(rng.uniform(-14, 6, 3000)) * rng.choice([-1, 1], 3000),
        mids, -mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9)]).astype(np.float32)
    vals = vals[np.abs(vals) <= 448]
    ours = np.array([oracle.e4m3_rne(float(v)) for v in vals], np.uint8)
    ref = _torch_e4m3_bits(vals)
    # torch maps -0-rounding values to 0x80 like the oracle's sign copy
    assert (ours == ref).all()
    assert oracle.e4m3_rne(1e6) == 0x7E and oracle.e4m3_rne(-500.0) == 0xFE   # satfinite


def test_e4m3_sr_rule():
    for b in range(127):
        v = oracle.e4m3_value(b)
        assert oracle.e4m3_sr(v, 0xFFFFFFFF) == b
    v = (oracle.e4m3_value(0x40) + oracle.e4m3_value(0x41)) / 2      # halfway
    assert oracle.e4m3_sr(v, 1 << 31) == 0x40 and oracle.e4m3_sr(v, (1 << 31) - 256) == 0x41
    assert oracle.e4m3_sr(1000.0, 0) == 0x7E


# --------------------------------------------------------------------- scales
def test_e8m0_values():
    assert oracle.e8m0_value(127) == 1.0 and oracle.e8m0_value(0) == 2.0 ** -127
    assert oracle.e8m0_value(254) == 2.0 ** 127 and math.isnan(oracle.e8m0_value(255))


def _mantissa_rule(amax, top_m, top_e):
    """least k with top * 2^k >= amax from the binary exponent of amax
    (amax = m * 2^e, m in [1, 2); top = top_m * 2^top_e, top_m in [1, 2)):
    k = e - top_e if m <= top_m, else e - top_e + 1."""
    m, e = math.frexp(amax)
    m, e = 2 * m, e - 1
    return e - top_e if m <= top_m else e - top_e + 1


@pytest.mark.parametrize("top,top_m,top_e", [(6.0, 1.5, 2), (448.0, 1.75, 8)])
def test_scale_exponent_truncation_free(top, top_m, top_e):
    rng = np.random.default_rng(2)
    vals = list(np.exp(rng.uniform(-80, 80, 3000)).astype(np.float32))
    for k in range(-20, 20):                         # adversarial: on and next to top * 2^k
        base = np.float32(top * 2.0 ** k)
        vals += [base, np.nextafter(base, np.float32(0)), np.nextafter(base, np.float32(1e30)),
                 np.float32(2.0 ** k), np.float32(1.5 * 2.0 ** k), np.float32(1.75 * 2.0 ** k)]
    vals += [np.float32(1e-40), np.float32(3.0e38)]   # subnormal, near the top of binary32
    for a in vals:
        a = float(a)
        k = oracle.scale_exp(a, top)
        assert top * 2.0 ** k >= a                    # never clips
        if k > -127:
            assert top * 2.0 ** (k - 1) < a           # and is the least such k
        want = max(-127, _mantissa_rule(a, top_m, top_e))
        assert k == want


# --------------------------------------------------------------------- Philox
def test_philox_known_answers():
    for row in _golden_lines("philox_kat.txt"):
        v = [int(t, 16) for t in row]
        assert oracle.philox4x32_10(v[0:4], v[4:6]) == v[6:10]


def test_sr_word_uses_counter_e_div_4_and_word_e_mod_4():
    seed = 0x0123456789ABCDEF
    for e in (0, 1, 2, 3, 4, 7, (1 << 34) + 5, (1 << 40) + 2):
        c = e >> 2
        want = oracle.philox4x32_10([c & 0xFFFFFFFF, c >> 32, 0, 0], [seed & 0xFFFFFFFF, seed >> 32])[e & 3]
        assert oracle.sr_word(seed, e) == want


# --------------------------------------------------------------------- FWHT
C128 = np.float32(np.uint32(0x3DB504F3).view(np.float32))


def test_fwht_constant_is_binary32_of_2_pow_minus_3_5():
    assert C128 == np.float32(2.0 ** -3.5)           # numpy's rounding of the binary64 value
    e0 = np.zeros(128, np.float32)
    e0[0] = 1
    assert oracle.fwht128(e0)[0] == C128


def test_fwht_unit_vectors_give_hadamard_columns_exactly():
    for j in range(128):
        e = np.zeros(128, np.float32)
        e[j] = 1.0
        y = oracle.fwht128(e)
        signs = np.array([(-1) ** bin(i & j).count("1") for i in range(128)], np.float32)
        assert (y == signs * C128).all()


def test_fwht_matches_scipy_hadamard_and_is_orthogonal():
    from scipy.linalg import hadamard
    H = hadamard(128).astype(np.float64) / math.sqrt(128)
    rng = np.random.default_rng(3)
    for _ in range(20):
        x = rng.standard_normal(128).astype(np.float32)
        y = oracle.fwht128(x).astype(np.float64)
        ref = H @ x.astype(np.float64)
        assert np.abs(y - ref).max() <= 1e-5 * np.abs(x).sum()
        # norm preservation ([LB] §7: the length is kept)
        assert abs(np.linalg.norm(y) - np.linalg.norm(x)) <= 1e-6 * np.linalg.norm(x)
        # applying twice returns x (H is symmetric and orthogonal)
        z = oracle.fwht128(y.astype(np.float32)).astype(np.float64)
        assert np.abs(z - x).max() <= 1e-6 * np.abs(x).max() + 1e-7
    assert np.allclose(H @ H.T, np.eye(128), atol=1e-12)


def test_fwht_spreads_an_outlier_to_one_over_sqrt_n():
    lines = {r[0]: r[1:] for r in _golden_lines("lowbit_blog_tables.txt")}
    n, shrink = (int(v) for v in lines["rotation_shrink"])
    assert shrink == math.isqrt(n)                   # the page's 256 -> 1/16 is 1/sqrt(n)
    x = np.zeros(128, np.float32)
    x[37] = 50.0
    y = oracle.fwht128(x)
    assert np.allclose(np.abs(y), 50.0 / math.sqrt(128), rtol=1e-6)


# --------------------------------------------------------------------- bf16
def test_f64_to_bf16_rounding():
    # exactly representable values, ties to even, subnormals
    cases = {1.0: 0x3F80, -2.0: 0xC000, 1.0 + 2 ** -8: 0x3F80, 1.0 + 3 * 2 ** -8: 0x3F82,
             1.0 + 2 ** -8 + 2 ** -40: 0x3F81, 2.0 ** -133: 0x0001, 2.0 ** -134: 0x0000,
             3 * 2.0 ** -134: 0x0002, 0.0: 0x0000}
    for v, want in cases.items():
        assert oracle.f64_to_bf16(v) == want, v
    # agrees with torch's float32 -> bfloat16 rounding where the value fits binary32
    rng = np.random.default_rng(4)
    v = (rng.standard_normal(2000) * np.exp(rng.uniform(-30, 30, 2000))).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.uint16).numpy()
    ours = np.array([oracle.f64_to_bf16(float(t)) for t in v], np.uint16)
    assert (ours == ref).all()


def test_dequantize_nan_scale_bytes():
    """E8M0 0xFF and E4M3 0x7F / 0xFF are the OCP NaN encodings: a group under
    such a byte dequantizes to NaN, every other byte to finite values."""
    codes16 = np.array([0x10, 0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE], np.uint8)   # codes 0..15
    for fmt, K, nan_bytes in ((oracle.NVFP4, 16, {0x7F, 0xFF}), (oracle.MXFP4, 32, {0xFF})):
        codes = np.tile(codes16, (256, K // 16))
        scales = np.arange(256, dtype=np.uint8).reshape(256, 1)
        ts = np.float32(0.5) if fmt == oracle.NVFP4 else None
        out = oracle.dequantize(codes, scales, ts, 256, K, fmt)
        for b in range(256):
            assert np.isnan(out[b]).all() == (b in nan_bytes), b
            if b not in nan_bytes:
                assert np.isfinite(out[b]).all()
