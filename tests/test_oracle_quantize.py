"""Pins of the oracle's quantize paths against the pages and the mathematics.

Brute force on small blocks, the pages' worked outlier example, the printed
tables' direction, effective bits, SR unbiasedness, transposition invariance
and four-over-six optimality.  No expected value comes from the CUDA path.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


def _tables():
    out = {}
    with open(os.path.join(GOLDEN, "lowbit_blog_tables.txt")) as f:
        for l in f:
            if l.strip() and not l.startswith("#"):
                t = l.split()
                out.setdefault(t[0], {})[t[1]] = [float(v) for v in t[2:]]
    return out


def _nib(codes, M, K):
    c = np.asarray(codes, np.uint8).reshape(M, K // 2)
    out = np.empty((M, K), np.uint8)
    out[:, 0::2] = c & 0x0F
    out[:, 1::2] = c >> 4
    return out


def _val(nib):
    mag = GRID[nib & 7]
    return np.where(nib & 8, -mag, mag)


def _f32(x):
    return synth.bf16_bits_to_f32(x) if x.dtype == np.uint16 else x


def _torch_e4m3(v):
    return int(torch.tensor([np.float32(v)]).to(torch.float8_e4m3fn).view(torch.uint8)[0])


# ------------------------------------------------------------ brute force 1x32
@pytest.mark.parametrize("seed", range(6))
def test_mxfp4_group_bruteforce(seed):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((1, 32)) * np.exp(rng.uniform(-20, 20))).astype(np.float32)
    q = oracle.quantize(x, oracle.MXFP4)
    amax = float(np.abs(x).max())
    # the scale byte: least k over [-127,127] (searched exhaustively) with 6*2^k >= amax
    k = min(k for k in range(-127, 128) if 6.0 * 2.0 ** k >= amax)
    assert q["scales"][0, 0] == k + 127
    v = x.astype(np.float64)[0] / 2.0 ** k
    assert np.abs(v).max() <= 6.0                      # truncation-free: nothing clips
    assert np.abs(v).max() > 3.0                       # and the scale is not wasteful
    got = _val(_nib(q["codes"], 1, 32))[0]
    for t in range(32):                                # each code is a nearest grid value
        d = np.abs(GRID - abs(v[t]))
        assert abs(abs(got[t]) - abs(v[t])) == d.min()


@pytest.mark.parametrize("seed", range(6))
def test_nvfp4_scales_bruteforce(seed):
    rng = np.random.default_rng(100 + seed)
    x = (rng.standard_normal((2, 64)) * np.exp(rng.uniform(-10, 10, (2, 64)))).astype(np.float32)
    q = oracle.quantize(x, oracle.NVFP4)
    amax_t = np.float32(np.abs(x).max())
    s_t = np.float32(amax_t / np.float32(2688.0))
    assert q["tscale"][0] == s_t                         # s_t = amax_t / (6 * 448) in binary32
    nib = _val(_nib(q["codes"], 2, 64))
    for i in range(2):
        for b in range(4):
            blk = x[i, 16 * b:16 * b + 16]
            amax = np.float32(np.abs(blk).max())
            r = np.float32(np.float32(amax / np.float32(6.0)) / s_t)
            enc = _torch_e4m3(r)                           # library E4M3 rounding of the block scale
            assert q["scales"][i, b] == enc
            S = np.float32(np.float32(oracle.e4m3_value(enc)) * s_t)
            v = (blk / S).astype(np.float64)
            for t in range(16):
                d = np.abs(GRID - min(abs(v[t]), 6.0))
                assert abs(abs(nib[i, 16 * b + t]) - min(abs(v[t]), 6.0)) == d.min()


def test_all_zero_groups_and_tensor():
    x = np.zeros((2, 64), np.float32)
    q = oracle.quantize(x, oracle.MXFP4)
    assert (q["scales"] == 0).all() and (q["codes"] == 0).all()
    q = oracle.quantize(x, oracle.NVFP4)
    assert q["tscale"][0] == 0 and (q["scales"] == 0).all() and (q["codes"] == 0).all()
    x[0, :32] = -0.0                                      # negative zeros in an all-zero group: +0 codes
    assert (oracle.quantize(x, oracle.MXFP4)["codes"] == 0).all()


def test_nvfp4_block_whose_scale_underflows_gets_plus_zero_codes():
    """Reading c6: a block whose E4M3 scale rounds to 0 under the tensor scale
    (values far below amax_t / 2688 * 2^-9) has S = 0 and +0 codes, also for
    its negative values, with RNE and SR alike."""
    x = np.zeros((1, 32), np.float32)
    x[0, :16] = np.array([1e-6, -2e-6, 3e-7, -1e-6] * 4, np.float32)
    x[0, 16], x[0, 17:] = 1000.0, -3.0
    for rounding in (oracle.RNE, oracle.SR):
        q = oracle.quantize(synth.f32_to_bf16_bits(x), oracle.NVFP4, rounding, seed=5)
        assert q["scales"][0, 0] == 0 and q["scales"][0, 1] == 0x7E      # 1000 / 6 / s_t = 448
        assert not q["codes"][0, :8].any()


def test_effective_bits_match_the_page():
    tb = _tables()["effective_bits"]
    M, K = 64, 256
    x = synth.gaussian_bf16(M, K, 5)
    q = oracle.quantize(x, oracle.MXFP4)
    bits = 8 * (q["codes"].nbytes + q["scales"].nbytes) / (M * K)
    assert bits == tb["mxfp4"][0] == 4 + 8 / 32
    # a 16-bit scale per 32 elements would cost 4.5 bits; NVFP4 (8-bit per 16) matches that
    q = oracle.quantize(x, oracle.NVFP4)
    bits = 8 * (q["codes"].nbytes + q["scales"].nbytes) / (M * K)
    assert bits == tb["fp16_scale_group32"][0] == 4 + 16 / 32 == 4 + 8 / 16


# ------------------------------------------------------------ stochastic rounding
def test_sr_is_unbiased_over_10k_seeds():
    rng = np.random.default_rng(7)
    x = rng.uniform(-5.9, 5.9, (1, 32)).astype(np.float32)
    x[0, 0] = 6.0                                         # amax 6 -> k = 0, v = x exactly
    n = 10_000
    acc = np.zeros(32)
    for s in range(n):
        acc += _val(_nib(oracle.quantize(x, oracle.MXFP4, oracle.SR, seed=s)["codes"], 1, 32))[0]
    mean = acc / n
    for t in range(32):
        a = abs(float(x[0, t]))
        lo = GRID[GRID <= a].max()
        hi = GRID[GRID > a].min() if a < 6 else 6.0
        sigma = (hi - lo) / (2 * math.sqrt(n))
        assert abs(mean[t] - x[0, t]) <= 4 * sigma + 1e-12


def test_sr_words_are_keyed_on_seed_and_index():
    x = synth.gaussian_bf16(8, 64, 9)
    a = oracle.quantize(x, oracle.MXFP4, oracle.SR, seed=11)["codes"]
    assert (a == oracle.quantize(x, oracle.MXFP4, oracle.SR, seed=11)["codes"]).all()
    assert (a != oracle.quantize(x, oracle.MXFP4, oracle.SR, seed=12)["codes"]).any()
    # the same values at another position draw other words: row 0 copied into row 1
    y = x.copy()
    y[1] = y[0]
    c = _nib(oracle.quantize(y, oracle.MXFP4, oracle.SR, seed=11)["codes"], 8, 64)
    assert (c[0] != c[1]).any()


# ------------------------------------------------------------ rotation
def test_rotate_applies_fwht_per_128_block_along_k():
    # rows that are scaled unit vectors rotate exactly to +-a*c, so the rotated
    # quantization must equal the plain quantization of the known rotated rows
    M, K = 4, 256
    x = np.zeros((M, K), np.float32)
    pos = [(0, 5, 3.0), (1, 130, -7.5), (2, 127, 0.25), (3, 200, 1e-3)]
    for i, j, a in pos:
        x[i, j] = a
    c = np.float32(np.uint32(0x3DB504F3).view(np.float32))
    xr = np.zeros_like(x)
    for i, j, a in pos:
        b0 = (j // 128) * 128
        for t in range(128):
            xr[i, b0 + t] = np.float32(a) * c * (-1) ** bin(t & (j - b0)).count("1")
    for fmt in (oracle.MXFP4, oracle.NVFP4):
        qa = oracle.quantize(x, fmt, rotate=True)
        qb = oracle.quantize(xr, fmt)
        assert (qa["codes"] == qb["codes"]).all() and (qa["scales"] == qb["scales"]).all()


def _kurtosis(v):
    v = np.asarray(v, np.float64).ravel()
    v = v - v.mean()
    return float((v ** 4).mean() / (v ** 2).mean() ** 2)


def test_rotation_flattens_outliers_direction_of_the_page():
    """[LB] §7: an injected x50 weight gives a huge kurtosis that rotation removes;
    rotation rescues per-tensor FP4 and does little for per-group scales."""
    tb = _tables()
    W = synth.cfg1_W()[:, :768].copy()                    # K multiple of 128
    W[17, 300] = 50 * np.abs(W).max()
    k0 = _kurtosis(W)
    Wr = np.stack([np.concatenate([oracle.fwht128(r[b:b + 128]) for b in range(0, 768, 128)]) for r in W])
    k1 = _kurtosis(Wr)
    page_k = tb["kurtosis"]["13717"]                     # row: 13717 54 3.4
    assert k0 > 1000 and k1 < k0 / 10                     # page: 13717 -> 54 (input side)
    assert page_k[0] < 13717 / 10

    def mse(q_codes, scales, X, gran):
        deq = _val(_nib(q_codes, X.shape[0], X.shape[1]))
        if gran == oracle.GRAN_TENSOR:
            deq = deq * scales[0]
        else:
            deq = deq * np.repeat(scales.reshape(X.shape[0], -1), 32, axis=1)
        return float(((deq - X) ** 2).mean())

    e_plain = mse((q := oracle.quantize_fp32scale(W, oracle.GRAN_TENSOR))["codes"], q["scales"], W,
                  oracle.GRAN_TENSOR)
    e_rot = mse((q := oracle.quantize_fp32scale(Wr, oracle.GRAN_TENSOR))["codes"], q["scales"], Wr,
                oracle.GRAN_TENSOR)
    assert e_rot < e_plain / 2                            # page: 0.859 -> 0.197 per tensor
    g_plain = mse((q := oracle.quantize_fp32scale(W, oracle.GRAN_GROUP32))["codes"], q["scales"], W,
                  oracle.GRAN_GROUP32)
    g_rot = mse((q := oracle.quantize_fp32scale(Wr, oracle.GRAN_GROUP32))["codes"], q["scales"], Wr,
                oracle.GRAN_GROUP32)
    assert g_rot > g_plain / 3                            # page: 0.043 -> 0.089, no gain per group


# ------------------------------------------------------------ outlier example
def _mse_excluding(deq, W, mask):
    return float(((deq - W)[mask] ** 2).mean())


def test_worked_outlier_example_per_tensor_row_group():
    """[LB] §1 table and text on a synthetic fc1-sized weight (256 x 784, N(0,0.04^2))."""
    tb = _tables()["outlier_mse"]
    W = synth.cfg1_W()
    Wo = W.copy()
    Wo[17, 300] = 50 * np.abs(W).max()
    normal = np.ones_like(W, bool)
    normal[17, 300] = False

    def run(X, gran, g):
        q = oracle.quantize_fp32scale(X, gran)
        nib = _nib(q["codes"], *X.shape)
        if gran == oracle.GRAN_TENSOR:
            S = np.full(X.shape, q["scales"][0], np.float64)
        elif gran == oracle.GRAN_ROW:
            S = np.repeat(q["scales"].astype(np.float64)[:, None], X.shape[1], axis=1)
        else:
            S = np.repeat(q["scales"].astype(np.float64).reshape(X.shape[0], -1), g, axis=1)
        return nib, _val(nib) * S

    # per-tensor: the smallest nonzero level 0.5*S exceeds every normal weight, almost all snap to 0
    nib0, d0 = run(W, oracle.GRAN_TENSOR, 0)
    nib1, d1 = run(Wo, oracle.GRAN_TENSOR, 0)
    S = np.abs(Wo).max() / 6
    assert 0.5 * S > np.abs(W).max()
    assert ((nib1[normal] & 7) == 0).mean() >= 0.999
    r_tensor = _mse_excluding(d1, W, normal) / _mse_excluding(d0, W, normal)
    assert r_tensor > 5 and tb["per-tensor"][1] / tb["per-tensor"][0] > 5
    # per-row: every row but the outlier's is bit-identical
    nib0, d0 = run(W, oracle.GRAN_ROW, 0)
    nib1, d1 = run(Wo, oracle.GRAN_ROW, 0)
    other = np.arange(256) != 17
    assert (nib0[other] == nib1[other]).all()
    # per-group (16 and 32 elements): every group but the outlier's is bit-identical; MSE ratio ~ 1
    for gran, g in ((oracle.GRAN_GROUP16, 16), (oracle.GRAN_GROUP32, 32)):
        Wg, Wog = W[:, :768], Wo[:, :768]
        nib0, d0 = run(Wg, gran, g)
        nib1, d1 = run(Wog, gran, g)
        diff = np.argwhere(nib0 != nib1)
        assert all(i == 17 and j // g == 300 // g for i, j in diff)
        m = normal[:, :768]
        r = _mse_excluding(d1, Wg, m) / _mse_excluding(d0, Wg, m)
        assert 0.9 < r < 1.1 and abs(tb["per-group32"][1] / tb["per-group32"][0] - 1) < 0.1
    # MXFP4 groups (K zero-padded 784 -> 800; pads change no amax)
    Wp, Wop = np.zeros((256, 800), np.float32), np.zeros((256, 800), np.float32)
    Wp[:, :784], Wop[:, :784] = W, Wo
    a = _nib(oracle.quantize(Wp, oracle.MXFP4)["codes"], 256, 800)
    b = _nib(oracle.quantize(Wop, oracle.MXFP4)["codes"], 256, 800)
    diff = np.argwhere(a != b)
    assert len(diff) and all(i == 17 and j // 32 == 300 // 32 for i, j in diff)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_fp32_scale_is_amax_over_six_and_never_clips(dtype):
    """[LB] "FP4" section: S = |W|max / 6, so the largest magnitude lands on
    the top grid value 6 and nothing is clipped.  Pinned independently of the
    oracle's arithmetic: numpy's maximum of |x| over the tensor, each row and
    each group, divided by 6 in binary32, must equal the oracle's scale for
    every granularity (a divisor of 4 or 8 fails here), the element holding
    the maximum must decode to +-6, and every code must be the grid value
    nearest to fl(x / S) (brute force over the 8 magnitudes)."""
    rng = np.random.default_rng(77)
    M, K = 24, 96
    x = (rng.standard_normal((M, K)) * np.exp(rng.uniform(-3, 3, (M, 1)))).astype(np.float32)
    x[3, 5] = 0.0
    x[7] = 0.0                                            # an all-zero row: S = 0, +0 codes
    if dtype == "bf16":
        x = synth.f32_to_bf16_bits(x)
    xf = _f32(x).astype(np.float32)
    ax = np.abs(xf)
    grans = {oracle.GRAN_TENSOR: ax.max().reshape(1), oracle.GRAN_ROW: ax.max(axis=1),
             oracle.GRAN_GROUP16: ax.reshape(M, K // 16, 16).max(axis=2).ravel(),
             oracle.GRAN_GROUP32: ax.reshape(M, K // 32, 32).max(axis=2).ravel()}
    width = {oracle.GRAN_TENSOR: M * K, oracle.GRAN_ROW: K, oracle.GRAN_GROUP16: 16, oracle.GRAN_GROUP32: 32}
    for gran, amax in grans.items():
        q = oracle.quantize_fp32scale(x, gran)
        want = (amax.astype(np.float32) / np.float32(6.0)).astype(np.float32)
        assert np.array_equal(q["scales"].view(np.uint32), want.view(np.uint32)), gran
        S = np.repeat(want.astype(np.float64), width[gran]).reshape(M, K)
        nib = _nib(q["codes"], M, K)
        S32 = S.astype(np.float32)                            # v = fl(x / S) in binary32 (reading c4)
        v = np.divide(xf, S32, out=np.zeros_like(xf), where=S32 > 0).astype(np.float64)
        dist = np.abs(np.abs(v)[..., None] - GRID)
        ok = dist[np.arange(M)[:, None], np.arange(K)[None, :], nib & 7] <= dist.min(axis=-1) + 1e-12
        assert ok.all(), gran
        top = (ax == np.repeat(amax, width[gran]).reshape(M, K)) & (ax > 0)
        assert ((nib[top] & 7) == 7).all(), gran          # the maximum decodes to +-6
        assert not (nib[S == 0] & 7).any()


def test_power_of_two_scale_costs_a_little_mse():
    """[LB] §3 table: a 2^k group scale costs 1.0-1.4x the MSE of an FP group scale."""
    tb = _tables()["scale_cost"]
    assert all(1.0 <= b / a < 1.5 for a, b in tb.values())
    W = np.zeros((256, 800), np.float32)
    W[:, :784] = synth.cfg1_W()
    qf = oracle.quantize_fp32scale(W, oracle.GRAN_GROUP32)
    deq_f = _val(_nib(qf["codes"], 256, 800)) * np.repeat(qf["scales"].astype(np.float64).reshape(256, -1), 32, 1)
    qm = oracle.quantize(W, oracle.MXFP4)
    deq_m = oracle.dequantize(qm["codes"], qm["scales"], None, 256, 800, oracle.MXFP4)
    r = float(((deq_m - W) ** 2).mean() / ((deq_f - W) ** 2).mean())
    assert 1.0 <= r < 2.0


# ------------------------------------------------------------ 2D / transposed
def _roundtrip_codesT(q, M, K):
    return _nib(q["codesT"], K, M)


@pytest.mark.parametrize("rounding", [oracle.RNE, oracle.SR])
def test_2d_blocks_are_transposition_invariant(rounding):
    M, K = 48, 64
    x = synth.cfg4_G(M, K, seed=21)
    q = oracle.quantize(x, oracle.NVFP4, rounding, block2d=True, seed=5, transposed=True)
    c = _nib(q["codes"], M, K)
    cT = _roundtrip_codesT(q, M, K)
    assert (cT == c.T).all()
    S, ST = q["scales"], q["scalesT"]
    for i in range(M):
        for j in range(K):
            assert S[i, j // 16] == ST[j, i // 16]
    # one scale per 16x16 tile, from the tile's amax
    xf = _f32(x)
    s_t = q["tscale"][0]
    for bi in range(0, M, 16):
        for bj in range(0, K, 16):
            amax = np.float32(np.abs(xf[bi:bi + 16, bj:bj + 16]).max())
            enc = _torch_e4m3(np.float32(np.float32(amax / np.float32(6)) / s_t))
            assert (S[bi:bi + 16, bj // 16] == enc).all()


def test_1d_column_output_is_quantization_of_the_transpose():
    M, K = 64, 96
    x = synth.gaussian_bf16(M, K, 23)
    for fmt in (oracle.MXFP4, oracle.NVFP4):
        q = oracle.quantize(x, fmt, transposed=True)
        qt = oracle.quantize(np.ascontiguousarray(x.T), fmt)
        assert (q["codesT"] == qt["codes"]).all() and (q["scalesT"] == qt["scales"]).all()
        # and it differs from the 2D-invariant one: 1D scales of X and X^T disagree
        assert (_nib(q["codesT"], K, M) != _nib(q["codes"], M, K).T).any()


# ------------------------------------------------------------ four over six
def test_four6_picks_the_lower_error_bruteforce():
    rng = np.random.default_rng(31)
    picked4 = 0
    for _ in range(400):
        x = (rng.standard_normal(16) * rng.uniform(0.1, 3)).astype(np.float32)
        s_t = np.float32(np.abs(x).max() * rng.uniform(1, 4) / 2688)
        pick, enc, codes = oracle.four6_pick(x, float(s_t))
        sse = {}
        for d in (6.0, 4.0):
            amax = np.float32(np.abs(x).max())
            e = oracle.e4m3_rne(float(np.float32(np.float32(amax / np.float32(d)) / s_t)))
            S = np.float32(np.float32(oracle.e4m3_value(e)) * s_t)
            c = np.array([oracle.e2m1_rne(float(np.float32(v / S))) for v in x]) if S else np.zeros(16, int)
            sse[d] = (e, c, float((((_val(c) * np.float64(S)) - x) ** 2).sum()))
        want = 4.0 if pick else 6.0
        other = 6.0 if pick else 4.0
        assert enc == sse[want][0] and (codes == sse[want][1]).all()
        assert sse[want][2] <= sse[other][2] * (1 + 1e-5) + 1e-30
        picked4 += pick
    assert 0 < picked4 < 400


def test_four6_prefers_amax_over_4_when_values_sit_in_the_4_to_6_gap():
    # [46]: FP4's largest error sits at the block's largest values; with amax/6 the
    # values 5 fall in the 4..6 gap, with amax/4 they land near 3 and 4.
    x = np.array([6, 5, 5, 5, 5, 5, 5, 5, -5, -5, 5, 5, 5, 5, 5, 5], np.float32)
    pick, enc, codes = oracle.four6_pick(x, 2.0 ** -8)
    assert pick == 1 and oracle.e4m3_value(enc) * 2.0 ** -8 == 1.5
    x = np.array([6, 1, 0.5, 0, 2, 3, 1, 0, 0, 0, 1, 1, 0.5, 2, 3, 4], np.float32)   # on the amax/6 grid
    pick, enc, _ = oracle.four6_pick(x, 2.0 ** -8)
    assert pick == 0


def test_four6_tie_keeps_amax_over_6():
    """Equal errors keep the amax/6 candidate (reading c7): when both
    candidate quotients saturate at 448 they encode the same scale, the
    codes and errors are identical, and the block must keep amax/6."""
    rng = np.random.default_rng(37)
    for _ in range(50):
        x = (rng.standard_normal(16) * rng.uniform(0.1, 3)).astype(np.float32)
        s_t = np.float32(np.abs(x).max() / np.float32(2 * 2688))        # both quotients >= 448
        pick, enc, _ = oracle.four6_pick(x, float(s_t))
        assert pick == 0 and enc == 0x7E
    pick, enc, codes = oracle.four6_pick(np.zeros(16, np.float32), 1.0)  # amax 0: both scales 0
    assert pick == 0 and enc == 0 and not codes.any()


def test_four6_in_quantize_matches_pick():
    M, K = 8, 64
    x = synth.cfg3_X(M, K, seed=33)
    q = oracle.quantize(x, oracle.NVFP4, four6=True)
    s_t = float(q["tscale"][0])
    xf = _f32(x)
    c = _nib(q["codes"], M, K)
    for i in range(M):
        for b in range(K // 16):
            _, enc, codes = oracle.four6_pick(xf[i, 16 * b:16 * b + 16], s_t)
            assert q["scales"][i, b] == enc and (c[i, 16 * b:16 * b + 16] == codes).all()


# ------------------------------------------------------------ MXFP8
@pytest.mark.parametrize("rounding", [oracle.RNE, oracle.SR])
def test_mxfp8_bruteforce(rounding):
    x = synth.cfg4_G(32, 64, seed=41)
    q = oracle.quantize_mxfp8(x, rounding, seed=3, transposed=True)
    xf = _f32(x).astype(np.float64)
    for i in range(32):
        for g in range(2):
            blk = xf[i, 32 * g:32 * g + 32]
            amax = np.abs(blk).max()
            k = int(q["scales"][i, g]) - 127
            assert 448 * 2.0 ** k >= amax and 448 * 2.0 ** (k - 1) < amax
            v = (blk / 2.0 ** k).astype(np.float32)
            got = q["codes"][i, 32 * g:32 * g + 32]
            if rounding == oracle.RNE:
                ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
                assert (got == ref).all()
            else:                                  # a neighbour of v on the E4M3 grid
                dec = np.array([oracle.e4m3_value(int(b)) for b in got])
                ulp = np.maximum(2.0 ** (np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** -6))) - 3), 2.0 ** -9)
                assert (np.abs(dec - v) < ulp).all()
    if rounding == oracle.RNE:
        qt = oracle.quantize_mxfp8(np.ascontiguousarray(x.T), rounding)
        assert (q["codesT"] == qt["codes"]).all() and (q["scalesT"] == qt["scales"]).all()


# ------------------------------------------------------------ argument checks
def test_argument_validation():
    x = np.zeros((32, 128), np.float32)
    st = oracle.quantize_status
    assert st(x, oracle.MXFP4) == oracle.OK
    assert st(x, oracle.MXFP4, four6=True) == oracle.OK              # MXFP4 four-over-six (32-groups)
    assert st(x, oracle.NVFP4, four6=True, rounding=oracle.SR) == oracle.ERR_UNSUPPORTED
    assert st(x, oracle.MXFP4, block2d=True) == oracle.OK            # 32 x 32 MXFP4 tiles
    assert st(np.zeros((48, 128), np.float32), oracle.MXFP4, block2d=True) == oracle.ERR_SHAPE
    assert st(x, oracle.MXFP4, block2d=True, four6=True) == oracle.ERR_UNSUPPORTED
    assert st(x, oracle.NVFP4, block2d=True, rotate=True) == oracle.ERR_UNSUPPORTED
    assert st(x, oracle.NVFP4, rotate=True, transposed=True) == oracle.ERR_UNSUPPORTED
    assert st(np.zeros((32, 48), np.float32), oracle.MXFP4) == oracle.ERR_SHAPE
    assert st(np.zeros((32, 96), np.float32), oracle.NVFP4, rotate=True) == oracle.ERR_SHAPE
    assert st(np.zeros((24, 64), np.float32), oracle.NVFP4, block2d=True) == oracle.ERR_SHAPE


def test_argument_validation_of_the_extended_call():
    x = np.zeros((32, 128), np.float32)
    st = oracle.quantize_ex_status
    assert st(x, oracle.MXFP4, rule=oracle.RULE_OCP_FLOOR) == oracle.OK
    assert st(x, oracle.NVFP4, rule=oracle.RULE_E4M3_UP) == oracle.OK
    assert st(x, oracle.NVFP4, rule=oracle.RULE_OCP_FLOOR) == oracle.ERR_UNSUPPORTED   # E8M0 rule only
    assert st(x, oracle.MXFP4, rule=oracle.RULE_E4M3_UP) == oracle.ERR_UNSUPPORTED     # E4M3 rule only
    assert st(x, oracle.MXFP4, rule=5) == oracle.ERR_ARG
    assert st(x, oracle.MXFP4, amax_in=1.0) == oracle.ERR_UNSUPPORTED                  # tensor amax: NVFP4
    assert st(x, oracle.NVFP4, amax_in=1.0) == oracle.OK
    assert st(x, oracle.NVFP4, row0=3) == oracle.OK
    assert st(x, oracle.NVFP4, row0=3, block2d=True) == oracle.ERR_UNSUPPORTED
    assert st(x, oracle.NVFP4, row0=-1) == oracle.ERR_ARG
