"""Pins of the oracle's scale-rule variants, MXFP4 four-over-six, MXFP4 2D
tiles, the caller-supplied tensor amax, row slices and the MXFP8 GEMM
reference.  Each is checked against brute force, a closed form or an
equivalence the pages fix; no expected value comes from the CUDA path.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synth

GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


def _nib(codes, M, K):
    c = np.asarray(codes, np.uint8).reshape(M, K // 2)
    out = np.empty((M, K), np.uint8)
    out[:, 0::2] = c & 0x0F
    out[:, 1::2] = c >> 4
    return out


def _val(nib):
    mag = GRID[nib & 7]
    return np.where(nib & 8, -mag, mag)


def _nearest_ok(v, nib):
    """nib is a nearest saturating E2M1 code of v (ties may go either way)."""
    a = np.minimum(np.abs(v), 6.0)
    d = np.abs(a[..., None] - GRID)
    return d[..., nib & 7] if np.ndim(v) == 0 else np.take_along_axis(d, (nib & 7)[..., None].astype(np.int64), -1)[..., 0] <= d.min(-1) + 1e-12


def _e4m3_table():
    b = torch.arange(127, dtype=torch.uint8)                 # 0x00 .. 0x7E: every finite non-negative byte
    return b.view(torch.float8_e4m3fn).to(torch.float64).numpy()


# ------------------------------------------------------------ OCP floor rule (E8M0)
@pytest.mark.parametrize("seed", range(6))
def test_ocp_floor_exponent_and_codes_bruteforce(seed):
    """k = the largest integer with 2^(k+2) <= amax (searched exhaustively
    over [-127, 127]); every code is the nearest E2M1 value of fl(x / 2^k),
    saturating at 6, so values above 6 * 2^k are clipped."""
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((3, 32)) * np.exp(rng.uniform(-30, 30, (3, 1)))).astype(np.float32)
    q = oracle.quantize_ex(x, oracle.MXFP4, rule=oracle.RULE_OCP_FLOOR)
    nib = _nib(q["codes"], 3, 32)
    for i in range(3):
        amax = float(np.abs(x[i]).max())
        k = max(k for k in range(-127, 128) if 2.0 ** (k + 2) <= amax)
        assert int(q["scales"][i, 0]) == k + 127
        assert oracle.scale_exp_floor(np.float32(amax), 2) == k
        v = (x[i] / np.float32(2.0 ** k)).astype(np.float64)
        assert _nearest_ok(v, nib[i]).all()


def test_ocp_floor_clips_where_truncation_free_does_not():
    """amax = 7 * 2^j: the floor rule takes k = j (7 > 6 is clipped to 6);
    the truncation-free rule takes j + 1 (6 * 2^(j+1) >= 7 * 2^j)."""
    for j in (-20, 0, 9):
        x = np.zeros((1, 32), np.float32)
        x[0, 0] = 7 * 2.0 ** j
        x[0, 1:] = np.linspace(-2, 2, 31, dtype=np.float32) * np.float32(2.0 ** j)
        f = oracle.quantize_ex(x, oracle.MXFP4, rule=oracle.RULE_OCP_FLOOR)
        t = oracle.quantize_ex(x, oracle.MXFP4)
        assert int(f["scales"][0, 0]) == j + 127 and int(t["scales"][0, 0]) == j + 128
        assert _nib(f["codes"], 1, 32)[0, 0] == 7                # decodes to 6 * 2^j < 7 * 2^j
        assert _val(_nib(t["codes"], 1, 32))[0, 0] * 2.0 ** (j + 1) == 8 * 2.0 ** j   # 7 -> 4 * 2^(j+1)


# ------------------------------------------------------------ E4M3 block scale rounded up
def test_e4m3_round_up_is_the_least_value_not_below():
    table = _e4m3_table()
    rng = np.random.default_rng(3)
    vs = np.concatenate([table, (table[1:] + table[:-1]) / 2, np.exp(rng.uniform(-12, 6.2, 4000)), [500.0, 1e30]])
    for v in vs.astype(np.float32):
        b = oracle.e4m3_up(v)
        want = int(np.argmax(table >= v)) if v <= 448 else 0x7E
        assert b == want, (v, b, want)
        assert oracle.e4m3_up(-v) == (want | 0x80)


@pytest.mark.parametrize("seed", range(4))
def test_nvfp4_round_up_rule_bruteforce(seed):
    """Block scale byte = the least E4M3 value >= fl(fl(amax / 6) / s_t)
    (numpy binary32 arithmetic, brute force over the byte table); codes are
    the nearest values of fl(x / S); no code clips by more than the
    binary32 rounding of S."""
    rng = np.random.default_rng(seed + 40)
    M, K = 2, 64
    x = (rng.standard_normal((M, K)) * np.exp(rng.uniform(-4, 4, (M, K // 16)).repeat(16, 1))).astype(np.float32)
    q = oracle.quantize_ex(x, oracle.NVFP4, rule=oracle.RULE_E4M3_UP)
    s_t = np.float32(np.abs(x).max()) / np.float32(2688.0)
    assert q["tscale"][0] == s_t
    table = _e4m3_table()
    nib = _nib(q["codes"], M, K)
    for i in range(M):
        for b in range(K // 16):
            blk = x[i, 16 * b:16 * b + 16]
            t = (np.float32(np.abs(blk).max()) / np.float32(6.0)) / s_t
            enc = int(np.argmax(table >= t)) if t <= 448 else 0x7E
            assert int(q["scales"][i, b]) == enc
            S = np.float32(table[enc]) * s_t
            v = (blk / S).astype(np.float64)
            assert _nearest_ok(v, nib[i, 16 * b:16 * b + 16]).all()
            assert np.abs(v).max() <= 6 * (1 + 2.0 ** -20)     # truncation-free: nothing clips


# ------------------------------------------------------------ four-over-six on MXFP4 groups
def test_mxfp4_four6_reduces_to_the_default_under_truncation_free_scales():
    """With power-of-two scales the amax/4 candidate is 2^k6 or 2^(k6+1), and
    below amax the E2M1 grid under 2^(k6+1) is a subset of the grid under
    2^k6, so its nearest-value error is never lower: the selection always
    keeps the truncation-free exponent.  Random and adversarial groups
    (values in the 4..6 gap, on midpoints, single outliers) agree bit for
    bit with plain MXFP4."""
    rng = np.random.default_rng(8)
    rows = [rng.standard_normal(32) * np.exp(rng.uniform(-10, 10)) for _ in range(300)]
    for base in (4.5, 5.0, 5.5, 5.9, 3.5, 2.5):
        rows.append(np.full(32, base) * np.where(np.arange(32) % 2, -1, 1))
    rows.append(np.r_[50.0, rng.standard_normal(31) * 0.1])
    x = np.asarray(rows, np.float32)
    a = oracle.quantize_ex(x, oracle.MXFP4, four6=True)
    b = oracle.quantize_ex(x, oracle.MXFP4)
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["scales"], b["scales"])


@pytest.mark.parametrize("seed", range(5))
def test_mxfp4_four6_under_the_floor_rule_keeps_the_lower_error(seed):
    """Under the OCP floor rule the candidates are the clipping exponent kf
    and kf + 1; the kept one has the lower squared error (binary64 here, with
    a margin for binary32 near-ties), and its byte is one of the two."""
    rng = np.random.default_rng(seed + 90)
    for _ in range(40):
        x32 = (rng.standard_normal(32) * np.exp(rng.uniform(-5, 5))).astype(np.float32)
        if rng.random() < 0.5:
            x32[rng.integers(32)] *= np.float32(rng.uniform(1.3, 1.99))
        pick, sb, codes = oracle.mxfp4_group(x32, four6=True, rule=oracle.RULE_OCP_FLOOR)
        amax = float(np.abs(x32).max())
        kf = max(k for k in range(-127, 128) if 2.0 ** (k + 2) <= amax)
        k4 = min(k for k in range(-127, 128) if 4 * 2.0 ** k >= amax)

        def sse(k):
            v = (x32 / np.float32(2.0 ** k)).astype(np.float64)
            a = np.minimum(np.abs(v), 6.0)
            near = GRID[np.abs(a[:, None] - GRID).argmin(1)] * np.sign(v)
            return float(((near * 2.0 ** k - x32) ** 2).sum())

        assert sb - 127 in (kf, k4)
        chosen, other = (sse(k4), sse(kf)) if pick else (sse(kf), sse(k4))
        assert chosen <= other * (1 + 1e-5) + 1e-300


def test_mxfp4_four6_picks_the_unclipped_candidate_when_clipping_dominates():
    """Every value at 7.5 * 2^j: the floor exponent clips them all to 6 (error
    1.5 each); the 4-candidate 2^(j+1) puts them on 3.75 -> 4 (error 0.5)."""
    x = np.full(32, 7.5 * 2.0 ** -3, np.float32)
    pick, sb, codes = oracle.mxfp4_group(x, four6=True, rule=oracle.RULE_OCP_FLOOR)
    assert pick == 1 and sb == 127 - 3 + 1


# ------------------------------------------------------------ MXFP4 2D 32x32 tiles
@pytest.mark.parametrize("rounding", [oracle.RNE, oracle.SR])
def test_mxfp4_2d_tiles_match_per_tile_scalar_quantization(rounding):
    """Each 32 x 32 tile has one E8M0 exponent (least k with 6 * 2^k >= the
    tile's amax, exhaustive), codes are the scalar E2M1 rounding of
    fl(x / 2^k) with the random word of X's index, X^T's codes are exactly
    the transpose, and both scale arrays hold the tile's byte."""
    M, K = 64, 96
    x = synth.cfg2_X(M, K, seed=23)
    xf = synth.bf16_bits_to_f32(x)
    q = oracle.quantize_ex(x, oracle.MXFP4, rounding, block2d=True, seed=77, transposed=True)
    nib, nibT = _nib(q["codes"], M, K), _nib(q["codesT"], K, M)
    assert np.array_equal(nibT, nib.T)
    for bi in range(0, M, 32):
        for bj in range(0, K, 32):
            t = xf[bi:bi + 32, bj:bj + 32]
            k = min(k for k in range(-127, 128) if 6 * 2.0 ** k >= float(np.abs(t).max()))
            assert (q["scales"][bi:bi + 32, bj // 32] == k + 127).all()
            assert (q["scalesT"][bj:bj + 32, bi // 32] == k + 127).all()
            for r in range(0, 32, 7):
                for c in range(0, 32, 5):
                    v = np.float32(t[r, c] / np.float32(2.0 ** k))
                    e = (bi + r) * K + bj + c
                    want = oracle.e2m1_rne(v) if rounding == oracle.RNE else oracle.e2m1_sr(v, oracle.sr_word(77, e))
                    assert nib[bi + r, bj + c] == want


# ------------------------------------------------------------ caller-supplied tensor amax, row slices
def test_own_amax_reported_and_reused_gives_the_same_result():
    x = synth.cfg3_X(48, 256, seed=5)
    for rotate in (False, True):
        ref = oracle.quantize(x, oracle.NVFP4, oracle.SR, rotate=rotate, seed=9)
        own = oracle.quantize_ex(x, oracle.NVFP4, oracle.SR, rotate=rotate, seed=9, want_amax=True)
        xf = synth.bf16_bits_to_f32(x)
        if rotate:
            rot = np.stack([oracle.fwht128(r) for r in xf.reshape(-1, 128)])
            want = np.float32(np.abs(rot).max())
        else:
            want = np.float32(np.abs(xf).max())
        assert own["amax"][0] == want
        given = oracle.quantize_ex(x, oracle.NVFP4, oracle.SR, rotate=rotate, seed=9, amax_in=float(want))
        for k in ("codes", "scales", "tscale"):
            assert np.array_equal(ref[k], own[k]) and np.array_equal(ref[k], given[k])


def test_smaller_given_amax_saturates_the_top_blocks():
    """A stale (too small) amax: s_t = fl(amax_in / 2688); blocks whose
    (amax_b / 6) / s_t exceeds 448 take byte 0x7E and their largest element
    saturates to +-6."""
    x = synth.cfg3_X(16, 128, seed=6)
    own = float(np.abs(synth.bf16_bits_to_f32(x)).max())
    q = oracle.quantize_ex(x, oracle.NVFP4, amax_in=own / 4)
    assert q["tscale"][0] == np.float32(np.float32(own / 4) / np.float32(2688))
    top = np.unravel_index(np.abs(synth.bf16_bits_to_f32(x)).argmax(), x.shape)
    assert q["scales"][top[0], top[1] // 16] == 0x7E
    assert (_nib(q["codes"], 16, 128)[top] & 7) == 7


@pytest.mark.parametrize("fmt", [oracle.MXFP4, oracle.NVFP4])
def test_row_slices_with_row_offsets_reassemble_the_whole(fmt):
    """Quantizing row slices apart (random words keyed on the logical index
    through row0, the whole tensor's amax given for NVFP4) reproduces the
    whole-tensor result bit for bit, stochastic rounding included."""
    x = synth.cfg5_A(40, 256, seed=31)
    whole = oracle.quantize(x, fmt, oracle.SR, rotate=True, seed=1234)
    amax = oracle.tensor_amax(x, rotate=True) if fmt == oracle.NVFP4 else None
    parts = [oracle.quantize_ex(x[a:b], fmt, oracle.SR, rotate=True, seed=1234, row0=a, amax_in=amax)
             for a, b in ((0, 7), (7, 8), (8, 33), (33, 40))]
    for k in ("codes", "scales"):
        assert np.array_equal(np.concatenate([p[k] for p in parts]), whole[k])


# ------------------------------------------------------------ MXFP8 GEMM reference
def test_mxfp8_gemm_reference_equals_integer_closed_form():
    """E4M3 codes of small integers under E8M0 scales 2^0 / 2^1: the
    reference equals the exact integer matmul times the scales."""
    rng = np.random.default_rng(12)
    M, N, K = 12, 10, 96
    ints = np.arange(-16, 17)
    enc = {int(v): int(torch.tensor([float(v)]).to(torch.float8_e4m3fn).view(torch.uint8)[0]) for v in ints}
    a = rng.choice(ints, (M, K))
    b = rng.choice(ints, (N, K))
    sa = rng.integers(127, 129, (M, K // 32)).astype(np.uint8)
    sb = rng.integers(127, 129, (N, K // 32)).astype(np.uint8)
    A = {"codes": np.vectorize(enc.get)(a).astype(np.uint8), "scales": sa}
    B = {"codes": np.vectorize(enc.get)(b).astype(np.uint8), "scales": sb}
    r, c = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
    got, mag = oracle.gemm_sampled(A, B, M, N, K, oracle.MXFP8, r.ravel(), c.ravel())
    wa = a * 2.0 ** (np.repeat(sa, 32, 1).astype(np.int64) - 127)
    wb = b * 2.0 ** (np.repeat(sb, 32, 1).astype(np.int64) - 127)
    want = (wa @ wb.T).ravel()
    assert np.array_equal(got, want)
    assert np.array_equal(mag, (np.abs(wa) @ np.abs(wb).T).ravel())
