"""CPU models of the kernels' index mappings and bit-level algorithms,
checked against the plain definitions they implement.  These are written
from the CUDA sources' arithmetic (task -> element mapping, shuffle-stage
data movement, byte-permute tables, the branch-free stochastic rule) and
run without a GPU; the GPU parity tests check the kernels themselves
against the oracle."""
import math
import struct

import numpy as np
import pytest

import oracle

U32 = 0xFFFFFFFF


def byte_perm(x, y, s):
    """CUDA __byte_perm: byte n of the result is byte (s >> 4n) & 7 of {y, x}."""
    b = [(x >> (8 * i)) & 0xFF for i in range(4)] + [(y >> (8 * i)) & 0xFF for i in range(4)]
    return sum(b[(s >> (4 * i)) & 7] << (8 * i) for i in range(4))


# ------------------------------------------------------------------ 2D NVFP4 task mapping
def _sim_quant2d(M, K):
    """k_quant2d: 64 x 32 warp tasks, lane (h, r); every X element read once,
    every output byte (codes, scales, codes^T, scales^T) written once, and
    the wide X^T stores aligned."""
    tiles_k, bands = K // 16, M // 16
    pairs, quads = (tiles_k + 1) // 2, (bands + 3) // 4
    rd = np.zeros((M, K), int)
    c = np.zeros(M * K // 2, int)
    s = np.zeros(M * tiles_k, int)
    cT = np.zeros(K * M // 2, int)
    sT = np.zeros(K * bands, int)
    for task in range(quads * pairs):
        bq = task // pairs
        for lane in range(32):
            h, r = lane >> 4, lane & 15
            tc = (task % pairs) * 2 + h
            if tc >= tiles_k:
                continue
            j0 = tc * 16
            for b in range(4):
                band = bq * 4 + b
                if band >= bands:
                    continue
                i = band * 16 + r
                rd[i, j0:j0 + 16] += 1
                a = (i * K + j0) // 2
                assert a % 8 == 0
                c[a:a + 8] += 1
                s[i * tiles_k + tc] += 1
            jr = j0 + r
            base = jr * M + bq * 64
            if M % 32 == 0 and (bq * 4 + 3) < bands:
                assert (base // 2) % 16 == 0 and (jr * bands + bq * 4) % 4 == 0
            for b in range(4):
                if bq * 4 + b < bands:
                    a = (base + 16 * b) // 2
                    cT[a:a + 8] += 1
                    sT[jr * bands + bq * 4 + b] += 1
    for arr in (rd, c, s, cT, sT):
        assert (arr == 1).all()


@pytest.mark.parametrize("M,K", [(16, 16), (48, 64), (64, 48), (512, 1024), (1008, 528), (1072, 64), (80, 16)])
def test_2d_task_mapping_covers_every_element_once(M, K):
    _sim_quant2d(M, K)


# ------------------------------------------------------------------ stochastic-rounding column kernel mapping
def _sim_cols_sr(M, K, fmt):
    """k_cols_sr: 32 x 64 tasks, lane pairs sharing 4 columns; reads, code
    and scale writes each exactly once, stores aligned to their width."""
    G = 16 if fmt == "nv" else 32
    col_blocks, row_blocks = (K + 63) // 64, (M + 31) // 32
    code_bytes = K * (M if fmt == "mx8" else M // 2)
    reads, wc, ws = {}, {}, {}
    for task in range(row_blocks * col_blocks):
        for lane in range(32):
            q = lane & 1
            i0 = (task // col_blocks) * 32
            jb = (task % col_blocks) * 64 + 4 * (lane >> 1)
            rows = min(32, M - i0)
            if jb >= K:
                continue
            j = jb + 2 * q
            for r in range(rows):
                e = (i0 + r) * K + j
                assert e % 2 == 0
                for d in (0, 1):
                    reads[e + d] = reads.get(e + d, 0) + 1
            for c in (0, 1):
                jr = j + c
                if fmt == "mx8":
                    off, n = jr * M + i0, 32
                    assert off % 16 == 0
                    idx = [jr * (M // 32) + i0 // 32]
                else:
                    off, n = (jr * M + i0) // 2, (16 if rows == 32 else 8)
                    assert off % (16 if (rows == 32 and M % 32 == 0) else 8) == 0
                    idx = ([jr * (M // 32) + i0 // 32] if G == 32 else
                           [jr * (M // 16) + i0 // 16 + g for g in range(rows // 16)])
                    if G == 16 and rows == 32 and M % 32 == 0:
                        assert idx[0] % 2 == 0
                for b in range(n):
                    wc[off + b] = wc.get(off + b, 0) + 1
                for k in idx:
                    ws[k] = ws.get(k, 0) + 1
    assert len(reads) == M * K and set(reads.values()) == {1}
    assert len(wc) == code_bytes and set(wc.values()) == {1} and max(wc) < code_bytes
    assert len(ws) == K * (M // G) and set(ws.values()) == {1}


@pytest.mark.parametrize("fmt,M,K", [("nv", 16, 16), ("nv", 48, 64), ("nv", 80, 36), ("nv", 128, 260),
                                     ("mx", 32, 32), ("mx", 96, 132), ("mx8", 64, 96), ("mx8", 128, 256)])
def test_stochastic_column_mapping_covers_every_element_once(fmt, M, K):
    _sim_cols_sr(M, K, fmt)


def _sim_cols_sr_words(M, K):
    """The Philox words each element of k_cols_sr gets: in step k the lower
    lane of a pair draws row k and the upper lane row 16 + k (counter
    ((i0 + row) K + jb) / 4), each keeps the two words of its own columns
    and passes the other two to its partner.  Returns {(i, j): (counter,
    word index)}."""
    col_blocks, row_blocks = (K + 63) // 64, (M + 31) // 32
    got_words = {}
    for task in range(row_blocks * col_blocks):
        i0 = (task // col_blocks) * 32
        rows = min(32, M - i0)
        for pair in range(16):
            jb = (task % col_blocks) * 64 + 4 * pair
            if jb >= K:
                continue
            for k in range(16):
                wd = [[(((i0 + k + 16 * q) * K + jb) >> 2, t) for t in range(4)] for q in (0, 1)]
                own = [(wd[q][2], wd[q][3]) if q else (wd[q][0], wd[q][1]) for q in (0, 1)]
                sent = [(wd[q][0], wd[q][1]) if q else (wd[q][2], wd[q][3]) for q in (0, 1)]
                got = [sent[1], sent[0]]
                for q in (0, 1):
                    j = jb + 2 * q
                    use_k = got[q] if q else own[q]
                    for c in (0, 1):
                        got_words[(i0 + k, j + c)] = use_k[c]
                    if 16 + k < rows:
                        use_16k = own[q] if q else got[q]
                        for c in (0, 1):
                            got_words[(i0 + 16 + k, j + c)] = use_16k[c]
    return got_words


@pytest.mark.parametrize("M,K", [(16, 16), (48, 64), (80, 36), (128, 260)])
def test_stochastic_column_words_are_each_elements_own(M, K):
    """Every element (i, j) rounds with word (i K + j) mod 4 of Philox call
    (i K + j) / 4, the word the row-wise pass and the oracle use for it."""
    words = _sim_cols_sr_words(M, K)
    assert len(words) == M * K
    for (i, j), w in words.items():
        e = i * K + j
        assert w == (e >> 2, e & 3), (i, j)


# ------------------------------------------------------------------ nibble transposes
M4, NM4 = 0x0F0F0F0F, 0xF0F0F0F0
PERM = {4: (0x5410, 0x7632, 0x3254, 0x5410, 0x3276, 0x7610),     # send up / lo, merge word 0 up / lo, word 1 up / lo
        2: (0x6420, 0x7531, 0x3514, 0x5240, 0x3716, 0x7260)}


def _pair_stages(W, n, pairs):
    """Stages 4, 2, 1 of the transpose on word pairs (2k, 2k + 1) of n lanes."""
    for s in (4, 2):
        su, sl, lu, ll, hu, hl = PERM[s]
        snd = [[byte_perm(W[r][2 * k], W[r][2 * k + 1], su if r & s else sl) for k in range(pairs)] for r in range(n)]
        for r in range(n):
            up = r & s
            for k in range(pairs):
                g = snd[r ^ s][k]
                W[r][2 * k] = byte_perm(W[r][2 * k], g, lu if up else ll)
                W[r][2 * k + 1] = byte_perm(W[r][2 * k + 1], g, hu if up else hl)
    snd = []
    for r in range(n):
        up = r & 1
        snd.append([(((W[r][2 * k] >> (0 if up else 4)) & M4) | ((W[r][2 * k + 1] << (4 if up else 0)) & NM4)) & U32
                    for k in range(pairs)])
    for r in range(n):
        up = r & 1
        km = NM4 if up else M4
        for k in range(pairs):
            g = snd[r ^ 1][k]
            W[r][2 * k] = ((W[r][2 * k] & km) | ((g << (0 if up else 4)) & ~km & U32)) & U32
            W[r][2 * k + 1] = ((W[r][2 * k + 1] & km) | ((g >> (4 if up else 0)) & ~km & U32)) & U32


def _transpose16(W):
    """transpose16x16_nibbles on 16 lanes of (lo, hi)."""
    W = [list(w) for w in W]
    snd = [(W[r][0] if r & 8 else W[r][1]) for r in range(16)]
    for r in range(16):
        W[r][0 if r & 8 else 1] = snd[r ^ 8]
    _pair_stages(W, 16, 1)
    return W


def _transpose32(W):
    """transpose32x32_nibbles on 32 lanes of 4 words."""
    W = [list(w) for w in W]
    snd = [((W[r][0], W[r][1]) if r & 16 else (W[r][2], W[r][3])) for r in range(32)]
    for r in range(32):
        if r & 16:
            W[r][0], W[r][1] = snd[r ^ 16]
        else:
            W[r][2], W[r][3] = snd[r ^ 16]
    snd = [((W[r][0], W[r][2]) if r & 8 else (W[r][1], W[r][3])) for r in range(32)]
    for r in range(32):
        if r & 8:
            W[r][0], W[r][2] = snd[r ^ 8]
        else:
            W[r][1], W[r][3] = snd[r ^ 8]
    _pair_stages(W, 32, 2)
    return W


@pytest.mark.parametrize("n", [16, 32])
def test_nibble_transposes_are_transposes(n):
    rng = np.random.default_rng(n)
    words = n // 8
    for _ in range(100):
        mat = rng.integers(0, 16, (n, n))
        W = [[int(sum(int(mat[r][8 * k + j]) << (4 * j) for j in range(8))) for k in range(words)] for r in range(n)]
        T = _transpose16(W) if n == 16 else _transpose32(W)
        got = np.array([[(T[r][j // 8] >> (4 * (j % 8))) & 0xF for j in range(n)] for r in range(n)])
        assert np.array_equal(got, mat.T)


# ------------------------------------------------------------------ E2M1 -> bf16 byte-permute decode
def test_e2m1_byte_permute_decode_is_exact_for_every_code_pair():
    mag = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for w16 in range(65536):
        sel = w16 & 0x7777
        hi = byte_perm(0x3F3F3F00, 0x40404040, sel)
        lo = byte_perm(0xC0800000, 0xC0804000, sel)
        p01 = byte_perm(lo, hi, 0x5140) | ((w16 << 12) & 0x8000) | ((w16 << 24) & 0x80000000)
        p23 = byte_perm(lo, hi, 0x7362) | ((w16 << 4) & 0x8000) | ((w16 << 16) & 0x80000000)
        got = [p01 & 0xFFFF, p01 >> 16, p23 & 0xFFFF, p23 >> 16]
        for t in range(4):
            c = (w16 >> (4 * t)) & 0xF
            want = struct.unpack("<I", struct.pack("<f", -mag[c & 7] if c & 8 else mag[c & 7]))[0] >> 16
            assert got[t] == want, (w16, t)


# ------------------------------------------------------------------ branch-free E4M3 stochastic rule
def _f2u(x):
    return struct.unpack("<I", struct.pack("<f", float(x)))[0]


def _u2f(u):
    return np.float32(struct.unpack("<f", struct.pack("<I", u & U32))[0])


def _e4m3_sr_definition(a, w):
    """The rule: lo <= a < hi adjacent E4M3 magnitudes, up iff
    (w >> 8) * 2^-24 < (a - lo) / (hi - lo), in exact rationals; <= 448."""
    from fractions import Fraction
    a = Fraction(float(a))
    e = max(math.floor(math.log2(a)) if a > 0 else -6, -6)
    sp = Fraction(2) ** (e - 3)
    lo = (a // sp) * sp
    up = Fraction(w >> 8, 1 << 24) < (a - lo) / sp
    return float(min(lo + sp if up else lo, Fraction(448)))


def _e4m3_sr2_model(a, w):
    """e4m3_sr2 on one value: the dither on the bits for |v| >= 2^-6, the
    2^-9 grid below, both in binary32 as the kernel computes them."""
    bits = _f2u(np.float32(a)) & 0x7FFFFFFF
    rn = (bits + (0xFFFFF - (w >> 12))) & 0xFFF00000
    t9 = np.float32(_u2f(bits) * np.float32(512))
    f9 = np.float32(np.trunc(t9))
    frac24 = np.float32(np.float32(t9 - f9) * np.float32(16777216))
    rs = np.float32((np.float32(f9 + 1) if np.float32(w >> 8) < frac24 else f9) * np.float32(2.0 ** -9))
    return float(min(_u2f(rn) if bits >= 0x3C800000 else rs, np.float32(448)))


def test_branch_free_e4m3_rule_equals_the_definition():
    rng = np.random.default_rng(5)
    vals = np.concatenate([np.abs(rng.standard_normal(400)) * s for s in (1e-4, 1e-2, 0.1, 1, 30, 200)] +
                          [np.array([2.0 ** -6, 2.0 ** -6 * (1 - 2.0 ** -24), 448, 449, 479, 2.0 ** -149, 2.0 ** -9])])
    with np.errstate(over="ignore", invalid="ignore"):
        for a in vals.astype(np.float32):
            if a == 0:
                continue
            for w in (int(rng.integers(0, 2 ** 32)), 0, U32, 0x80000000, 0x7FFFF000):
                assert _e4m3_sr2_model(a, w) == _e4m3_sr_definition(a, w), (float(a), w)


# ------------------------------------------------------------------ KL calibration, one warp per candidate
def _e2m1_level(b, i):
    num, mid8, level = 24 * (2 * b + 1), (2, 6, 10, 14, 20, 28, 40), 0
    for t in range(7):
        rhs = mid8[t] * i
        if num > rhs:
            level = t + 1
        else:
            if num == rhs:
                level = t + 1 if t & 1 else t
            break
    return level


def _kl_warp_model(hist, levels, grid):
    """k_kl as written: prefix sums, level runs from floor(i / levels) or a
    binary search on the E2M1 level function, terms rounded then added in
    ascending bin order."""
    bins = len(hist)
    first = 8 if grid else levels
    ph, pnz = [0], [0]
    for h in hist:
        ph.append(ph[-1] + int(h))
        pnz.append(pnz[-1] + (h != 0))
    out = []
    for i in range(first, bins + 1):
        kept, outl = ph[i], ph[bins] - ph[i]
        tp, tq = float(kept + outl), float(kept)
        start = [0] * 9
        if grid:
            for t in range(7):
                lo, hi = 0, i
                while lo < hi:
                    mid = (lo + hi) >> 1
                    lo, hi = (lo, mid) if _e2m1_level(mid, i) >= t + 1 else (mid + 1, hi)
                start[t + 1] = lo
            start[8] = i
        per = 1 if grid else i // levels
        d = 0.0
        if tp != 0.0:
            if tq == 0.0:
                d = math.inf
            else:
                for b in range(i):
                    pb = int(hist[b]) + (outl if b == i - 1 else 0)
                    term = 0.0
                    if pb:
                        if grid:
                            lvl = _e2m1_level(b, i)
                            b0, b1 = start[lvl], start[lvl + 1]
                        else:
                            lvl = min(b // per, levels - 1)
                            b0, b1 = lvl * per, (i if lvl == levels - 1 else lvl * per + per)
                        mass, nz = ph[b1] - ph[b0], pnz[b1] - pnz[b0]
                        if b1 == i and hist[i - 1] == 0 and outl != 0:
                            nz += 1
                        qb = mass / nz if nz else 0.0
                        if qb == 0.0:
                            term = math.inf
                        else:
                            pp, qq = pb / tp, qb / tq
                            term = pp * math.log(pp / qq)
                    d += term
        out.append(d)
    return np.array(out)


def test_kl_warp_kernel_algorithm_matches_the_oracle():
    rng = np.random.default_rng(3)
    cases = []
    for trial in range(8):
        bins = int(rng.choice([16, 64, 200, 256]))
        h = rng.integers(0, 50, bins).astype(np.uint64)
        h[rng.random(bins) < 0.4] = 0
        if trial % 3 == 0:
            h[bins // 2:] = 0
            h[-1] = 7
        cases.append(h)
    h = np.zeros(64, np.uint64)
    h[:8], h[63] = 100, 5
    cases.append(h)
    for h in cases:
        for grid, levels in ((0, 4), (0, 8), (1, 8), (0, 2)):
            if levels > len(h):
                continue
            _, ref = oracle.kl_calibrate(h, levels, grid)
            new = _kl_warp_model(h, levels, grid)
            assert np.array_equal(np.isinf(ref), np.isinf(new))
            f = np.isfinite(ref)
            assert np.allclose(new[f], ref[f], rtol=1e-13, atol=1e-300)


# ------------------------------------------------------------------ packed E2M1 stochastic grid
def _rz_f32(x):
    """An exact positive rational rounded toward zero to binary32 (normal range)."""
    from fractions import Fraction
    e = x.numerator.bit_length() - x.denominator.bit_length()
    if Fraction(2) ** e > x:
        e -= 1
    ulp = Fraction(2) ** (e - 23)
    return np.float32(float((x // ulp) * ulp))


def _e2m1_sr_grid2_model(v, w):
    """e2m1_sr_grid2 on one element of the pair, step by step in binary32 as
    the kernel computes it: the spacing exponent clamped below at 127, the
    round-toward-zero add of 1.5 * 2^47 that leaves floor(q24 / 2^24) * 2^24,
    the integer compare of the random word's top 24 bits against the
    fraction, the sign copied; then the saturating E2M1 conversion."""
    from fractions import Fraction
    b = _f2u(v) & 0x7FFFFFFF
    m = max(b >> 23, 127)
    inv, sp = _u2f((279 - m) << 23), _u2f((m - 25) << 23)
    C = np.float32(1.5 * 2.0 ** 47)
    q24 = np.float32(_u2f(b) * inv)
    assert Fraction(float(q24)) == Fraction(float(_u2f(b))) * Fraction(float(inv))   # a power-of-two scaling
    fl24 = np.float32(_rz_f32(Fraction(float(q24)) + Fraction(float(C))) - C)
    frac = np.float32(q24 - fl24)
    up = np.float32(w >> 8) < frac
    r = np.float32(np.float32(fl24 + (np.float32(16777216.0) if up else np.float32(0))) * sp)
    r_signed = _u2f(_f2u(r) | (_f2u(v) & 0x80000000))
    return oracle.e2m1_rne(float(r_signed))          # cvt.rn.satfinite.e2m1x2: r is a grid value or >= 6


def test_packed_e2m1_stochastic_grid_equals_the_definition():
    rng = np.random.default_rng(11)
    vals = np.concatenate([rng.standard_normal(500) * s for s in (1e-3, 0.1, 0.4, 1, 2.5, 5)] +
                          [rng.uniform(-7.9, 7.9, 500),
                           np.array([0.0, -0.0, 0.25, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, 6.5, 8.0, 100.0, 1e30,
                                     2.0 ** -149, -(2.0 ** -126), 0.5 - 2.0 ** -26, 6.0 - 2.0 ** -21])])
    for v in vals.astype(np.float32):
        for w in (int(rng.integers(0, 2 ** 32)), int(rng.integers(0, 2 ** 32)), 0, U32, 0x80000000, 0xFF):
            assert _e2m1_sr_grid2_model(v, w) == oracle.e2m1_sr(float(v), w), (float(v), w)


# ------------------------------------------------------------------ scale exponents and E4M3 scale bytes
def _scale_exp_model(amax, top_frac, top_e):
    """scale_exp: amax = (1 + f 2^-23) 2^e from its bits (subnormals
    normalised by their leading one), k = e - top_e, plus one when the
    fraction exceeds top's, clamped to [-127, 127]."""
    u = _f2u(amax) & 0x7FFFFFFF
    if u == 0:
        return -127
    E = u >> 23
    if E == 0:
        lead = u.bit_length() - 1
        e, f = lead - 149, (u << (23 - lead)) & 0x7FFFFF
    else:
        e, f = E - 127, u & 0x7FFFFF
    k = e - top_e if f <= top_frac else e - top_e + 1
    return max(-127, min(127, k))


def _scale_exp_floor_model(amax, emax):
    u = _f2u(amax) & 0x7FFFFFFF
    if u == 0:
        return -127
    E = u >> 23
    e = (u.bit_length() - 1) - 149 if E == 0 else E - 127
    return max(-127, min(127, e - emax))


def _amax_cases(rng):
    v = [0.0, 2.0 ** -149, 3 * 2.0 ** -149, 2.0 ** -127, 2.0 ** -126, 3.4028234663852886e38, 1.0, 6.0, 4.0, 448.0]
    for top in (4.0, 6.0, 448.0, 1.0, 8.0):
        for k in (-149, -140, -130, -127, -126, -120, -3, 0, 1, 7, 100, 119, 120, 125, 126):
            b = top * 2.0 ** k
            if b < 3.4e38:
                f = np.float32(b)
                v += [float(f), float(np.nextafter(f, np.float32(np.inf))), float(np.nextafter(f, np.float32(0)))]
    v += list(np.abs(rng.standard_normal(400)) * 10.0 ** rng.integers(-40, 38, 400))
    return [np.float32(x) for x in v if np.isfinite(np.float32(x))]


def test_scale_exponents_from_bits_equal_the_definitions():
    rng = np.random.default_rng(17)
    for a in _amax_cases(rng):
        for top_frac, top_e, top in ((0x400000, 2, 6.0), (0, 2, 4.0), (0x600000, 8, 448.0)):
            assert _scale_exp_model(a, top_frac, top_e) == oracle.scale_exp(float(a), top), (float(a), top)
        assert _scale_exp_floor_model(a, 2) == oracle.scale_exp_floor(float(a), 2), float(a)


def _e4m3_value_model(b):
    E, m = (b >> 3) & 15, b & 7
    mag = np.float32(m) * _u2f(118 << 23) if E == 0 else _u2f(((E + 120) << 23) | (m << 20))
    return -mag if b & 0x80 else mag


def _nv_scale_round_model(r, up):
    """The last stage of nv_scale_byte: a quotient of 448 or more (or NaN)
    takes 0x7E; else the nearest E4M3 byte, stepped up once when its value
    lies below r (rule E4M3_UP)."""
    if not r < 448.0:
        return 0x7E
    enc = oracle.e4m3_rne(float(r))         # the hardware E4M3 conversion, pinned on the GPU
    if up and enc < 0x7E and _e4m3_value_model(enc) < r:
        enc += 1
    return enc


def test_e4m3_bit_field_decode_and_round_up_equal_the_definitions():
    for b in range(256):
        if b & 0x7F != 0x7F:                 # 0x7F / 0xFF are NaN
            assert float(_e4m3_value_model(b)) == oracle.e4m3_value(b), b
    rng = np.random.default_rng(19)
    ts = [np.float32(x) for x in np.abs(rng.standard_normal(3000)) * 10.0 ** rng.integers(-4, 3, 3000)]
    ts += [np.float32(oracle.e4m3_value(b)) for b in range(0x7F)]
    ts += [np.nextafter(t, np.float32(np.inf)) for t in ts[-0x7F:]]
    ts += [np.float32(x) for x in (2.0 ** -10, 1e-30, 0.0, 448.0, 449.0, 1e30)]
    for t in ts:
        assert _nv_scale_round_model(t, True) == oracle.e4m3_up(float(t)), float(t)


def _e4m3_sr_scalar_model(v, w):
    """e4m3_sr (one value): in the normal binades lo keeps three mantissa
    bits, the spacing and its inverse come from the exponent field; below
    2^-6 both come from the 2^-9 grid; up iff fl((w >> 8) 2^-24) < fl((a -
    lo) / spacing); the result saturates at 448 and takes v's sign bit."""
    sign = (_f2u(v) >> 24) & 0x80
    a = np.float32(abs(v))
    bits = _f2u(a)
    if a >= np.float32(0.015625):
        spb = (bits & 0x7F800000) - (3 << 23)
        lo, sp, inv = _u2f(bits & 0x7FF00000), _u2f(spb), _u2f((254 << 23) - spb)
    else:
        lo = np.float32(np.float32(np.trunc(np.float32(a * np.float32(512)))) * np.float32(0.001953125))
        sp, inv = np.float32(0.001953125), np.float32(512)
    p = np.float32(np.float32(a - lo) * inv)
    u = np.float32(np.float32(w >> 8) * np.float32(5.9604644775390625e-08))
    rr = np.float32(lo + sp) if u < p else lo
    rr = min(rr, np.float32(448))
    return oracle.e4m3_rne(float(rr)) | sign


def test_scalar_e4m3_stochastic_rule_equals_the_oracle():
    rng = np.random.default_rng(23)
    vals = np.concatenate([rng.standard_normal(300) * s for s in (1e-4, 3e-3, 0.02, 1, 30, 200)] +
                          [np.array([2.0 ** -6, -(2.0 ** -6) * (1 - 2.0 ** -24), 448, -449, 479, 2.0 ** -149,
                                     2.0 ** -9, 0.0, -0.0])])
    with np.errstate(over="ignore", invalid="ignore"):
        for v in vals.astype(np.float32):
            for w in (int(rng.integers(0, 2 ** 32)), 0, U32, 0x80000000, 0x7FFFF000):
                assert _e4m3_sr_scalar_model(v, w) == oracle.e4m3_sr(float(v), w), (float(v), w)


def _e2m1_sr_grid_scalar_model(v, w):
    """e2m1_sr_grid (one value): the spacing exponent clamped to [127, 129],
    so values from 8 on stay in the 4..6 spacing and the result is clamped
    to 6 in binary32 before the conversion."""
    from fractions import Fraction
    a = np.float32(abs(v))
    m = min(max(_f2u(a) >> 23, 127), 129)
    inv, sp = _u2f((279 - m) << 23), _u2f((m - 25) << 23)
    C = np.float32(211106232532992.0)
    q24 = np.float32(a * inv)
    fl24 = np.float32(_rz_f32(Fraction(float(q24)) + Fraction(float(C))) - C)
    frac = np.float32(q24 - fl24)
    r24 = np.float32(fl24 + np.float32(16777216.0)) if np.float32(w >> 8) < frac else fl24
    r = min(np.float32(r24 * sp), np.float32(6.0))
    return oracle.e2m1_rne(float(_u2f(_f2u(r) | (_f2u(v) & 0x80000000))))


def test_scalar_e2m1_stochastic_grid_equals_the_definition():
    rng = np.random.default_rng(29)
    vals = np.concatenate([rng.standard_normal(400) * s for s in (1e-3, 0.3, 1, 2.5, 5)] +
                          [rng.uniform(-7.9, 7.9, 400),
                           np.array([0.0, -0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, 6.5, 8.0, 100.0, 1e6,
                                     2.0 ** -149, 0.5 - 2.0 ** -26, 6.0 - 2.0 ** -21])])
    for v in vals.astype(np.float32):
        for w in (int(rng.integers(0, 2 ** 32)), 0, U32, 0x80000000):
            assert _e2m1_sr_grid_scalar_model(v, w) == oracle.e2m1_sr(float(v), w), (float(v), w)


# ------------------------------------------------------------------ folded rotation normalisation (MXFP4 RNE)
def test_folded_normalisation_gives_the_same_codes():
    """The plain MXFP4 round-to-nearest path multiplies the unnormalised
    butterfly sums once by fl(c 2^-k), c = fl(2^-3.5), instead of by c and
    then by 2^-k.  For k <= 120 the folded multiplier is exact and both give
    the same E2M1 code: equal values when the product is normal, and a zero
    of x's sign both ways when it is subnormal.  The group maximum is
    fl(amax_raw c) either way (rounding is monotone)."""
    c = _u2f(0x3DB504F3)
    rng = np.random.default_rng(31)
    xs = (rng.standard_normal(4000) * 10.0 ** rng.integers(-38, 38, 4000)).astype(np.float32)
    xs = np.concatenate([xs, np.array([0.0, -0.0, 2.0 ** -149, -(2.0 ** -126), 3.0e38], np.float32)])
    for k in (-127, -126, -60, -3, 0, 2, 5, 40, 100, 119, 120):
        folded = np.float32(c * np.float32(2.0 ** -k))
        assert float(folded) == float(c) * 2.0 ** -k            # exact for k <= 120
        with np.errstate(over="ignore"):
            for x in xs:
                a = np.float32(x * folded)
                b = np.float32(np.float32(x * c) * np.float32(2.0 ** -k))
                if not (np.isfinite(a) and np.isfinite(b)):
                    continue                                    # beyond any group's range
                assert oracle.e2m1_rne(float(a)) == oracle.e2m1_rne(float(b)), (float(x), k)
    raw = np.abs(xs[:64])
    assert np.float32(raw.max() * c) == np.max(np.abs((raw * c).astype(np.float32)))
