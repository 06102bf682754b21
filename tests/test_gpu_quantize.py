"""GPU parity of the 1D quantize paths, dequantize and the FP32-scale modes.

Every test calls libqfp4 through its C ABI (the Python binding only marshals)
and compares with the CPU oracle element by element: codes, scales and the
tensor scale bit-exactly.
"""
import numpy as np
import pytest
import torch

import bit_fwht_hadamard_b200 as q
import oracle
import synth
import gpu_util as G
from gpu_util import blocks_to_rows, encode_input, host, mismatch_report, nvfp4_boundary_blocks, to_dev

pytestmark = pytest.mark.gpu

FMTS = [(q.MXFP4, oracle.MXFP4), (q.NVFP4, oracle.NVFP4)]


def _cmp(got: dict, ref: dict, keys=("codes", "scales", "codesT", "scalesT", "tscale")):
    for k in keys:
        if k in ref:
            g = host(got[k]).reshape(ref[k].shape)
            assert np.array_equal(g.view(np.uint8), np.asarray(ref[k]).view(np.uint8)), mismatch_report(
                g.view(np.uint8), np.asarray(ref[k]).view(np.uint8), k)


# shapes spanning several 32K-element tiles, tiles with ragged ends, tails
# that are not a multiple of 64 elements, single rows
SHAPES = [(1, 128), (3, 256), (37, 384), (600, 512), (1000, 640), (7, 96), (5, 48), (1, 32)]


@pytest.mark.parametrize("M,K", SHAPES)
@pytest.mark.parametrize("fmt", FMTS, ids=["mxfp4", "nvfp4"])
@pytest.mark.parametrize("rounding", [q.RNE, q.SR], ids=["rne", "sr"])
@pytest.mark.parametrize("rotate", [False, True], ids=["plain", "rot"])
def test_quantize_1d_matches_oracle(M, K, fmt, rounding, rotate):
    g = 32 if fmt[0] == q.MXFP4 else 16
    if K % g or (rotate and K % 128):
        pytest.skip("shape not valid for this mode")
    x = synth.cfg2_X(M, K, seed=M * 1000 + K)
    got = G.quantize(to_dev(x), fmt[0], rounding, rotate=rotate, seed=0xDEADBEEF12345)
    ref = oracle.quantize(x, fmt[1], rounding, rotate=rotate, seed=0xDEADBEEF12345)
    _cmp(got, ref)


@pytest.mark.parametrize("M,K", [(1, 16), (37, 384), (600, 512), (5, 48)])
@pytest.mark.parametrize("rotate", [False, True], ids=["plain", "rot"])
def test_four_over_six_matches_oracle(M, K, rotate):
    if rotate and K % 128:
        pytest.skip()
    x = synth.cfg3_X(M, K, seed=M + K)
    got = G.quantize(to_dev(x), q.NVFP4, q.RNE, rotate=rotate, four6=True)
    ref = oracle.quantize(x, oracle.NVFP4, oracle.RNE, rotate=rotate, four6=True)
    _cmp(got, ref)


@pytest.mark.parametrize("fmt", FMTS, ids=["mxfp4", "nvfp4"])
@pytest.mark.parametrize("rounding", [q.RNE, q.SR], ids=["rne", "sr"])
def test_float32_input(fmt, rounding):
    W = np.zeros((256, 800), np.float32)
    W[:, :784] = synth.cfg1_W()
    W[17, 300] = 50 * np.abs(W).max()
    got = G.quantize(to_dev(W), fmt[0], rounding, seed=3)
    ref = oracle.quantize(W, fmt[1], rounding, seed=3)
    _cmp(got, ref)


def test_full_size_activation_quantize_rne_and_sr():
    """X bf16 4096 x 4096 with 40 x20 channels, FWHT-128 + MXFP4, RNE and SR seed 7."""
    x = synth.cfg2_X()
    xd = to_dev(x)
    for rounding, seed in ((q.RNE, 0), (q.SR, 7)):
        got = G.quantize(xd, q.MXFP4, rounding, rotate=True, seed=seed)
        ref = oracle.quantize(x, oracle.MXFP4, rounding, rotate=True, seed=seed)
        _cmp(got, ref)


def test_full_size_nvfp4_four6_forward_operands():
    """X 8192 x 4096 Student-t(3)*0.5 and W 11008 x 4096 N(0, 0.02^2), NVFP4 + four-over-six."""
    for x in (synth.cfg3_X(), synth.cfg3_W()):
        got = G.quantize(to_dev(x), q.NVFP4, q.RNE, four6=True)
        ref = oracle.quantize(x, oracle.NVFP4, oracle.RNE, four6=True)
        _cmp(got, ref)


def test_degenerate_inputs():
    z = np.zeros((64, 256), np.uint16)
    for fmt in FMTS:
        got = G.quantize(to_dev(z), fmt[0], q.RNE)
        _cmp(got, oracle.quantize(z, fmt[1], oracle.RNE))
    z[3, 5] = 0x8000                                   # a negative zero
    x = synth.cfg2_X(64, 256, seed=9)
    x[10, :64] = 0                                     # an all-zero group inside a nonzero tensor
    x[11, :64] = 0x8000
    x[12, 0] = 0x0001                                  # a bf16 subnormal
    for fmt in FMTS:
        for rounding in (q.RNE, q.SR):
            for arr in (z, x):
                _cmp(G.quantize(to_dev(arr), fmt[0], rounding, seed=1),
                     oracle.quantize(arr, fmt[1], rounding, seed=1))
    # M = 0 is a no-op that succeeds
    e = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    G.quantize(e, q.MXFP4)


@pytest.mark.parametrize("rounding", [q.RNE, q.SR], ids=["rne", "sr"])
def test_every_bf16_value_up_to_6(rounding):
    """Every finite bf16 value with |x| <= 6 (both signs, zeros and subnormals)
    goes through an MXFP4 group whose first element is 6.0, so k = 0 and the
    code is the rounding of x itself: pins the E2M1 conversion, its ties and
    the sign of zero on the GPU against the oracle."""
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    f = synth.bf16_bits_to_f32(h)
    vals = h[np.isfinite(f) & (np.abs(f) <= 6.0)]
    per = 31
    n_groups = -(-len(vals) // per)
    x = np.zeros((n_groups, 32), np.uint16)
    x[:, 0] = 0x40C0                                    # 6.0
    flat = np.zeros(n_groups * per, np.uint16)
    flat[:len(vals)] = vals
    x[:, 1:] = flat.reshape(n_groups, per)
    rows = -(-n_groups // 4)
    X = np.zeros((rows * 4, 32), np.uint16)
    X[:n_groups] = x
    X[n_groups:, 0] = 0x40C0
    X = X.reshape(rows, 128)
    got = G.quantize(to_dev(X), q.MXFP4, rounding, seed=77)
    ref = oracle.quantize(X, oracle.MXFP4, rounding, seed=77)
    assert (ref["scales"] == 127).all()
    _cmp(got, ref)


def test_large_dynamic_range():
    rng = np.random.default_rng(5)
    z = rng.standard_normal(64 * 512) * np.exp(rng.uniform(-60, 60, 64 * 512))
    x = synth.to_bf16(z, (64, 512))
    for fmt in FMTS:
        for rounding in (q.RNE, q.SR):
            _cmp(G.quantize(to_dev(x), fmt[0], rounding, seed=2), oracle.quantize(x, fmt[1], rounding, seed=2))


@pytest.mark.parametrize("kind", ["bf16", "f32"])
@pytest.mark.parametrize("four6", [False, True], ids=["rne", "four6"])
def test_nvfp4_rounding_boundaries(kind, four6):
    """Quotients x / S exactly on (bf16 input) or within 3 ulps of (float32
    input) every E2M1 midpoint, and block maxima on or next to the E4M3
    midpoints (normal and subnormal): codes and scales agree with the
    oracle's IEEE divisions bit for bit, through the TMA kernel (bf16) and
    the direct kernel (float32)."""
    x = encode_input(blocks_to_rows(nvfp4_boundary_blocks(kind)), kind)
    got = G.quantize(to_dev(x), q.NVFP4, q.RNE, four6=four6)
    ref = oracle.quantize(x, oracle.NVFP4, oracle.RNE, four6=four6)
    _cmp(got, ref)


def test_misaligned_pointer_is_rejected():
    x = torch.zeros(64 * 128 + 8, dtype=torch.bfloat16, device="cuda")
    codes = torch.empty(64 * 64, dtype=torch.uint8, device="cuda")
    scales = torch.empty(64 * 4, dtype=torch.uint8, device="cuda")
    st = q.qfp4_quantize(x.data_ptr() + 2, q.BF16, 64, 128, q.MXFP4, q.RNE, 0, 0, 0, 0, codes.data_ptr(),
                         scales.data_ptr(), None, None, None, None, 0, torch.cuda.current_stream().cuda_stream)
    assert st == q.ERR_ALIGN
    assert q.qfp4_last_device_error() == 0


# ------------------------------------------------------------------ dequantize
@pytest.mark.parametrize("fmt", FMTS, ids=["mxfp4", "nvfp4"])
@pytest.mark.parametrize("out", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_dequantize_matches_oracle(fmt, out):
    M, K = 300, 512
    x = synth.cfg3_X(M, K, seed=77)
    ref_q = oracle.quantize(x, fmt[1])
    gq = G.quantize(to_dev(x), fmt[0])
    got = host(G.dequantize(gq, M, K, fmt[0], out))
    exact = oracle.dequantize(ref_q["codes"], ref_q["scales"], ref_q.get("tscale"), M, K, fmt[1])
    if out == torch.float32:
        assert np.array_equal(got, oracle.f64_to_f32_array(exact))
    else:
        sub = np.s_[:8, :]                          # the bf16 rounding reference is scalar: check a slice
        want = oracle.f64_to_bf16_array(exact[sub])
        assert np.array_equal(got[sub].view(np.uint16), want)


# ------------------------------------------------------------------ fp32-scale modes
@pytest.mark.parametrize("gran", [q.GRAN_TENSOR, q.GRAN_ROW, q.GRAN_GROUP16, q.GRAN_GROUP32])
def test_fp32_scale_modes_match_oracle(gran):
    W = np.zeros((256, 800), np.float32)
    W[:, :784] = synth.cfg1_W()
    W[17, 300] = 50 * np.abs(W).max()
    got = G.quantize_fp32scale(to_dev(W), gran)
    ref = oracle.quantize_fp32scale(W, gran)
    assert np.array_equal(host(got["codes"]), ref["codes"])
    assert np.array_equal(host(got["scales"]).view(np.uint32), ref["scales"].view(np.uint32))


# every code under every scale byte, tensor scales that reach each rounding case
_CODES16 = np.array([0x10, 0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE], np.uint8)   # codes 0..15 in order
_TSCALES = [1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, (1 + 2.0 ** -8) / 3, (1 + 2.0 ** -8) / 5,
            (1 + 2.0 ** -7) / 7, 2.0 ** -130, 1.0e35]


@pytest.mark.parametrize("out", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_dequantize_every_code_and_scale(out):
    """All 16 codes under each of the 256 scale bytes, NVFP4 (one block per
    byte) under tensor scales whose products land on bfloat16 midpoints --
    exactly, and with a nonzero remainder -- below 2^-100 and near the top
    of the range; MXFP4 likewise over its 256 bytes.  NaN scale bytes give
    NaN; every other output equals the exact value rounded once."""
    midpoint_with_remainder = 0
    cases = [(q.NVFP4, oracle.NVFP4, 16, np.float32(t)) for t in _TSCALES] + [(q.MXFP4, oracle.MXFP4, 32, None)]
    for fmt, ofmt, K, ts in cases:
        M = 256
        codes = np.tile(_CODES16, (M, K // 16))                    # K / 2 bytes a row
        scales = np.arange(256, dtype=np.uint8).reshape(M, 1)      # row r: scale byte r
        dq = {"codes": torch.from_numpy(codes).cuda(), "scales": torch.from_numpy(scales).cuda()}
        if ts is not None:
            dq["tscale"] = torch.tensor([float(ts)], dtype=torch.float32, device="cuda")
        got = host(G.dequantize(dq, M, K, fmt, out))
        exact = oracle.dequantize(codes, scales, None if ts is None else np.float32(ts), M, K, ofmt)
        nan = np.isnan(exact)
        assert nan.any()                                           # E8M0 0xFF / E4M3 0x7F, 0xFF
        fin = ~nan
        if out == torch.float32:
            assert np.isnan(got[nan]).all()
            assert np.array_equal(got[fin].view(np.uint32), oracle.f64_to_f32_array(exact[fin]).view(np.uint32))
        else:
            g16 = got.view(np.uint16)
            assert (((g16[nan] & 0x7F80) == 0x7F80) & ((g16[nan] & 0x7F) != 0)).all()
            assert np.array_equal(g16[fin], oracle.f64_to_bf16_array(exact[fin]))
            p = oracle.f64_to_f32_array(exact[fin])
            midpoint_with_remainder += int(np.sum(((p.view(np.uint32) & 0xFFFF) == 0x8000) &
                                                  (p.astype(np.float64) != exact[fin])))
    if out == torch.bfloat16:
        assert midpoint_with_remainder > 0


def test_quantize_repeatable_full_size():
    """Repeated calls on one full-size input (G 8192 x 4096) give bit-identical
    outputs for every format of the TMA-fed kernel: guards its shared-memory
    ring against a refill landing before the reads of a stage are done."""
    x = to_dev(synth.cfg4_G())
    calls = [lambda: G.quantize(x, q.MXFP4, q.RNE), lambda: G.quantize(x, q.MXFP4, q.RNE, rotate=True),
             lambda: G.quantize(x, q.NVFP4, q.RNE), lambda: G.quantize(x, q.NVFP4, q.SR, seed=3),
             lambda: G.quantize_mxfp8(x, q.RNE), lambda: G.quantize_mxfp8(x, q.SR, seed=3)]
    for f in calls:
        first = {k: host(v) for k, v in f().items()}
        for _ in range(3):
            again = f()
            for k, v in first.items():
                assert np.array_equal(host(again[k]).view(np.uint8), v.view(np.uint8)), k
