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
from gpu_util import host, mismatch_report, to_dev

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
    got = q.quantize(to_dev(x), fmt[0], rounding, rotate=rotate, seed=0xDEADBEEF12345)
    ref = oracle.quantize(x, fmt[1], rounding, rotate=rotate, seed=0xDEADBEEF12345)
    _cmp(got, ref)


@pytest.mark.parametrize("M,K", [(1, 16), (37, 384), (600, 512), (5, 48)])
@pytest.mark.parametrize("rotate", [False, True], ids=["plain", "rot"])
def test_four_over_six_matches_oracle(M, K, rotate):
    if rotate and K % 128:
        pytest.skip()
    x = synth.cfg3_X(M, K, seed=M + K)
    got = q.quantize(to_dev(x), q.NVFP4, q.RNE, rotate=rotate, four6=True)
    ref = oracle.quantize(x, oracle.NVFP4, oracle.RNE, rotate=rotate, four6=True)
    _cmp(got, ref)


@pytest.mark.parametrize("fmt", FMTS, ids=["mxfp4", "nvfp4"])
@pytest.mark.parametrize("rounding", [q.RNE, q.SR], ids=["rne", "sr"])
def test_float32_input(fmt, rounding):
    W = np.zeros((256, 800), np.float32)
    W[:, :784] = synth.cfg1_W()
    W[17, 300] = 50 * np.abs(W).max()
    got = q.quantize(to_dev(W), fmt[0], rounding, seed=3)
    ref = oracle.quantize(W, fmt[1], rounding, seed=3)
    _cmp(got, ref)


def test_full_size_activation_quantize_rne_and_sr():
    """X bf16 4096 x 4096 with 40 x20 channels, FWHT-128 + MXFP4, RNE and SR seed 7."""
    x = synth.cfg2_X()
    xd = to_dev(x)
    for rounding, seed in ((q.RNE, 0), (q.SR, 7)):
        got = q.quantize(xd, q.MXFP4, rounding, rotate=True, seed=seed)
        ref = oracle.quantize(x, oracle.MXFP4, rounding, rotate=True, seed=seed)
        _cmp(got, ref)


def test_full_size_nvfp4_four6_forward_operands():
    """X 8192 x 4096 Student-t(3)*0.5 and W 11008 x 4096 N(0, 0.02^2), NVFP4 + four-over-six."""
    for x in (synth.cfg3_X(), synth.cfg3_W()):
        got = q.quantize(to_dev(x), q.NVFP4, q.RNE, four6=True)
        ref = oracle.quantize(x, oracle.NVFP4, oracle.RNE, four6=True)
        _cmp(got, ref)


def test_degenerate_inputs():
    z = np.zeros((64, 256), np.uint16)
    for fmt in FMTS:
        got = q.quantize(to_dev(z), fmt[0], q.RNE)
        _cmp(got, oracle.quantize(z, fmt[1], oracle.RNE))
    z[3, 5] = 0x8000                                   # a negative zero
    x = synth.cfg2_X(64, 256, seed=9)
    x[10, :64] = 0                                     # an all-zero group inside a nonzero tensor
    x[11, :64] = 0x8000
    x[12, 0] = 0x0001                                  # a bf16 subnormal
    for fmt in FMTS:
        for rounding in (q.RNE, q.SR):
            for arr in (z, x):
                _cmp(q.quantize(to_dev(arr), fmt[0], rounding, seed=1),
                     oracle.quantize(arr, fmt[1], rounding, seed=1))
    # M = 0 is a no-op that succeeds
    e = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    q.quantize(e, q.MXFP4)


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
    got = q.quantize(to_dev(X), q.MXFP4, rounding, seed=77)
    ref = oracle.quantize(X, oracle.MXFP4, rounding, seed=77)
    assert (ref["scales"] == 127).all()
    _cmp(got, ref)


def test_large_dynamic_range():
    rng = np.random.default_rng(5)
    z = rng.standard_normal(64 * 512) * np.exp(rng.uniform(-60, 60, 64 * 512))
    x = synth.to_bf16(z, (64, 512))
    for fmt in FMTS:
        for rounding in (q.RNE, q.SR):
            _cmp(q.quantize(to_dev(x), fmt[0], rounding, seed=2), oracle.quantize(x, fmt[1], rounding, seed=2))


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
    gq = q.quantize(to_dev(x), fmt[0])
    got = host(q.dequantize(gq, M, K, fmt[0], out))
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
    got = q.quantize_fp32scale(to_dev(W), gran)
    ref = oracle.quantize_fp32scale(W, gran)
    assert np.array_equal(host(got["codes"]), ref["codes"])
    assert np.array_equal(host(got["scales"]).view(np.uint32), ref["scales"].view(np.uint32))
