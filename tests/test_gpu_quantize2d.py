"""GPU parity of the 2D transposition-invariant NVFP4 quantize, the 1D
column-wise (X^T) quantize and the MXFP8 quantize, plus the Quartet-style
backward GEMMs on 2D-quantized operands -- all bit-exact against the oracle
(GEMMs within 1e-5 * sum|a||b|)."""
import numpy as np
import pytest
import torch

import bit_fwht_hadamard_b200 as q
import oracle
import synth
import gpu_util as GU
from gpu_util import (blocks_to_rows, blocks_to_tiles, encode_input, host, mismatch_report, nvfp4_boundary_blocks,
                      to_dev)

pytestmark = pytest.mark.gpu


def _cmp(got, ref, keys=("codes", "scales", "codesT", "scalesT", "tscale")):
    for k in keys:
        if k in ref:
            g = host(got[k]).reshape(np.asarray(ref[k]).shape).view(np.uint8)
            r = np.asarray(ref[k]).view(np.uint8)
            assert np.array_equal(g, r), mismatch_report(g, r, k)


# ------------------------------------------------------------------ 2D
@pytest.mark.parametrize("M,K", [(16, 16), (48, 64), (64, 48), (512, 1024), (1008, 528)])
@pytest.mark.parametrize("rounding", [q.RNE, q.SR], ids=["rne", "sr"])
@pytest.mark.parametrize("transposed", [False, True], ids=["x", "x+xT"])
def test_2d_matches_oracle(M, K, rounding, transposed):
    x = synth.cfg4_G(M, K, seed=M + K)
    got = GU.quantize(to_dev(x), q.NVFP4, rounding, block2d=True, seed=1004, transposed=transposed)
    ref = oracle.quantize(x, oracle.NVFP4, rounding, block2d=True, seed=1004, transposed=transposed)
    _cmp(got, ref)
    if transposed:                                   # X^T codes are exactly the transpose of X's
        c = host(got["codes"])
        cT = host(got["codesT"])
        n = np.empty((M, K), np.uint8)
        n[:, 0::2], n[:, 1::2] = c & 15, c >> 4
        nT = np.empty((K, M), np.uint8)
        nT[:, 0::2], nT[:, 1::2] = cT & 15, cT >> 4
        assert np.array_equal(nT, n.T)


def test_2d_float32_input():
    x = synth.bf16_bits_to_f32(synth.cfg4_G(64, 96, seed=5))
    for rounding in (q.RNE, q.SR):
        _cmp(GU.quantize(to_dev(x), q.NVFP4, rounding, block2d=True, seed=3, transposed=True),
             oracle.quantize(x, oracle.NVFP4, rounding, block2d=True, seed=3, transposed=True))


def test_2d_full_size_gradient_sr():
    """G bf16 8192 x 4096 ~ N(0, 1e-3^2) with 0.1% entries x100: 2D 16x16 NVFP4 + Philox SR (seed 1004),
    G and G^T operands from one pass."""
    g = synth.cfg4_G()
    got = GU.quantize(to_dev(g), q.NVFP4, q.SR, block2d=True, seed=1004, transposed=True)
    ref = oracle.quantize(g, oracle.NVFP4, oracle.SR, block2d=True, seed=1004, transposed=True)
    _cmp(got, ref)


@pytest.mark.parametrize("kind", ["bf16", "f32"])
def test_2d_rounding_boundaries(kind):
    """16 x 16 tiles whose quotients sit on (bf16) or next to (float32) the
    E2M1 midpoints and whose maxima put the scale on or next to E4M3
    midpoints: X and X^T codes and scales bit-exact."""
    x = encode_input(blocks_to_tiles(nvfp4_boundary_blocks(kind)), kind)
    for transposed in (False, True):
        got = GU.quantize(to_dev(x), q.NVFP4, q.RNE, block2d=True, transposed=transposed)
        ref = oracle.quantize(x, oracle.NVFP4, oracle.RNE, block2d=True, transposed=transposed)
        _cmp(got, ref)


# ------------------------------------------------------------------ 1D column-wise
@pytest.mark.parametrize("M,K", [(32, 32), (64, 96), (48, 64), (96, 80), (256, 512)])
@pytest.mark.parametrize("fmt", [(q.MXFP4, oracle.MXFP4), (q.NVFP4, oracle.NVFP4)], ids=["mxfp4", "nvfp4"])
@pytest.mark.parametrize("mode", ["rne", "sr", "four6"])
def test_1d_columnwise_matches_oracle(M, K, fmt, mode):
    g = 32 if fmt[0] == q.MXFP4 else 16
    if M % g or K % g or (mode == "four6" and fmt[0] == q.MXFP4):
        pytest.skip("shape / option not valid for this format")
    x = synth.cfg2_X(M, K, seed=M * 7 + K)
    rounding = q.SR if mode == "sr" else q.RNE
    got = GU.quantize(to_dev(x), fmt[0], rounding, four6=(mode == "four6"), seed=99, transposed=True)
    ref = oracle.quantize(x, fmt[1], rounding, four6=(mode == "four6"), seed=99, transposed=True)
    _cmp(got, ref)


@pytest.mark.parametrize("kind", ["bf16", "f32"])
@pytest.mark.parametrize("four6", [False, True], ids=["rne", "four6"])
def test_columnwise_rounding_boundaries(kind, four6):
    """The rounding-boundary blocks laid down the columns (groups along M)."""
    rows = blocks_to_rows(nvfp4_boundary_blocks(kind))            # (R, 128), blocks along K
    R = -(-rows.shape[0] // 16) * 16
    padded = np.zeros((R, rows.shape[1]))
    padded[:rows.shape[0]] = rows
    x = encode_input(np.ascontiguousarray(padded.T), kind)        # (128, R), blocks along M
    got = GU.quantize(to_dev(x), q.NVFP4, q.RNE, four6=four6, transposed=True)
    ref = oracle.quantize(x, oracle.NVFP4, oracle.RNE, four6=four6, transposed=True)
    _cmp(got, ref)


# ------------------------------------------------------------------ MXFP8
@pytest.mark.parametrize("M,K", [(1, 32), (37, 64), (64, 96), (256, 512)])
@pytest.mark.parametrize("rounding", [q.RNE, q.SR], ids=["rne", "sr"])
@pytest.mark.parametrize("transposed", [False, True], ids=["x", "x+xT"])
def test_mxfp8_matches_oracle(M, K, rounding, transposed):
    if transposed and M % 32:
        pytest.skip("column output needs M % 32 == 0")
    x = synth.cfg4_G(M, K, seed=M + 3 * K)
    got = GU.quantize_mxfp8(to_dev(x), rounding, seed=1004, transposed=transposed)
    ref = oracle.quantize_mxfp8(x, rounding, seed=1004, transposed=transposed)
    _cmp(got, ref)


def test_mxfp8_full_size_gradient():
    g = synth.cfg4_G()
    for rounding in (q.RNE, q.SR):
        got = GU.quantize_mxfp8(to_dev(g), rounding, seed=1004, transposed=True)
        ref = oracle.quantize_mxfp8(g, rounding, seed=1004, transposed=True)
        _cmp(got, ref)


# ------------------------------------------------------------------ backward GEMMs on 2D operands
def test_backward_gemms_on_2d_operands():
    """dX = G W (A = G, B = W^T) and dW = G^T X (A = G^T, B = X^T), all operands
    2D-quantized NVFP4 (G with SR, W and X with RNE); the GEMM reads the
    transposed operands straight from codesT / scalesT."""
    T, O, I = 512, 256, 384                      # tokens, out features, in features
    G = synth.cfg4_G(T, O, seed=41)
    W = synth.cfg4_W(O, I, seed=42)
    X = synth.cfg4_X(T, I, seed=43)
    qg = oracle.quantize(G, oracle.NVFP4, oracle.SR, block2d=True, seed=1004, transposed=True)
    qw = oracle.quantize(W, oracle.NVFP4, oracle.RNE, block2d=True, transposed=True)
    qx = oracle.quantize(X, oracle.NVFP4, oracle.RNE, block2d=True, transposed=True)
    dg = GU.quantize(to_dev(G), q.NVFP4, q.SR, block2d=True, seed=1004, transposed=True)
    dw = GU.quantize(to_dev(W), q.NVFP4, q.RNE, block2d=True, transposed=True)
    dx = GU.quantize(to_dev(X), q.NVFP4, q.RNE, block2d=True, transposed=True)
    for got, ref in ((dg, qg), (dw, qw), (dx, qx)):
        _cmp(got, ref)

    def op(d, t):
        return {"codes": d["codesT" if t else "codes"], "scales": d["scalesT" if t else "scales"],
                "tscale": d["tscale"]}

    def rop(d, t):
        return {"codes": d["codesT" if t else "codes"], "scales": d["scalesT" if t else "scales"],
                "tscale": d["tscale"]}

    for (A, B, rA, rB, M, N, K) in ((op(dg, False), op(dw, True), rop(qg, False), rop(qw, True), T, I, O),
                                    (op(dg, True), op(dx, True), rop(qg, True), rop(qx, True), O, I, T)):
        y = host(GU.gemm(A, B, M, N, K, q.NVFP4))
        r, c = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
        ref, mag = oracle.gemm_sampled(rA, rB, M, N, K, oracle.NVFP4, r.ravel(), c.ravel())
        err = np.abs(y[r.ravel(), c.ravel()] - ref)
        assert np.all(err <= 1e-5 * mag + 1e-30)
