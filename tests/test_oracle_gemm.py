"""Pins of the oracle's dequantize and block-scaled GEMM reference.

Dequantized values are checked against exact rational arithmetic from the
format definitions; the GEMM against numpy's binary64 matmul of the
dequantized operands, an integer closed form, and the rotation identity
y = xW^T = (xH)(WH)^T of the Quartet notes.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synth

GRID = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3), Fraction(4), Fraction(6)]


def _e4m3_exact(b):
    return Fraction(float(torch.tensor([b], dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)[0]))


def _nibble(codes, M, K, i, j):
    byte = int(codes.reshape(M, K // 2)[i, j // 2])
    return (byte >> (4 * (j & 1))) & 0xF


@pytest.mark.parametrize("fmt", [oracle.MXFP4, oracle.NVFP4])
def test_dequantize_is_exact(fmt):
    M, K = 6, 64
    x = synth.cfg3_X(M, K, seed=51)
    q = oracle.quantize(x, fmt)
    deq = oracle.dequantize(q["codes"], q["scales"], q.get("tscale"), M, K, fmt)
    g = 32 if fmt == oracle.MXFP4 else 16
    for i in range(M):
        for j in range(K):
            c = _nibble(q["codes"], M, K, i, j)
            v = GRID[c & 7] * (-1 if c & 8 else 1)
            sb = int(q["scales"][i, j // g])
            if fmt == oracle.MXFP4:
                want = v * Fraction(2) ** (sb - 127)
            else:
                want = v * _e4m3_exact(sb) * Fraction(float(q["tscale"][0]))
            assert Fraction(deq[i, j]) == want


def test_dequantize_mxfp8_is_exact():
    x = synth.cfg4_G(4, 64, seed=52)
    q = oracle.quantize_mxfp8(x)
    deq = oracle.dequantize_mxfp8(q["codes"], q["scales"], 4, 64)
    for i in range(4):
        for j in range(64):
            want = _e4m3_exact(int(q["codes"][i, j])) * Fraction(2) ** (int(q["scales"][i, j // 32]) - 127)
            assert Fraction(deq[i, j]) == want


@pytest.mark.parametrize("fmt", [oracle.MXFP4, oracle.NVFP4])
def test_gemm_matches_binary64_matmul_of_dequantized(fmt):
    M, N, K = 24, 40, 160
    a = synth.cfg3_X(M, K, seed=53)
    b = synth.cfg3_W(N, K, seed=54)
    A, B = oracle.quantize(a, fmt), oracle.quantize(b, fmt)
    dA = oracle.dequantize(A["codes"], A["scales"], A.get("tscale"), M, K, fmt)
    dB = oracle.dequantize(B["codes"], B["scales"], B.get("tscale"), N, K, fmt)
    ref = dA @ dB.T                                      # numpy binary64 matmul
    rows, cols = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
    y, mag = oracle.gemm_sampled(A, B, M, N, K, fmt, rows.ravel(), cols.ravel())
    y, mag = y.reshape(M, N), mag.reshape(M, N)
    assert np.all(np.abs(y - ref) <= 1e-12 * mag)
    assert np.allclose(mag, np.abs(dA) @ np.abs(dB).T, rtol=1e-12)


def test_gemm_integer_closed_form():
    # A codes cycle through the grid, scales 2^0 / 2^1; B codes constant 1.0, scale 2^-1:
    # every product is a small dyadic rational, the sum is exact.
    M, N, K = 3, 2, 64
    A = {"codes": np.zeros((M, K // 2), np.uint8), "scales": np.zeros((M, K // 32), np.uint8)}
    B = {"codes": np.zeros((N, K // 2), np.uint8), "scales": np.zeros((N, K // 32), np.uint8)}
    want = np.zeros((M, N))
    for i in range(M):
        for j in range(K):
            c = (i + j) % 16
            A["codes"][i, j // 2] |= c << (4 * (j & 1))
    A["scales"][:, 0], A["scales"][:, 1] = 127, 128
    for n in range(N):
        for j in range(K):
            B["codes"][n, j // 2] |= (2 if n == 0 else 10) << (4 * (j & 1))    # +1.0 / -1.0
    B["scales"][:] = 126
    for i in range(M):
        for n in range(N):
            s = Fraction(0)
            for j in range(K):
                c = (i + j) % 16
                av = GRID[c & 7] * (-1 if c & 8 else 1) * (1 if j < 32 else 2)
                s += av * (1 if n == 0 else -1) * Fraction(1, 2)
            want[i, n] = float(s)
    rows, cols = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
    y, _ = oracle.gemm_sampled(A, B, M, N, K, oracle.MXFP4, rows.ravel(), cols.ravel())
    assert (y.reshape(M, N) == want).all()


def test_gemm_rotation_identity():
    """Quartet notes: y = xW^T = (xH)(WH)^T for orthogonal symmetric H, so the
    quantized GEMM of the rotated operands approximates the unrotated product."""
    M, N, K = 32, 48, 256
    a = synth.cfg5_A(M, K, seed=55)
    b = synth.cfg5_B(N, K, seed=56)
    af, bf = synth.bf16_bits_to_f32(a).astype(np.float64), synth.bf16_bits_to_f32(b).astype(np.float64)
    exact = af @ bf.T
    rows, cols = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
    for fmt in (oracle.MXFP4, oracle.NVFP4):
        A = oracle.quantize(a, fmt, rotate=True)
        B = oracle.quantize(b, fmt, rotate=True)
        y, _ = oracle.gemm_sampled(A, B, M, N, K, fmt, rows.ravel(), cols.ravel())
        rel = np.linalg.norm(y.reshape(M, N) - exact) / np.linalg.norm(exact)
        assert rel < 0.2
        # rotating only one side breaks the identity
        B0 = oracle.quantize(b, fmt)
        y0, _ = oracle.gemm_sampled(A, B0, M, N, K, fmt, rows.ravel(), cols.ravel())
        assert np.linalg.norm(y0.reshape(M, N) - exact) / np.linalg.norm(exact) > 0.5
