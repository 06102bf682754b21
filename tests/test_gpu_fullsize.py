"""GPU parity at the full sizes of the synthetic workloads, against the
oracle (run row-parallel on the host cores, tests/oracle_par.py).

- 7B-class fused rotate + quantize + GEMM, (M, N, K) in {(16384, 4096, 4096),
  (16384, 14336, 4096), (16384, 4096, 14336)}: A bf16 with outlier channels
  quantized inside the call (FWHT-128, NVFP4, RNE), B pre-rotated and
  quantized by the oracle.  A's codes, scales and tensor scale left in the
  workspace must equal the oracle's bit for bit; >= 64k sampled outputs plus
  the full 128 x 128 corner tiles must lie within 1e-5 * sum_k |a||b| (+ the
  bf16 output rounding) of the binary64 reference.  K = 14336 is the longest
  accumulation the GEMM meets.
- Quartet-style backward at full size: G 8192 x 4096 (2D 16 x 16 NVFP4,
  Philox SR), W 4096 x 4096 and X 8192 x 4096 (2D NVFP4 RNE), every operand
  checked bit for bit, then dX = G W (8192 x 4096 x 4096) and
  dW = G^T X (4096 x 4096 x 8192) through the transposed operands.
- The MNIST-MLP-sized GEMM of the fc1 workload on its own data: X 64 x 784
  N(0,1) by W^T with W 256 x 784 N(0, 0.04^2) plus its 50x outlier, both
  fp32 and zero-padded to K = 800, in MXFP4 and NVFP4: every output checked.
"""
import numpy as np
import pytest
import torch

import bit_fwht_hadamard_b200 as q
import gpu_util as G
import oracle
import oracle_par
import synth
from gpu_util import host, mismatch_report, to_dev

pytestmark = pytest.mark.gpu
TOL = 1e-5


def _upload(ref: dict) -> dict:
    out = {"codes": torch.from_numpy(ref["codes"]).cuda(), "scales": torch.from_numpy(ref["scales"]).cuda()}
    if "tscale" in ref:
        out["tscale"] = torch.from_numpy(np.asarray(ref["tscale"], np.float32).reshape(1)).cuda()
    return out


def _same(got: np.ndarray, want: np.ndarray, name: str):
    got = np.asarray(got).reshape(want.shape)
    assert np.array_equal(got.view(np.uint8), np.asarray(want).view(np.uint8)), mismatch_report(
        got.view(np.uint8), np.asarray(want).view(np.uint8), name)


def _samples(M, N, n, seed):
    rng = np.random.default_rng(seed)
    r, c = rng.integers(0, M, n), rng.integers(0, N, n)
    cr, cc = np.meshgrid(np.arange(min(M, 128)), np.arange(min(N, 128)), indexing="ij")
    cr, cc = cr.ravel(), cc.ravel()
    return np.concatenate([r, cr, M - 1 - cr]), np.concatenate([c, cc, N - 1 - cc])


def _check_gemm(y: np.ndarray, A, B, M, N, K, fmt, rows, cols, bf16):
    ref, mag = oracle_par.gemm_sampled(A, B, M, N, K, fmt, rows, cols)
    got = y[rows, cols].astype(np.float64)
    bound = TOL * mag + (2.0 ** -8 * np.abs(ref) if bf16 else 0.0) + 1e-30
    bad = np.flatnonzero(np.abs(got - ref) > bound)
    assert bad.size == 0, (f"{bad.size} of {len(rows)} outside the bound; worst at {(rows[bad[0]], cols[bad[0]])}: "
                           f"got {got[bad[0]]} want {ref[bad[0]]} mag {mag[bad[0]]}")


CFG5 = [(16384, 4096, 4096), (16384, 14336, 4096), (16384, 4096, 14336)]


@pytest.mark.parametrize("M,N,K", CFG5, ids=["16384x4096x4096", "16384x14336x4096", "16384x4096x14336"])
def test_fused_rotate_quantize_gemm_7b_shapes(M, N, K):
    a = synth.cfg5_A(M, K)
    B = oracle_par.quantize(synth.cfg5_B(N, K), oracle.NVFP4, rotate=True)   # weights rotated offline
    A = oracle_par.quantize(a, oracle.NVFP4, rotate=True)
    wsb = q.qfp4_gemm_fused_rq_workspace_bytes(M, N, K, q.NVFP4)
    ws = G.guarded((wsb,), torch.uint8)
    out = G.guarded((M, N), torch.bfloat16)
    q.gemm_fused_rq(to_dev(a), _upload(B), N, fmt=q.NVFP4, rotate=True, out=out, workspace=ws)
    torch.cuda.synchronize()
    co, so, to = q.qfp4_gemm_fused_rq_workspace_layout(M, N, K, q.NVFP4)
    wsh = host(ws)
    _same(wsh[co:co + M * K // 2], A["codes"], "A codes in the workspace")
    _same(wsh[so:so + M * K // 16], A["scales"], "A scales in the workspace")
    _same(wsh[to:to + 4].view(np.float32), A["tscale"], "A tensor scale")
    y = synth.bf16_bits_to_f32(host(out))
    rows, cols = _samples(M, N, 65536, seed=M + N + K)
    _check_gemm(y, A, B, M, N, K, oracle.NVFP4, rows, cols, bf16=True)
    assert q.qfp4_last_device_error() == 0


def test_backward_full_size_on_2d_sr_operands():
    g, x, w = synth.cfg4_G(), synth.cfg4_X(), synth.cfg4_W()
    Gq = G.quantize(to_dev(g), q.NVFP4, q.SR, block2d=True, seed=1004, transposed=True)
    Wq = G.quantize(to_dev(w), q.NVFP4, q.RNE, block2d=True, transposed=True)
    Xq = G.quantize(to_dev(x), q.NVFP4, q.RNE, block2d=True, transposed=True)
    ref = {"G": oracle.quantize(g, oracle.NVFP4, oracle.SR, block2d=True, seed=1004, transposed=True),
           "W": oracle.quantize(w, oracle.NVFP4, oracle.RNE, block2d=True, transposed=True),
           "X": oracle.quantize(x, oracle.NVFP4, oracle.RNE, block2d=True, transposed=True)}
    for name, got in (("G", Gq), ("W", Wq), ("X", Xq)):
        for k in ("codes", "scales", "codesT", "scalesT", "tscale"):
            _same(host(got[k]), ref[name][k], f"{name} {k}")
    T = lambda o: {"codes": o["codesT"], "scales": o["scalesT"], "tscale": o["tscale"]}    # noqa: E731
    # dX = G W: A = G (8192 x 4096 along N_out), B = W^T (4096 x 4096 along N_out)
    dX = host(G.gemm(Gq, T(Wq), 8192, 4096, 4096, q.NVFP4))
    r, c = _samples(8192, 4096, 65536, seed=41)
    _check_gemm(dX, ref["G"], T(ref["W"]), 8192, 4096, 4096, oracle.NVFP4, r, c, bf16=False)
    # dW = G^T X: A = G^T (4096 x 8192 along M), B = X^T (4096 x 8192 along M)
    dW = host(G.gemm(T(Gq), T(Xq), 4096, 4096, 8192, q.NVFP4))
    r, c = _samples(4096, 4096, 65536, seed=42)
    _check_gemm(dW, T(ref["G"]), T(ref["X"]), 4096, 4096, 8192, oracle.NVFP4, r, c, bf16=False)
    assert q.qfp4_last_device_error() == 0


@pytest.mark.parametrize("fmt", [(q.MXFP4, oracle.MXFP4), (q.NVFP4, oracle.NVFP4)], ids=["mxfp4", "nvfp4"])
def test_fc1_gemm_on_its_own_data(fmt):
    W = np.zeros((256, 800), np.float32)
    W[:, :784] = synth.cfg1_W()
    W[17, 300] = 50 * np.abs(W).max()
    X = np.zeros((64, 800), np.float32)
    X[:, :784] = synth.cfg1_X()
    Wq, Xq = G.quantize(to_dev(W), fmt[0]), G.quantize(to_dev(X), fmt[0])
    Wr, Xr = oracle.quantize(W, fmt[1]), oracle.quantize(X, fmt[1])
    for got, want, name in ((Wq, Wr, "W"), (Xq, Xr, "X")):
        for k in want:
            _same(host(got[k]), want[k], f"{name} {k}")
    y = host(G.gemm(Xq, Wq, 64, 256, 800, fmt[0]))
    r, c = np.meshgrid(np.arange(64), np.arange(256), indexing="ij")
    _check_gemm(y, Xr, Wr, 64, 256, 800, fmt[1], r.ravel(), c.ravel(), bf16=False)
