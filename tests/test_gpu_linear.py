"""GPU parity of the MXFP8 block-scaled GEMM (tcgen05 kind::mxf8f6f4) and of
the Quartet-style linear layer (qfp4_linear_forward / qfp4_linear_backward)
against the oracle: operands bit for bit where the test can see them, GEMM
outputs within |err| <= 1e-5 * sum_k |a||b| (+ 2^-8 |y| for bf16 outputs) of
the binary64 reference over the oracle's own quantized operands."""
import numpy as np
import pytest
import torch

import bit_fwht_hadamard_b200 as q
import gpu_util as GU
import oracle
import oracle_par
import synth
from gpu_util import host, to_dev

pytestmark = pytest.mark.gpu
TOL = 1e-5


def _upload(ref: dict, keys=("codes", "scales")) -> dict:
    out = {k: torch.from_numpy(np.ascontiguousarray(ref[k])).cuda() for k in keys}
    if "tscale" in ref:
        out["tscale"] = torch.from_numpy(np.asarray(ref["tscale"], np.float32).reshape(1)).cuda()
    return out


def _T(o: dict) -> dict:
    t = {"codes": o["codesT"], "scales": o["scalesT"]}
    if "tscale" in o:
        t["tscale"] = o["tscale"]
    return t


def _pairs(M, N, n=60_000, seed=0):
    if M * N <= 300_000:
        r, c = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
        return r.ravel(), c.ravel()
    rng = np.random.default_rng(seed)
    cr, cc = np.meshgrid(np.arange(min(M, 128)), np.arange(min(N, 128)), indexing="ij")
    cr, cc = cr.ravel(), cc.ravel()
    return (np.concatenate([rng.integers(0, M, n), cr, M - 1 - cr]),
            np.concatenate([rng.integers(0, N, n), cc, N - 1 - cc]))


def _check(y, A, B, M, N, K, fmt, bf16=False, seed=0):
    if y.dtype == np.uint16:
        y = synth.bf16_bits_to_f32(y)
    rows, cols = _pairs(M, N, seed=seed)
    ref, mag = oracle_par.gemm_sampled(A, B, M, N, K, fmt, rows, cols)
    got = y[rows, cols].astype(np.float64)
    bound = TOL * mag + (2.0 ** -8 * np.abs(ref) if bf16 else 0.0) + 1e-30
    bad = np.flatnonzero(np.abs(got - ref) > bound)
    assert bad.size == 0, (f"{bad.size} of {len(rows)} outside the bound; worst at {(rows[bad[0]], cols[bad[0]])}: "
                           f"got {got[bad[0]]} want {ref[bad[0]]} mag {mag[bad[0]]}")


# ------------------------------------------------------------------ MXFP8 GEMM
SHAPES = [(128, 256, 256), (200, 264, 544), (37, 8, 64), (512, 1024, 1024), (300, 520, 2080), (64, 256, 800)]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_mxfp8_gemm_matches_oracle(M, N, K, out):
    A = oracle.quantize_mxfp8(synth.cfg4_G(M, K, seed=M + K))
    B = oracle.quantize_mxfp8(synth.cfg4_W(N, K, seed=N + 3 * K))
    od = torch.float32 if out == "f32" else torch.bfloat16
    y = host(GU.gemm(_upload(A), _upload(B), M, N, K, q.MXFP8, out_dtype=od))
    _check(y, A, B, M, N, K, oracle.MXFP8, bf16=out == "bf16")


def test_mxfp8_gemm_exact_on_representable_inputs():
    """E4M3 codes of small integers under E8M0 scales 2^0 / 2^1: every
    partial sum is an exact binary32 integer, so the result is exact."""
    M, N, K = 256, 256, 512
    rng = np.random.default_rng(13)
    ints = np.arange(-8, 9)
    enc = {int(v): int(torch.tensor([float(v)]).to(torch.float8_e4m3fn).view(torch.uint8)[0]) for v in ints}
    A = {"codes": np.vectorize(enc.get)(rng.choice(ints, (M, K))).astype(np.uint8),
         "scales": rng.integers(127, 129, (M, K // 32)).astype(np.uint8)}
    B = {"codes": np.vectorize(enc.get)(rng.choice(ints, (N, K))).astype(np.uint8),
         "scales": rng.integers(127, 129, (N, K // 32)).astype(np.uint8)}
    y = host(GU.gemm(_upload(A), _upload(B), M, N, K, q.MXFP8))
    r, c = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
    ref, _ = oracle.gemm_sampled(A, B, M, N, K, oracle.MXFP8, r.ravel(), c.ravel())
    assert np.array_equal(y.ravel().astype(np.float64), ref)


@pytest.mark.parametrize("out", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_mxfp8_gemm_bitwise_deterministic(out):
    M, N, K = 4096, 9216, 2048
    X = q.quantize_mxfp8(to_dev(synth.cfg4_G(M, K, seed=11)))
    W = q.quantize_mxfp8(to_dev(synth.cfg4_W(N, K, seed=12)))
    ys = [q.gemm(X, W, M, N, K, q.MXFP8, out_dtype=out) for _ in range(4)]
    torch.cuda.synchronize()
    ref = ys[0].view(torch.int32 if out == torch.float32 else torch.int16)
    for y in ys[1:]:
        assert int((y.view(ref.dtype) != ref).sum()) == 0
    assert q.qfp4_last_device_error() == 0


# ------------------------------------------------------------------ linear forward
@pytest.mark.parametrize("M,N,K", [(256, 512, 1024), (100, 264, 384), (8192, 11008, 4096)])
@pytest.mark.parametrize("mode", ["nvfp4", "nvfp4-four6", "mxfp4"])
def test_linear_forward_matches_oracle(M, N, K, mode):
    fmt = (q.MXFP4, oracle.MXFP4) if mode == "mxfp4" else (q.NVFP4, oracle.NVFP4)
    four6 = mode == "nvfp4-four6"
    x, w = synth.cfg3_X(M, K, seed=M + K), synth.cfg3_W(N, K, seed=N + K)
    y = GU.guarded((M, N), torch.bfloat16)
    q.linear_forward(to_dev(x), to_dev(w), fmt=fmt[0], four6=four6, out=y)
    A = oracle_par.quantize(x, fmt[1], rotate=True, four6=four6)
    B = oracle_par.quantize(w, fmt[1], rotate=True, four6=four6)
    _check(host(y), A, B, M, N, K, fmt[1], bf16=True, seed=M)
    assert q.qfp4_last_device_error() == 0


# ------------------------------------------------------------------ linear backward
def _backward_refs(g, x, w, fmt, seed):
    if fmt == q.NVFP4:
        G = oracle.quantize(g, oracle.NVFP4, oracle.SR, block2d=True, seed=seed, transposed=True)
        W = oracle.quantize(w, oracle.NVFP4, oracle.RNE, block2d=True, transposed=True)
        X = oracle.quantize(x, oracle.NVFP4, oracle.RNE, block2d=True, transposed=True)
        return G, W, X, oracle.NVFP4
    G = oracle.quantize_mxfp8(g, oracle.SR, seed=seed, transposed=True)
    W = oracle.quantize_mxfp8(w, oracle.RNE, transposed=True)
    X = oracle.quantize_mxfp8(x, oracle.RNE, transposed=True)
    return G, W, X, oracle.MXFP8


@pytest.mark.parametrize("M,N,K", [(256, 384, 512), (96, 64, 160), (8192, 4096, 4096)])
@pytest.mark.parametrize("fmt", [q.NVFP4, q.MXFP8], ids=["fp4-2d", "mxfp8"])
def test_linear_backward_matches_oracle(M, N, K, fmt):
    if fmt == q.MXFP8 and K % 32:
        pytest.skip()
    seed = 1004
    g, x, w = synth.cfg4_G(M, N), synth.cfg4_X(M, K), synth.cfg4_W(N, K)
    out = {"dX": GU.guarded((M, K), torch.float32), "dW": GU.guarded((N, K), torch.float32)}
    dX, dW = q.linear_backward(to_dev(g), to_dev(x), to_dev(w), fmt=fmt, seed=seed, out=out)
    G, W, X, of = _backward_refs(g, x, w, fmt, seed)
    _check(host(dX), G, _T(W), M, K, N, of, seed=1)          # dX = G W
    _check(host(dW), _T(G), _T(X), N, K, M, of, seed=2)      # dW = G^T X
    assert q.qfp4_last_device_error() == 0


def test_linear_backward_one_output_only():
    M, N, K = 128, 96, 64
    g, x, w = synth.cfg4_G(M, N, seed=3), synth.cfg4_X(M, K, seed=4), synth.cfg4_W(N, K, seed=5)
    dX, dW = q.linear_backward(to_dev(g), None, to_dev(w), fmt=q.MXFP8, seed=9, want_dw=False)
    assert dW is None
    G, W, _, of = _backward_refs(g, x, w, q.MXFP8, 9)
    _check(host(dX), G, _T(W), M, K, N, of)
    dX, dW = q.linear_backward(to_dev(g), to_dev(x), None, fmt=q.NVFP4, seed=9, want_dx=False)
    G, _, X, of = _backward_refs(g, x, w, q.NVFP4, 9)
    _check(host(dW), _T(G), _T(X), N, K, M, of)
