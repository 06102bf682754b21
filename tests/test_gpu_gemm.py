"""GPU parity of the block-scaled FP4 GEMM (tcgen05) and the fused
rotate + quantize + GEMM path against the oracle's binary64 reference.

Operands are quantized by the oracle on the CPU and uploaded, so these tests
check the GEMM alone.  Bar: |y_gpu - y_ref| <= 1e-5 * sum_k |a_k||b_k| per
element (plus the bf16 output rounding, 2^-8 |y_ref|, for bf16 outputs).
"""
import numpy as np
import pytest
import torch

import bit_fwht_hadamard_b200 as q
import oracle
import synth
import gpu_util as G
from gpu_util import host, to_dev

pytestmark = pytest.mark.gpu

FMTS = [(q.MXFP4, oracle.MXFP4), (q.NVFP4, oracle.NVFP4)]
TOL = 1e-5


def _upload(ref: dict) -> dict:
    out = {"codes": torch.from_numpy(ref["codes"]).cuda(), "scales": torch.from_numpy(ref["scales"]).cuda()}
    if "tscale" in ref:
        out["tscale"] = torch.from_numpy(np.asarray(ref["tscale"], np.float32).reshape(1)).cuda()
    return out


def _check(y, A, B, M, N, K, fmt, rows, cols, bf16=False):
    ref, mag = oracle.gemm_sampled(A, B, M, N, K, fmt, rows, cols)
    got = y[rows, cols].astype(np.float64)
    bound = TOL * mag + (2.0 ** -8 * np.abs(ref) if bf16 else 0.0) + 1e-30
    err = np.abs(got - ref)
    bad = np.argwhere(err > bound).ravel()
    assert bad.size == 0, (f"{bad.size} of {len(rows)} outside the bound; worst at "
                           f"{(rows[bad[0]], cols[bad[0]])}: got {got[bad[0]]} want {ref[bad[0]]} mag {mag[bad[0]]}")


def _all_pairs(M, N):
    r, c = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
    return r.ravel(), c.ravel()


def _sample_pairs(M, N, n, seed=0):
    rng = np.random.default_rng(seed)
    r = rng.integers(0, M, n)
    c = rng.integers(0, N, n)
    # plus complete 128 x 128 corner tiles
    cr, cc = _all_pairs(min(M, 128), min(N, 128))
    r2, c2 = M - 1 - cr, N - 1 - cc
    return np.concatenate([r, cr, r2]), np.concatenate([c, cc, c2])


# several tiles, ragged M / N edges, a K tail short of the 256 tile, tiny M
SHAPES = [(128, 256, 256), (200, 264, 512), (64, 256, 800), (512, 1024, 1024), (37, 8, 64), (300, 520, 2048)]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("fmt", FMTS, ids=["mxfp4", "nvfp4"])
@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_gemm_matches_oracle(M, N, K, fmt, out):
    a = synth.cfg3_X(M, K, seed=M + 3 * K)
    b = synth.cfg3_W(N, K, seed=N + 5 * K)
    A, B = oracle.quantize(a, fmt[1]), oracle.quantize(b, fmt[1])
    od = torch.float32 if out == "f32" else torch.bfloat16
    y = G.gemm(_upload(A), _upload(B), M, N, K, fmt[0], out_dtype=od)
    yh = host(y)
    if out == "bf16":
        yh = synth.bf16_bits_to_f32(yh)
    rows, cols = _all_pairs(M, N) if M * N <= 300_000 else _sample_pairs(M, N, 50_000)
    _check(yh, A, B, M, N, K, fmt[1], rows, cols, bf16=(out == "bf16"))


@pytest.mark.parametrize("fmt", FMTS, ids=["mxfp4", "nvfp4"])
def test_gemm_exact_on_representable_inputs(fmt):
    """Small-integer codes and unit-ish scales: every partial sum is exact in
    binary32, so the tensor-core result must equal the reference exactly."""
    M, N, K = 256, 256, 512
    rng = np.random.default_rng(11)
    g = 32 if fmt[1] == oracle.MXFP4 else 16
    A = {"codes": rng.integers(0, 256, (M, K // 2), dtype=np.uint8),
         "scales": np.full((M, K // g), 127 if g == 32 else 0x38, np.uint8)}   # 2^0 / E4M3 1.0
    B = {"codes": rng.integers(0, 256, (N, K // 2), dtype=np.uint8),
         "scales": np.full((N, K // g), 127 if g == 32 else 0x38, np.uint8)}
    A["scales"][::3] += 1                                                     # 2.0 / 1.125
    if fmt[1] == oracle.NVFP4:
        A["tscale"] = np.array([1.0], np.float32)
        B["tscale"] = np.array([1.0], np.float32)
    y = host(G.gemm(_upload(A), _upload(B), M, N, K, fmt[0]))
    rows, cols = _all_pairs(M, N)
    ref, _ = oracle.gemm_sampled(A, B, M, N, K, fmt[1], rows, cols)
    assert np.array_equal(y[rows, cols].astype(np.float64), ref)


def test_gemm_full_size_forward_linear():
    """X 8192 x 4096 (Student-t(3)*0.5), W 11008 x 4096 (N(0, 0.02^2)), NVFP4 +
    four-over-six on both, Y = X W^T in binary32; sampled outputs plus full
    128 x 128 corner tiles."""
    M, N, K = 8192, 11008, 4096
    x, w = synth.cfg3_X(), synth.cfg3_W()
    X = G.quantize(to_dev(x), q.NVFP4, four6=True)
    W = G.quantize(to_dev(w), q.NVFP4, four6=True)
    y = host(G.gemm(X, W, M, N, K, q.NVFP4))
    A = {k: host(v) for k, v in X.items()}
    B = {k: host(v) for k, v in W.items()}
    rows, cols = _sample_pairs(M, N, 20_000, seed=3)
    _check(y, A, B, M, N, K, oracle.NVFP4, rows, cols)


@pytest.mark.parametrize("fmt", FMTS, ids=["mxfp4", "nvfp4"])
@pytest.mark.parametrize("out", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_gemm_bitwise_deterministic(fmt, out):
    """Every output element is accumulated in one fixed order (k-tiles in
    sequence, one CTA pair per tile), so repeated calls must agree bit for
    bit.  Several tiles per CTA pair, so the accumulator hand-off between
    tiles and the wrap-around of every stage, scale-slot and scale-buffer ring
    are exercised; a hand-off race would show up as differing elements."""
    M, N, K = 4096, 9216, 2048          # 16 x 36 = 576 tiles of 256 x 256 on 74 pairs, 8 k-tiles each
    X = G.quantize(to_dev(synth.cfg3_X(M, K, seed=11)), fmt[0])
    W = G.quantize(to_dev(synth.cfg3_W(N, K, seed=12)), fmt[0])
    ys = [G.gemm(X, W, M, N, K, fmt[0], out_dtype=out) for _ in range(4)]
    torch.cuda.synchronize()
    ref = ys[0].view(torch.int32 if out == torch.float32 else torch.int16)
    for y in ys[1:]:
        diff = int((y.view(ref.dtype) != ref).sum())
        assert diff == 0, f"{diff} elements differ between calls"
    assert q.qfp4_last_device_error() == 0


@pytest.mark.parametrize("fmt", FMTS, ids=["mxfp4", "nvfp4"])
@pytest.mark.parametrize("four6", [False, True])
def test_fused_rotate_quantize_gemm(fmt, four6):
    if four6 and fmt[1] == oracle.MXFP4:
        pytest.skip("four-over-six is an NVFP4 option")
    M, N, K = 384, 512, 1024
    a = synth.cfg5_A(M, K, seed=21)
    b = synth.cfg5_B(N, K, seed=22)
    B = oracle.quantize(b, fmt[1], rotate=True)                  # weights rotated offline
    y = host(G.gemm_fused_rq(to_dev(a), _upload(B), N, fmt=fmt[0], rotate=True, four6=four6))
    A = oracle.quantize(a, fmt[1], rotate=True, four6=four6)
    rows, cols = _all_pairs(M, N)
    _check(y, A, B, M, N, K, fmt[1], rows, cols)


def test_gemm_argument_errors():
    A = {"codes": torch.zeros((128, 128), dtype=torch.uint8, device="cuda"),
         "scales": torch.zeros((128, 8), dtype=torch.uint8, device="cuda")}
    with pytest.raises(q.QFP4Error) as e:
        G.gemm(A, A, 128, 130, 256, q.MXFP4)                      # N % 4
    assert e.value.status == q.ERR_SHAPE
    assert q.qfp4_last_device_error() == 0


# fused-call shapes on the CTA-pair kernel: ragged M, a K tail short of the
# 256-element k-tile, several 128-row blocks of A
FUSED_SHAPES = [(300, 264, 640), (256, 512, 1024), (1000, 768, 384), (129, 256, 2048)]


@pytest.mark.parametrize("M,N,K", FUSED_SHAPES)
@pytest.mark.parametrize("fmt", FMTS, ids=["mxfp4", "nvfp4"])
@pytest.mark.parametrize("rotate", [True, False], ids=["rot", "plain"])
def test_fused_call_shapes(M, N, K, fmt, rotate):
    """A's codes, scales and tensor scale left in the workspace equal the
    oracle's bit for bit, and every output is within the bound of the
    binary64 reference."""
    if rotate and K % 128:
        pytest.skip()
    a = synth.cfg5_A(M, K, seed=M + 7 * K)
    b = synth.cfg5_B(N, K, seed=N + 5 * K)
    B = oracle.quantize(b, fmt[1], rotate=rotate)
    A = oracle.quantize(a, fmt[1], rotate=rotate)
    wsb = q.qfp4_gemm_fused_rq_workspace_bytes(M, N, K, fmt[0])
    ws = G.guarded((wsb,), torch.uint8)
    y = G.guarded((M, N), torch.float32)
    q.gemm_fused_rq(to_dev(a), _upload(B), N, fmt=fmt[0], rotate=rotate, out=y, workspace=ws)
    co, so, to = q.qfp4_gemm_fused_rq_workspace_layout(M, N, K, fmt[0])
    g = 32 if fmt[1] == oracle.MXFP4 else 16
    w = host(ws)
    assert np.array_equal(w[co:co + M * K // 2], A["codes"].ravel())
    assert np.array_equal(w[so:so + M * K // g], A["scales"].ravel())
    if fmt[1] == oracle.NVFP4:
        assert w[to:to + 4].view(np.float32)[0] == A["tscale"][0]
    rows, cols = _all_pairs(M, N)
    _check(host(y), A, B, M, N, K, fmt[1], rows, cols)
    assert q.qfp4_last_device_error() == 0


def test_fused_call_is_repeatable():
    """Kernels of the call overlap through dependent launches differently from
    call to call; the output must not depend on it."""
    M, N, K = 2048, 4096, 4096
    a = to_dev(synth.cfg5_A(M, K, seed=3))
    B = q.quantize(to_dev(synth.cfg5_B(N, K, seed=4)), q.NVFP4, rotate=True)
    ys = [q.gemm_fused_rq(a, B, N, fmt=q.NVFP4, rotate=True, out_dtype=torch.bfloat16) for _ in range(4)]
    torch.cuda.synchronize()
    for y in ys[1:]:
        assert int((y.view(torch.int16) != ys[0].view(torch.int16)).sum()) == 0
    assert q.qfp4_last_device_error() == 0


@pytest.mark.parametrize("M,N,K", [(300, 264, 640), (1000, 768, 384), (100, 256, 512)])
@pytest.mark.parametrize("scale", [1.0, 0.5])
def test_fused_with_given_and_reported_amax(M, N, K, scale):
    """NVFP4 fused call under a supplied tensor amax of A (the own amax, or a
    stale one x0.5 that saturates the top blocks): A's operand and the
    outputs follow the oracle under the same amax, and the amax the call
    reports is A's own (rotated) amax bit for bit (M = 100 runs on the
    single-CTA GEMM kernel)."""
    a = synth.cfg5_A(M, K, seed=M + K)
    B = oracle.quantize(synth.cfg5_B(N, K, seed=N), oracle.NVFP4, rotate=True)
    own = oracle.tensor_amax(a, rotate=True)
    amax = float(np.float32(own * scale))
    A = oracle.quantize_ex(a, oracle.NVFP4, rotate=True, amax_in=amax)
    got_amax = G.guarded((1,), torch.float32)
    wsb = q.qfp4_gemm_fused_rq_workspace_bytes(M, N, K, q.NVFP4)
    ws = G.guarded((wsb,), torch.uint8)
    y = G.guarded((M, N), torch.float32)
    q.gemm_fused_rq(to_dev(a), _upload(B), N, fmt=q.NVFP4, rotate=True, out=y, workspace=ws,
                    A_amax_in=torch.tensor([amax], dtype=torch.float32, device="cuda"), A_amax_out=got_amax)
    co, so, to = q.qfp4_gemm_fused_rq_workspace_layout(M, N, K, q.NVFP4)
    w = host(ws)
    assert np.array_equal(w[co:co + M * K // 2], A["codes"].ravel())
    assert np.array_equal(w[so:so + M * K // 16], A["scales"].ravel())
    assert w[to:to + 4].view(np.float32)[0] == A["tscale"][0]
    assert host(got_amax)[0] == np.float32(own)
    rows, cols = _all_pairs(M, N)
    _check(host(y), A, B, M, N, K, oracle.NVFP4, rows, cols)
