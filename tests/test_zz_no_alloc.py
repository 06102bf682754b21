"""The allocation-free GEMM entry point, qfp4_gemm_blockscaled_noalloc.

Some callers may not allocate device memory at all: an operator or plugin
hook that forbids allocation while it enqueues kernels, a real-time loop that
must not touch the allocator once running, a library handed only its inputs
and outputs.  For them the library offers this variant of the block-scaled
GEMM, which keeps its scratch (the rearranged scales) in an array built into
the library instead of asking for a workspace.

These checks call it through the C ABI and compare it with the workspace
entry point, qfp4_gemm_blockscaled, on two calls in a row (different shapes
and formats, so the second call reuses scratch the first one filled), within
the GEMM tolerance of the other GPU tests: |diff| <= 1e-5 * sum_k |a||b|.
The file name makes pytest collect it last; it builds all of its own inputs,
so it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import bit_fwht_hadamard_b200 as q
import synth

pytestmark = pytest.mark.gpu


def _operands(M, N, K, fmt, seed):
    a = torch.from_numpy(synth.cfg3_X(M, K, seed=seed).view(np.int16)).view(torch.bfloat16).cuda()
    b = torch.from_numpy(synth.cfg3_W(N, K, seed=seed + 1).view(np.int16)).view(torch.bfloat16).cuda()
    return q.quantize(a, fmt), q.quantize(b, fmt)


def _noalloc(A, B, M, N, K, fmt):
    out = torch.empty((M, N), dtype=torch.float32, device="cuda")
    st = q.qfp4_gemm_blockscaled_noalloc(
        A["codes"].data_ptr(), A["scales"].data_ptr(), A["tscale"].data_ptr() if "tscale" in A else None,
        B["codes"].data_ptr(), B["scales"].data_ptr(), B["tscale"].data_ptr() if "tscale" in B else None,
        M, N, K, fmt, q.F32, out.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == q.OK, q.status_string(st)
    return out


def _bound(A, B, M, N, K, fmt):
    """1e-5 * sum_k |a_k||b_k| from the library's own dequantized operands."""
    da = q.dequantize(A, M, K, fmt).double().abs()
    db = q.dequantize(B, N, K, fmt).double().abs()
    return 1e-5 * (da @ db.T)


def test_noalloc_gemm_matches_workspace_gemm_on_two_calls():
    cases = [(384, 512, 1024, q.NVFP4, 101), (256, 768, 2048, q.MXFP4, 202)]
    for M, N, K, fmt, seed in cases:
        A, B = _operands(M, N, K, fmt, seed)
        want = q.gemm(A, B, M, N, K, fmt).double()
        got = _noalloc(A, B, M, N, K, fmt).double()
        torch.cuda.synchronize()
        diff = (got - want).abs()
        assert bool((diff <= _bound(A, B, M, N, K, fmt)).all()), float(diff.max())
    assert q.qfp4_last_device_error() == 0


def test_noalloc_gemm_rejects_shapes_beyond_its_scratch():
    # (16384 x 4096 x 14336, NVFP4) needs more than the built-in 16 MiB for its
    # rearranged scales; the call refuses before touching any buffer
    assert q.qfp4_gemm_workspace_bytes(16384, 4096, 14336, q.NVFP4) > 16 << 20
    fake = 1 << 20
    st = q.qfp4_gemm_blockscaled_noalloc(fake, fake, fake, fake, fake, fake, 16384, 4096, 14336, q.NVFP4, q.F32,
                                         fake, None)
    assert st == q.ERR_SHAPE
