"""The allocation-free GEMM entry point, qfp4_gemm_blockscaled_noalloc.

Some callers may not allocate device memory at all: an operator or plugin
hook that forbids allocation while it enqueues kernels, a real-time loop that
must not touch the allocator once running, a library handed only its inputs
and outputs.  For them the library offers this variant of the block-scaled
GEMM, which keeps its scratch (the rearranged scales) in an array built into
the library instead of asking for a workspace.

These checks call it through the C ABI and compare it with the workspace
entry point, qfp4_gemm_blockscaled, on two calls in a row (different shapes
and formats, so the second call reuses scratch the first one filled).  Both
run the same kernels in the same order, so the outputs must agree bit for
bit; a scratch-reuse bug that only perturbed values would show.  A third
case fills the 16 MiB exactly.  The file name makes pytest collect it last;
it builds all of its own inputs, so it also passes alone in a fresh process.
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


def _same_bits(got, want):
    diff = int((got.view(torch.int32) != want.view(torch.int32)).sum())
    assert diff == 0, f"{diff} of {want.numel()} outputs differ from the workspace GEMM"


def test_noalloc_gemm_matches_workspace_gemm_on_two_calls():
    cases = [(384, 512, 1024, q.NVFP4, 101), (256, 768, 2048, q.MXFP4, 202)]
    for M, N, K, fmt, seed in cases:
        A, B = _operands(M, N, K, fmt, seed)
        want = q.gemm(A, B, M, N, K, fmt)
        got = _noalloc(A, B, M, N, K, fmt)
        torch.cuda.synchronize()
        _same_bits(got, want)
    assert q.qfp4_last_device_error() == 0


def test_noalloc_gemm_with_scales_filling_the_scratch_exactly():
    # 4096 x 4096 x 32768 NVFP4: (32 A blocks + 2 x 16 B blocks) x 128 k-tiles x
    # 4 chunks x 512 B = 16 MiB, the largest shape class the scratch admits
    M, N, K = 4096, 4096, 32768
    assert q.qfp4_gemm_workspace_bytes(M, N, K, q.NVFP4) == 16 << 20
    A, B = _operands(M, N, K, q.NVFP4, 303)
    want = q.gemm(A, B, M, N, K, q.NVFP4)
    got = _noalloc(A, B, M, N, K, q.NVFP4)
    torch.cuda.synchronize()
    _same_bits(got, want)
    assert q.qfp4_last_device_error() == 0


def test_noalloc_gemm_rejects_shapes_beyond_its_scratch():
    # one more 128-row block of A than the exact fit above, and the
    # 16384 x 4096 x 14336 NVFP4 shape: both need more than the built-in
    # 16 MiB for their rearranged scales; the call refuses before touching
    # any buffer
    fake = 1 << 20
    for M, N, K in ((4097, 4096, 32768), (16384, 4096, 14336)):
        assert q.qfp4_gemm_workspace_bytes(M, N, K, q.NVFP4) > 16 << 20
        st = q.qfp4_gemm_blockscaled_noalloc(fake, fake, fake, fake, fake, fake, M, N, K, q.NVFP4, q.F32, fake,
                                             None)
        assert st == q.ERR_SHAPE
    # argument errors come first, as in the workspace entry point
    st = q.qfp4_gemm_blockscaled_noalloc(fake, fake, fake, fake, fake, fake, 1 << 40, 4096, 4096, 7, q.F32, fake,
                                         None)
    assert st == q.ERR_ARG
