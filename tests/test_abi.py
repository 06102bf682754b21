"""The C-ABI library loads and exports every entry point include/qfp4.h declares
(no compute calls: runs without a GPU)."""
import os
import re

import bit_fwht_hadamard_b200 as q

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "qfp4.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(qfp4_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_entry_point():
    from bit_fwht_hadamard_b200 import build
    build.build()
    L = q.lib()
    names = _declared()
    assert len(names) >= 11
    for n in names:
        assert hasattr(L, n), n
    assert sorted(q.EXPORTS) == names


def test_host_only_calls():
    assert q.qfp4_version() >= 100
    assert "unsupported" in q.status_string(q.ERR_UNSUPPORTED)
    assert q.qfp4_quantize_workspace_bytes(4096, 4096, q.NVFP4) >= 4 * 148
    assert q.qfp4_quantize_workspace_bytes(4096, 4096, q.MXFP4) == 0


def test_argument_errors_return_before_any_launch():
    # invalid shapes / combinations are rejected on the host (no device pointer is touched)
    fake = 1 << 20                      # never dereferenced: validation fails first
    st = q.qfp4_quantize(fake, q.BF16, 4, 48, q.MXFP4, q.RNE, 0, 0, 0, 0, fake, fake, None, None, None, None, 0, None)
    assert st == q.ERR_SHAPE
    st = q.qfp4_quantize(fake, q.BF16, 4, 64, q.MXFP4, q.RNE, 0, 0, 1, 0, fake, fake, None, None, None, None, 0, None)
    assert st == q.ERR_UNSUPPORTED
    st = q.qfp4_quantize(fake + 2, q.BF16, 4, 64, q.MXFP4, q.RNE, 0, 0, 0, 0, fake, fake, None, None, None, None, 0,
                         None)
    assert st == q.ERR_ALIGN
    st = q.qfp4_quantize(fake, q.BF16, 4, 64, q.NVFP4, q.RNE, 0, 0, 0, 0, fake, fake, None, None, fake, None, 0, None)
    assert st == q.ERR_ARG                                  # NVFP4 without workspace
    st = q.qfp4_gemm_blockscaled(fake, fake, None, fake, fake, None, 64, 64, 48, q.MXFP4, q.F32, fake, fake, 1 << 20,
                                 None)
    assert st == q.ERR_SHAPE
    st = q.qfp4_gemm_blockscaled(fake, fake, None, fake, fake, None, 64, 66, 64, q.MXFP4, q.F32, fake, fake, 1 << 20,
                                 None)
    assert st == q.ERR_SHAPE                                # N % 4
    st = q.qfp4_gemm_blockscaled(fake, fake, None, fake, fake, None, 64, 64, 64, q.MXFP4, q.F32, fake, fake, 16, None)
    assert st == q.ERR_ARG                                  # workspace too small
