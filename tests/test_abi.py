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
    st = q.qfp4_quantize(fake, q.BF16, 4, 64, q.MXFP4, q.SR, 0, 0, 1, 0, fake, fake, None, None, None, None, 0, None)
    assert st == q.ERR_UNSUPPORTED                          # four-over-six is round-to-nearest only
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


def test_more_argument_errors_follow_the_header():
    """The remaining documented rejections, all decided on the host."""
    f = 1 << 20
    Q = q.qfp4_quantize
    # four-over-six only with NVFP4, 1D, round-to-nearest
    assert Q(f, q.BF16, 16, 64, q.NVFP4, q.SR, 0, 0, 1, 0, f, f, None, None, f, f, 4096, None) == q.ERR_UNSUPPORTED
    assert Q(f, q.BF16, 16, 64, q.NVFP4, q.RNE, 0, 1, 1, 0, f, f, None, None, f, f, 4096, None) == q.ERR_UNSUPPORTED
    # 2D blocks without rotation; MXFP4 tiles are 32 x 32
    assert Q(f, q.BF16, 16, 128, q.MXFP4, q.RNE, 0, 1, 0, 0, f, f, None, None, None, None, 0, None) == q.ERR_SHAPE
    assert Q(f, q.BF16, 32, 128, q.MXFP4, q.RNE, 1, 1, 0, 0, f, f, None, None, None, None, 0, None) == q.ERR_UNSUPPORTED
    assert Q(f, q.BF16, 16, 128, q.NVFP4, q.RNE, 1, 1, 0, 0, f, f, None, None, f, f, 4096, None) == q.ERR_UNSUPPORTED
    # 1D column-wise output not with rotation; codesT and scalesT together
    assert Q(f, q.BF16, 32, 128, q.MXFP4, q.RNE, 1, 0, 0, 0, f, f, f, f, None, None, 0, None) == q.ERR_UNSUPPORTED
    assert Q(f, q.BF16, 32, 128, q.MXFP4, q.RNE, 0, 0, 0, 0, f, f, f, None, None, None, 0, None) == q.ERR_ARG
    # shapes: rotation needs K % 128, 2D needs M % 16, 1D columns need M % g
    assert Q(f, q.BF16, 16, 96, q.MXFP4, q.RNE, 1, 0, 0, 0, f, f, None, None, None, None, 0, None) == q.ERR_SHAPE
    assert Q(f, q.BF16, 24, 64, q.NVFP4, q.RNE, 0, 1, 0, 0, f, f, f, f, f, f, 4096, None) == q.ERR_SHAPE
    assert Q(f, q.BF16, 48, 64, q.MXFP4, q.RNE, 0, 0, 0, 0, f, f, f, f, None, None, 0, None) == q.ERR_SHAPE
    # enum values
    assert Q(f, q.BF16, 16, 64, 7, q.RNE, 0, 0, 0, 0, f, f, None, None, None, None, 0, None) == q.ERR_ARG
    assert Q(f, 9, 16, 64, q.MXFP4, q.RNE, 0, 0, 0, 0, f, f, None, None, None, None, 0, None) == q.ERR_ARG
    # MXFP8: K % 32; column output needs M % 32
    M8 = q.qfp4_quantize_mxfp8
    assert M8(f, q.BF16, 32, 48, q.RNE, 0, f, f, None, None, None) == q.ERR_SHAPE
    assert M8(f, q.BF16, 48, 64, q.RNE, 0, f, f, f, f, None) == q.ERR_SHAPE
    assert M8(f, q.BF16, 32, 64, 5, 0, f, f, None, None, None) == q.ERR_ARG
    # dequantize: K % g, NVFP4 needs the tensor scale, output type
    D = q.qfp4_dequantize
    assert D(f, f, None, 4, 48, q.MXFP4, q.F32, f, None) == q.ERR_SHAPE
    assert D(f, f, None, 4, 64, q.NVFP4, q.F32, f, None) == q.ERR_ARG
    assert D(f, f, None, 4, 64, q.MXFP4, 3, f, None) == q.ERR_ARG
    assert D(f + 4, f, None, 4, 64, q.MXFP4, q.F32, f, None) == q.ERR_ALIGN


def test_selftest_wait_limit_is_checked_on_the_host():
    assert q.qfp4_selftest_wait_timeout(0, None) == q.ERR_ARG
    assert q.qfp4_selftest_wait_timeout(1_000_001, None) == q.ERR_ARG


def test_quantize_ex_argument_errors():
    """qfp4_quantize_ex's own rejections, decided on the host."""
    f = 1 << 20
    X = q.qfp4_quantize_ex

    def call(fmt, rule=q.SCALE_DEFAULT, rounding=q.RNE, four6=0, block2d=0, amax_in=None, amax_out=None,
             M=32, K=128, T=False, ws=None, wsb=0):
        return X(f, q.BF16, M, K, fmt, rounding, 0, block2d, four6, rule, 0, amax_in, amax_out, f, f,
                 f if T else None, f if T else None, f, ws, wsb, None)

    assert call(q.MXFP4, rule=3) == q.ERR_ARG
    assert call(q.NVFP4, rule=q.SCALE_OCP_FLOOR, ws=f, wsb=4096) == q.ERR_UNSUPPORTED
    assert call(q.MXFP4, rule=q.SCALE_E4M3_UP) == q.ERR_UNSUPPORTED
    assert call(q.MXFP4, amax_in=f) == q.ERR_UNSUPPORTED
    assert call(q.MXFP4, amax_out=f) == q.ERR_UNSUPPORTED
    assert call(q.MXFP4, four6=1, T=True) == q.ERR_UNSUPPORTED          # MXFP4 four-over-six: rows only
    assert call(q.NVFP4, amax_out=f) == q.ERR_ARG                        # own amax needs the workspace
    assert call(q.MXFP4, block2d=1, M=48) == q.ERR_SHAPE


def test_kl_calibrate_argument_errors():
    f = 1 << 20
    C = q.qfp4_kl_calibrate
    assert C(f, q.BF16, 64, 4, 2, 0, f, None, None, None, f, 1 << 20, None) == q.ERR_ARG        # bins < 8
    assert C(f, q.BF16, 64, 9000, 8, 0, f, None, None, None, f, 1 << 20, None) == q.ERR_ARG     # bins > 8192
    assert C(f, q.BF16, 64, 64, 65, 0, f, None, None, None, f, 1 << 20, None) == q.ERR_ARG      # levels > bins
    assert C(f, q.BF16, 64, 64, 8, 2, f, None, None, None, f, 1 << 20, None) == q.ERR_ARG       # grid
    assert C(f, q.BF16, 64, 64, 8, 0, None, None, None, None, f, 1 << 20, None) == q.ERR_ARG    # no clip output
    assert C(f, q.BF16, 64, 64, 8, 0, f, None, None, None, f, 16, None) == q.ERR_ARG            # short workspace
    assert q.qfp4_kl_calibrate_workspace_bytes(2048, 8, 0) > 2048 * 8


def test_linear_argument_errors_return_before_any_launch():
    """Every case below is refused by the host checks before a CUDA call (the
    pointers are never dereferenced); empty shapes, which may issue memsets,
    are left out."""
    f = 1 << 20
    big = 1 << 40
    Fw = q.qfp4_linear_forward
    ok_ws = q.qfp4_linear_forward_workspace_bytes(256, 512, 1024, q.NVFP4)
    assert ok_ws > 0 and q.qfp4_linear_forward_workspace_bytes(256, 512, 1024, 7) == 0
    assert Fw(f, f, 256, 512, 1024, 7, 0, q.BF16, f, f, big, None) == q.ERR_ARG                 # format
    assert Fw(f, f, 256, 512, 1024, q.NVFP4, 0, 9, f, f, big, None) == q.ERR_ARG                # output type
    assert Fw(f, f, 256, 512, 1024, q.MXFP4, 1, q.BF16, f, f, big, None) == q.ERR_UNSUPPORTED   # four6 on MXFP4
    assert Fw(f, f, -1, 512, 1024, q.NVFP4, 0, q.BF16, f, f, big, None) == q.ERR_SHAPE
    assert Fw(f, f, 256, 512, 1000, q.NVFP4, 0, q.BF16, f, f, big, None) == q.ERR_SHAPE         # K % 128
    assert Fw(f, f, 256, 12, 1024, q.NVFP4, 0, q.BF16, f, f, big, None) == q.ERR_SHAPE          # N % 8, bf16 out
    assert Fw(f, f, 256, 512, 1024, q.NVFP4, 0, q.BF16, None, f, big, None) == q.ERR_ARG        # no output
    assert Fw(f + 4, f, 256, 512, 1024, q.NVFP4, 0, q.BF16, f, f, big, None) == q.ERR_ALIGN
    assert Fw(f, f, 256, 512, 1024, q.NVFP4, 0, q.BF16, f, f, ok_ws - 1, None) == q.ERR_ARG     # short workspace
    Bw = q.qfp4_linear_backward
    bws = q.qfp4_linear_backward_workspace_bytes(256, 384, 512, q.NVFP4)
    assert bws > 0 and q.qfp4_linear_backward_workspace_bytes(256, 384, 512, q.MXFP4) == 0
    assert Bw(f, f, f, 256, 384, 512, q.MXFP4, 1, q.F32, f, f, f, big, None) == q.ERR_ARG       # format
    assert Bw(f, f, f, 250, 384, 512, q.NVFP4, 1, q.F32, f, f, f, big, None) == q.ERR_SHAPE     # M % 32
    assert Bw(f, f, f, 256, 384, 520, q.NVFP4, 1, q.F32, f, f, f, big, None) == q.ERR_SHAPE     # K % 16
    assert Bw(f, f, f, 256, 384, 528, q.MXFP8, 1, q.F32, f, f, f, big, None) == q.ERR_SHAPE     # K % 32
    assert Bw(f, f, f, 256, 384, 512, q.NVFP4, 1, q.F32, None, None, f, big, None) == q.ERR_ARG  # no output
    assert Bw(f, f, None, 256, 384, 512, q.NVFP4, 1, q.F32, f, None, f, big, None) == q.ERR_ARG  # dX without W
    assert Bw(f, None, f, 256, 384, 512, q.NVFP4, 1, q.F32, None, f, f, big, None) == q.ERR_ARG  # dW without X
    assert Bw(f, f, f, 256, 384, 512, q.NVFP4, 1, q.F32, f, f + 8, f, big, None) == q.ERR_ALIGN
    assert Bw(f, f, f, 256, 384, 512, q.NVFP4, 1, q.F32, f, f, f, bws - 1, None) == q.ERR_ARG    # short workspace


def test_size_limits_are_shape_errors():
    """Operands above 2^38 elements (or with M * K past int64) are refused as
    shape errors before any launch, as are GEMM dimensions of 2^30 or more."""
    f = 1 << 20
    for M, K in ((1 << 20, 1 << 19), (1 << 40, 1 << 40), (1 << 62, 1 << 6)):
        assert q.qfp4_quantize(f, q.BF16, M, K, q.MXFP4, q.RNE, 0, 0, 0, 0, f, f, None, None, None, None, 0,
                               None) == q.ERR_SHAPE
        assert q.qfp4_quantize_mxfp8(f, q.BF16, M, K, q.RNE, 0, f, f, None, None, None) == q.ERR_SHAPE
        assert q.qfp4_quantize_fp32scale(f, q.BF16, M, K, q.GRAN_ROW, f, f, None, 0, None) == q.ERR_SHAPE
        assert q.qfp4_dequantize(f, f, f, M, K, q.MXFP4, q.F32, f, None) == q.ERR_SHAPE
    ws = q.qfp4_kl_calibrate_workspace_bytes(2048, 8, 0)
    assert ws > 0
    assert q.qfp4_kl_calibrate(f, q.BF16, (1 << 38) + 32, 2048, 8, 0, f, None, None, None, f, ws, None) == q.ERR_SHAPE
    big = 1 << 30
    assert q.qfp4_gemm_blockscaled(f, f, None, f, f, None, big, 256, 256, q.MXFP4, q.F32, f, f, 1 << 40,
                                   None) == q.ERR_SHAPE
    assert q.qfp4_status_string(q.ERR_SHAPE) == "shape violates the call's divisibility or size rules"


def test_header_is_plain_c_and_a_c_program_links_and_runs(tmp_path):
    """include/qfp4.h compiles as strict C99 (warnings are errors), a C
    program links against libqfp4.so taking the address of every declared
    entry point, and its host-only calls and a validation error run."""
    import subprocess
    from bit_fwht_hadamard_b200 import build
    build.build()
    names = _declared()
    refs = ",\n    ".join(f"(void (*)(void)){n}" for n in names)
    src = f"""#include <stdio.h>
#include <string.h>
#include "qfp4.h"
static void (*const entry_points[])(void) = {{
    {refs}
}};
int main(void)
{{
    size_t i;
    for (i = 0; i < sizeof entry_points / sizeof entry_points[0]; ++i)
        if (!entry_points[i]) return 10;
    if (qfp4_version() < 100) return 11;
    if (strcmp(qfp4_status_string(QFP4_OK), "ok") != 0) return 12;
    if (qfp4_quantize((const void *)0, QFP4_BF16, 4, 64, (qfp4_fmt)7, QFP4_RNE, 0, 0, 0, 0,
                      (unsigned char *)0, (unsigned char *)0, (unsigned char *)0, (unsigned char *)0,
                      (float *)0, (void *)0, 0, (qfp4_stream_t)0) != QFP4_ERR_ARG) return 13;
    printf("%u entry points\\n", (unsigned)(sizeof entry_points / sizeof entry_points[0]));
    return 0;
}}
"""
    c = tmp_path / "abi_check.c"
    c.write_text(src)
    exe = tmp_path / "abi_check"
    libdir = os.path.join(ROOT, "bit_fwht_hadamard_b200")
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                         "-I", os.path.join(ROOT, "include"), str(c), "-o", str(exe),
                         "-L", libdir, "-l:libqfp4.so", f"-Wl,-rpath,{libdir}"],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, (run.returncode, run.stderr)
    assert run.stdout.strip() == f"{len(names)} entry points"


def test_python_wrappers_refuse_inputs_the_c_abi_cannot_read():
    """The torch-level wrappers pass plain pointers, so they refuse a host
    tensor, a non-contiguous view or a wrong rank before any call."""
    import pytest
    import torch
    x = torch.zeros((64, 64), dtype=torch.bfloat16)
    cases = [
        (lambda: q.quantize(x, q.MXFP4), "CUDA"),
        (lambda: q.quantize_mxfp8(x), "CUDA"),
        (lambda: q.quantize_fp32scale(x, q.GRAN_ROW), "CUDA"),
        (lambda: q.gemm_fused_rq(x, {}, 64), "CUDA"),
        (lambda: q.linear_forward(x, x), "CUDA"),
        (lambda: q.linear_backward(x, None, x), "CUDA"),
        (lambda: q.kl_calibrate(x), "CUDA"),
    ]
    for call, what in cases:
        with pytest.raises(ValueError, match=what):
            call()
    with pytest.raises(ValueError, match="contiguous"):
        q._input(_FakeCuda(False, 2), "x")
    with pytest.raises(ValueError, match="dimensions"):
        q._input(_FakeCuda(True, 3), "x")
    q._input(_FakeCuda(True, 2), "x")
    q._input(_FakeCuda(True, 1), "x", dims=None)


class _FakeCuda:
    """Stands in for a CUDA tensor's attributes (no GPU here)."""
    is_cuda = True

    def __new__(cls, contiguous=True, dims=2):
        o = object.__new__(cls)
        o._c, o._d = contiguous, dims
        return o

    def is_contiguous(self):
        return self._c

    def dim(self):
        return self._d


def test_a_missing_library_fails_loudly(monkeypatch, tmp_path):
    """No CPU fallback: without the built library every call path raises."""
    import pytest
    monkeypatch.setattr(q, "_lib", None)
    monkeypatch.setattr(q, "LIB_PATH", str(tmp_path / "libqfp4.so"))
    with pytest.raises(ImportError, match="not built"):
        q.lib()
    with pytest.raises(ImportError):
        q.qfp4_version()


def test_product_path_never_touches_the_oracle():
    """The package and its native sources neither import, load nor name the
    oracle library; importing the package and loading libqfp4 leaves the
    oracle unloaded; the library does not link it."""
    import subprocess
    import sys
    pkg = os.path.join(ROOT, "bit_fwht_hadamard_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, re.M), f
                assert "liboracle" not in text and "qfp4_oracle" not in text, f
    code = ("import sys; import bit_fwht_hadamard_b200 as q; q.lib(); "
            "print('oracle' in sys.modules, any('liboracle' in l for l in open('/proc/self/maps')))")
    out = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    assert out.stdout.split() == ["False", "False"]
    ldd = subprocess.run(["ldd", os.path.join(pkg, "libqfp4.so")], capture_output=True, text=True)
    assert "oracle" not in ldd.stdout


def test_oracle_shares_no_code_with_the_product():
    """The oracle and the input generators include no product header and
    import nothing from the product package."""
    for d in ("oracle", "synth"):
        for f in os.listdir(os.path.join(ROOT, d)):
            if f.endswith((".py", ".c", ".h")):
                text = open(os.path.join(ROOT, d, f), encoding="utf-8").read()
                assert '#include "qfp4.h"' not in text and "csrc/" not in text, f
                assert not re.search(r"^\s*(import|from)\s+bit_fwht_hadamard_b200\b", text, re.M), f
