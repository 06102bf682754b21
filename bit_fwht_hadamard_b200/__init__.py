"""libqfp4: B200-native FP4 microscaling quantization and block-scaled FP4 GEMM.

Thin Python binding over the C ABI in ``include/qfp4.h``.  Every step of the
method runs in the CUDA kernels of ``libqfp4.so``; this module only marshals
arguments (torch tensors for device memory, CUDA streams) and allocates the
output tensors.  There is no CPU fallback: if the library is missing the
import of the functions below raises.

The ``qfp4_*`` functions mirror the C entry points one to one (pointers as
integers); ``quantize``, ``quantize_mxfp8``, ``dequantize``, ``gemm`` and
``gemm_fused_rq`` are conveniences that allocate outputs.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import c_int, c_int64, c_size_t, c_uint64, c_void_p, c_char_p

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqfp4.so")

MXFP4, NVFP4, MXFP8 = 0, 1, 2
RNE, SR = 0, 1
BF16, F32 = 0, 1
GRAN_TENSOR, GRAN_ROW, GRAN_GROUP16, GRAN_GROUP32 = 0, 1, 2, 3
SCALE_DEFAULT, SCALE_OCP_FLOOR, SCALE_E4M3_UP = 0, 1, 2
OK, ERR_ARG, ERR_SHAPE, ERR_UNSUPPORTED, ERR_ALIGN, ERR_CUDA, ERR_TIMEOUT = 0, -1, -2, -3, -4, -5, -6
DEV_ERR_TIMEOUT = 1

EXPORTS = [
    "qfp4_quantize_workspace_bytes", "qfp4_quantize", "qfp4_quantize_ex", "qfp4_quantize_mxfp8", "qfp4_quantize_fp32scale",
    "qfp4_dequantize", "qfp4_gemm_workspace_bytes", "qfp4_gemm_blockscaled", "qfp4_gemm_fused_rq_workspace_bytes",
    "qfp4_gemm_fused_rq", "qfp4_gemm_fused_rq_ex", "qfp4_gemm_fused_rq_workspace_layout", "qfp4_gemm_blockscaled_noalloc",
    "qfp4_linear_forward_workspace_bytes", "qfp4_linear_forward", "qfp4_linear_backward_workspace_bytes",
    "qfp4_linear_backward", "qfp4_kl_calibrate_workspace_bytes", "qfp4_kl_calibrate",
    "qfp4_status_string", "qfp4_last_device_error", "qfp4_selftest_wait_timeout", "qfp4_version",
    "qfp4_launch_count",
]

_lib = None


class QFP4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: status {status} ({status_string(status)})")
        self.status = status


def lib():
    """Load libqfp4.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libqfp4.so not built at {LIB_PATH}; run __graft_entry__.build() or "
                              f"python -m bit_fwht_hadamard_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        P = c_void_p
        L.qfp4_quantize_workspace_bytes.restype = c_size_t
        L.qfp4_quantize_workspace_bytes.argtypes = [c_int64, c_int64, c_int, c_int, c_int]
        L.qfp4_quantize.restype = c_int
        L.qfp4_quantize.argtypes = [P, c_int, c_int64, c_int64, c_int, c_int, c_int, c_int, c_int, c_uint64,
                                    P, P, P, P, P, P, c_size_t, P]
        L.qfp4_quantize_ex.restype = c_int
        L.qfp4_quantize_ex.argtypes = [P, c_int, c_int64, c_int64, c_int, c_int, c_int, c_int, c_int, c_int,
                                       c_uint64, P, P, P, P, P, P, P, P, c_size_t, P]
        L.qfp4_quantize_mxfp8.restype = c_int
        L.qfp4_quantize_mxfp8.argtypes = [P, c_int, c_int64, c_int64, c_int, c_uint64, P, P, P, P, P]
        L.qfp4_quantize_fp32scale.restype = c_int
        L.qfp4_quantize_fp32scale.argtypes = [P, c_int, c_int64, c_int64, c_int, P, P, P, c_size_t, P]
        L.qfp4_dequantize.restype = c_int
        L.qfp4_dequantize.argtypes = [P, P, P, c_int64, c_int64, c_int, c_int, P, P]
        L.qfp4_gemm_workspace_bytes.restype = c_size_t
        L.qfp4_gemm_workspace_bytes.argtypes = [c_int64, c_int64, c_int64, c_int]
        L.qfp4_gemm_blockscaled.restype = c_int
        L.qfp4_gemm_blockscaled.argtypes = [P, P, P, P, P, P, c_int64, c_int64, c_int64, c_int, c_int, P, P,
                                            c_size_t, P]
        L.qfp4_gemm_blockscaled_noalloc.restype = c_int
        L.qfp4_gemm_blockscaled_noalloc.argtypes = [P, P, P, P, P, P, c_int64, c_int64, c_int64, c_int, c_int, P, P]
        L.qfp4_gemm_fused_rq_workspace_bytes.restype = c_size_t
        L.qfp4_gemm_fused_rq_workspace_bytes.argtypes = [c_int64, c_int64, c_int64, c_int]
        L.qfp4_gemm_fused_rq.restype = c_int
        L.qfp4_gemm_fused_rq.argtypes = [P, c_int64, c_int64, c_int, c_int, c_int, P, P, P, c_int64, P, c_size_t,
                                         c_int, P, P]
        L.qfp4_gemm_fused_rq_ex.restype = c_int
        L.qfp4_gemm_fused_rq_ex.argtypes = [P, c_int64, c_int64, c_int, c_int, c_int, P, P, P, P, P, c_int64, P,
                                            c_size_t, c_int, P, P]
        L.qfp4_gemm_fused_rq_workspace_layout.restype = c_int
        L.qfp4_gemm_fused_rq_workspace_layout.argtypes = [c_int64, c_int64, c_int64, c_int, P, P, P]
        L.qfp4_linear_forward_workspace_bytes.restype = c_size_t
        L.qfp4_linear_forward_workspace_bytes.argtypes = [c_int64, c_int64, c_int64, c_int]
        L.qfp4_linear_forward.restype = c_int
        L.qfp4_linear_forward.argtypes = [P, P, c_int64, c_int64, c_int64, c_int, c_int, c_int, P, P, c_size_t, P]
        L.qfp4_linear_backward_workspace_bytes.restype = c_size_t
        L.qfp4_linear_backward_workspace_bytes.argtypes = [c_int64, c_int64, c_int64, c_int]
        L.qfp4_linear_backward.restype = c_int
        L.qfp4_linear_backward.argtypes = [P, P, P, c_int64, c_int64, c_int64, c_int, c_uint64, c_int, P, P, P,
                                           c_size_t, P]
        L.qfp4_kl_calibrate_workspace_bytes.restype = c_size_t
        L.qfp4_kl_calibrate_workspace_bytes.argtypes = [c_int, c_int, c_int]
        L.qfp4_kl_calibrate.restype = c_int
        L.qfp4_kl_calibrate.argtypes = [P, c_int, c_int64, c_int, c_int, c_int, P, P, P, P, P, c_size_t, P]
        L.qfp4_status_string.restype = c_char_p
        L.qfp4_status_string.argtypes = [c_int]
        L.qfp4_last_device_error.restype = c_int
        L.qfp4_last_device_error.argtypes = []
        L.qfp4_selftest_wait_timeout.restype = c_int
        L.qfp4_selftest_wait_timeout.argtypes = [c_int64, P]
        L.qfp4_version.restype = c_int
        L.qfp4_version.argtypes = []
        L.qfp4_launch_count.restype = c_uint64
        L.qfp4_launch_count.argtypes = []
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().qfp4_status_string(status).decode()


# ------------------------------------------------------------------ raw C entry points
def qfp4_quantize_workspace_bytes(M, K, fmt, rotate=0, block2d=0):
    return lib().qfp4_quantize_workspace_bytes(M, K, fmt, int(rotate), int(block2d))


def qfp4_quantize(x, xdt, M, K, fmt, rounding, rotate, block2d, four6, seed, codes, scales, codesT, scalesT,
                  tscale, workspace, workspace_bytes, stream):
    return lib().qfp4_quantize(x, xdt, M, K, fmt, rounding, rotate, block2d, four6, seed & ((1 << 64) - 1), codes,
                               scales, codesT, scalesT, tscale, workspace, workspace_bytes, stream)


def qfp4_quantize_ex(x, xdt, M, K, fmt, rounding, rotate, block2d, four6, rule, seed, amax_in, amax_out, codes,
                     scales, codesT, scalesT, tscale, workspace, workspace_bytes, stream):
    return lib().qfp4_quantize_ex(x, xdt, M, K, fmt, rounding, rotate, block2d, four6, rule, seed & ((1 << 64) - 1),
                                  amax_in, amax_out, codes, scales, codesT, scalesT, tscale, workspace,
                                  workspace_bytes, stream)


def qfp4_quantize_mxfp8(x, xdt, M, K, rounding, seed, codes, scales, codesT, scalesT, stream):
    return lib().qfp4_quantize_mxfp8(x, xdt, M, K, rounding, seed & ((1 << 64) - 1), codes, scales, codesT,
                                     scalesT, stream)


def qfp4_quantize_fp32scale(x, xdt, M, K, gran, codes, scales, workspace, workspace_bytes, stream):
    return lib().qfp4_quantize_fp32scale(x, xdt, M, K, gran, codes, scales, workspace, workspace_bytes, stream)


def qfp4_dequantize(codes, scales, tscale, M, K, fmt, out_dt, out, stream):
    return lib().qfp4_dequantize(codes, scales, tscale, M, K, fmt, out_dt, out, stream)


def qfp4_gemm_workspace_bytes(M, N, K, fmt):
    return lib().qfp4_gemm_workspace_bytes(M, N, K, fmt)


def qfp4_gemm_blockscaled(A_codes, A_scales, A_tscale, B_codes, B_scales, B_tscale, M, N, K, fmt, out_dt, out,
                          workspace, workspace_bytes, stream):
    return lib().qfp4_gemm_blockscaled(A_codes, A_scales, A_tscale, B_codes, B_scales, B_tscale, M, N, K, fmt,
                                       out_dt, out, workspace, workspace_bytes, stream)


def qfp4_gemm_blockscaled_noalloc(A_codes, A_scales, A_tscale, B_codes, B_scales, B_tscale, M, N, K, fmt, out_dt,
                                  out, stream):
    """The GEMM without a workspace argument (built-in 16 MiB scratch), for
    callers that may not allocate device memory."""
    return lib().qfp4_gemm_blockscaled_noalloc(A_codes, A_scales, A_tscale, B_codes, B_scales, B_tscale, M, N, K,
                                               fmt, out_dt, out, stream)


def qfp4_gemm_fused_rq_workspace_bytes(M, N, K, fmt):
    return lib().qfp4_gemm_fused_rq_workspace_bytes(M, N, K, fmt)


def qfp4_gemm_fused_rq(A_bf16, M, K, rotate, four6, fmt, B_codes, B_scales, B_tscale, N, workspace,
                       workspace_bytes, out_dt, out, stream):
    return lib().qfp4_gemm_fused_rq(A_bf16, M, K, rotate, four6, fmt, B_codes, B_scales, B_tscale, N, workspace,
                                    workspace_bytes, out_dt, out, stream)


def qfp4_gemm_fused_rq_ex(A_bf16, M, K, rotate, four6, fmt, A_amax_in, A_amax_out, B_codes, B_scales, B_tscale, N,
                          workspace, workspace_bytes, out_dt, out, stream):
    return lib().qfp4_gemm_fused_rq_ex(A_bf16, M, K, rotate, four6, fmt, A_amax_in, A_amax_out, B_codes, B_scales,
                                       B_tscale, N, workspace, workspace_bytes, out_dt, out, stream)


def qfp4_gemm_fused_rq_workspace_layout(M, N, K, fmt):
    """(codes, scales, tscale) byte offsets of A's quantized operand in the
    fused call's workspace."""
    offs = [ctypes.c_size_t() for _ in range(3)]
    st = lib().qfp4_gemm_fused_rq_workspace_layout(M, N, K, fmt, *[ctypes.byref(o) for o in offs])
    _check(st, "qfp4_gemm_fused_rq_workspace_layout")
    return tuple(o.value for o in offs)


def qfp4_linear_forward_workspace_bytes(M, N, K, fmt):
    return lib().qfp4_linear_forward_workspace_bytes(M, N, K, fmt)


def qfp4_linear_forward(X, W, M, N, K, fmt, four6, out_dt, Y, workspace, workspace_bytes, stream):
    return lib().qfp4_linear_forward(X, W, M, N, K, fmt, four6, out_dt, Y, workspace, workspace_bytes, stream)


def qfp4_linear_backward_workspace_bytes(M, N, K, fmt):
    return lib().qfp4_linear_backward_workspace_bytes(M, N, K, fmt)


def qfp4_linear_backward(G, X, W, M, N, K, fmt, seed, out_dt, dX, dW, workspace, workspace_bytes, stream):
    return lib().qfp4_linear_backward(G, X, W, M, N, K, fmt, seed & ((1 << 64) - 1), out_dt, dX, dW, workspace,
                                      workspace_bytes, stream)


def qfp4_kl_calibrate_workspace_bytes(bins, levels, grid):
    return lib().qfp4_kl_calibrate_workspace_bytes(bins, levels, grid)


def qfp4_kl_calibrate(x, xdt, n, bins, levels, grid, clip_out, best_bins_out, kl_out, hist_out, workspace,
                      workspace_bytes, stream):
    return lib().qfp4_kl_calibrate(x, xdt, n, bins, levels, grid, clip_out, best_bins_out, kl_out, hist_out,
                                   workspace, workspace_bytes, stream)


def qfp4_status_string(status):
    return status_string(status)


def qfp4_last_device_error():
    return lib().qfp4_last_device_error()


def qfp4_selftest_wait_timeout(limit_us, stream):
    return lib().qfp4_selftest_wait_timeout(limit_us, stream)


def qfp4_version():
    return lib().qfp4_version()


def qfp4_launch_count():
    return lib().qfp4_launch_count()


# ------------------------------------------------------------------ torch conveniences
def _torch():
    import torch
    return torch


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream=None):
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _xdt(x):
    torch = _torch()
    if x.dtype == torch.bfloat16:
        return BF16
    if x.dtype == torch.float32:
        return F32
    raise TypeError("x must be bfloat16 or float32")


def _check(st, where):
    if st != OK:
        raise QFP4Error(st, where)


def _input(t, name, dims=2):
    """An input tensor the C ABI can read as a plain pointer: on a CUDA
    device, contiguous (row-major), with `dims` dimensions (None: any)."""
    if not getattr(t, "is_cuda", False):
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (row-major)")
    if dims is not None and t.dim() != dims:
        raise ValueError(f"{name} must have {dims} dimensions, not {t.dim()}")


def quantize(x, fmt=MXFP4, rounding=RNE, rotate=False, block2d=False, four6=False, seed=0, transposed=False,
             stream=None, out=None, workspace=None, rule=SCALE_DEFAULT, amax_in=None, amax_out=None):
    """Quantize a contiguous (M, K) bf16/fp32 CUDA tensor; returns a dict of
    uint8 codes (M, K/2), scales (M, K/g), optional codesT/scalesT, and the
    float32 tscale (NVFP4).  ``out`` may supply preallocated buffers.
    ``rule``, ``amax_in`` / ``amax_out`` (one-element float32 CUDA tensors)
    are qfp4_quantize_ex's scale rule and tensor-amax options."""
    torch = _torch()
    _input(x, "x")
    M, K = x.shape
    g = 32 if fmt == MXFP4 else 16
    dev = x.device
    o = dict(out) if out is not None else {}
    if "codes" not in o:
        o["codes"] = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
        o["scales"] = torch.empty((M, K // g), dtype=torch.uint8, device=dev)
        if transposed:
            o["codesT"] = torch.empty((K, M // 2), dtype=torch.uint8, device=dev)
            o["scalesT"] = torch.empty((K, M // g), dtype=torch.uint8, device=dev)
        if fmt == NVFP4:
            o["tscale"] = torch.empty(1, dtype=torch.float32, device=dev)
    wsb = qfp4_quantize_workspace_bytes(M, K, fmt, rotate, block2d)
    if workspace is None and wsb:
        workspace = torch.empty(wsb, dtype=torch.uint8, device=dev)
    st = qfp4_quantize_ex(_ptr(x), _xdt(x), M, K, fmt, rounding, int(rotate), int(block2d), int(four6), rule, seed,
                          _ptr(amax_in), _ptr(amax_out), _ptr(o["codes"]), _ptr(o["scales"]), _ptr(o.get("codesT")),
                          _ptr(o.get("scalesT")), _ptr(o.get("tscale")), _ptr(workspace), wsb, _stream(stream))
    _check(st, "qfp4_quantize_ex")
    return o


def quantize_mxfp8(x, rounding=RNE, seed=0, transposed=False, stream=None, out=None):
    torch = _torch()
    _input(x, "x")
    M, K = x.shape
    dev = x.device
    o = dict(out) if out is not None else {}
    if "codes" not in o:
        o["codes"] = torch.empty((M, K), dtype=torch.uint8, device=dev)
        o["scales"] = torch.empty((M, K // 32), dtype=torch.uint8, device=dev)
        if transposed:
            o["codesT"] = torch.empty((K, M), dtype=torch.uint8, device=dev)
            o["scalesT"] = torch.empty((K, M // 32), dtype=torch.uint8, device=dev)
    st = qfp4_quantize_mxfp8(_ptr(x), _xdt(x), M, K, rounding, seed, _ptr(o["codes"]), _ptr(o["scales"]),
                             _ptr(o.get("codesT")), _ptr(o.get("scalesT")), _stream(stream))
    _check(st, "qfp4_quantize_mxfp8")
    return o


def quantize_fp32scale(x, gran, stream=None, out=None):
    torch = _torch()
    _input(x, "x")
    M, K = x.shape
    dev = x.device
    n_scales = {GRAN_TENSOR: 1, GRAN_ROW: M, GRAN_GROUP16: M * K // 16, GRAN_GROUP32: M * K // 32}[gran]
    o = dict(out) if out is not None else {
        "codes": torch.empty((M, K // 2), dtype=torch.uint8, device=dev),
        "scales": torch.empty(n_scales, dtype=torch.float32, device=dev)}
    wsb = qfp4_quantize_workspace_bytes(M, K, NVFP4)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    st = qfp4_quantize_fp32scale(_ptr(x), _xdt(x), M, K, gran, _ptr(o["codes"]), _ptr(o["scales"]), _ptr(ws), wsb,
                                 _stream(stream))
    _check(st, "qfp4_quantize_fp32scale")
    return o


def dequantize(q, M, K, fmt, out_dtype=None, stream=None, out=None):
    torch = _torch()
    if out is None:
        out_dtype = torch.float32 if out_dtype is None else out_dtype
        out = torch.empty((M, K), dtype=out_dtype, device=q["codes"].device)
    out_dtype = out.dtype
    st = qfp4_dequantize(_ptr(q["codes"]), _ptr(q["scales"]), _ptr(q.get("tscale")), M, K, fmt,
                         F32 if out_dtype == torch.float32 else BF16, _ptr(out), _stream(stream))
    _check(st, "qfp4_dequantize")
    return out


def gemm(A, B, M, N, K, fmt, out_dtype=None, out=None, workspace=None, stream=None):
    """Y = deq(A) deq(B)^T for operands as returned by ``quantize``."""
    torch = _torch()
    out_dtype = torch.float32 if out_dtype is None else out_dtype
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=A["codes"].device)
    wsb = qfp4_gemm_workspace_bytes(M, N, K, fmt)
    if workspace is None:
        workspace = torch.empty(max(wsb, 16), dtype=torch.uint8, device=A["codes"].device)
    st = qfp4_gemm_blockscaled(_ptr(A["codes"]), _ptr(A["scales"]), _ptr(A.get("tscale")), _ptr(B["codes"]),
                               _ptr(B["scales"]), _ptr(B.get("tscale")), M, N, K, fmt,
                               F32 if out.dtype == torch.float32 else BF16, _ptr(out), _ptr(workspace), wsb,
                               _stream(stream))
    _check(st, "qfp4_gemm_blockscaled")
    return out


def gemm_fused_rq(A_bf16, B, N, fmt=NVFP4, rotate=True, four6=False, out_dtype=None, out=None, workspace=None,
                  stream=None, A_amax_in=None, A_amax_out=None):
    """Y = Q(rot(A)) deq(B)^T with A bf16 (M, K) quantized inside the call;
    A_amax_in / A_amax_out: NVFP4 tensor amax of A supplied / reported
    (one-element float32 CUDA tensors)."""
    torch = _torch()
    _input(A_bf16, "A_bf16")
    M, K = A_bf16.shape
    out_dtype = torch.float32 if out_dtype is None else out_dtype
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=A_bf16.device)
    wsb = qfp4_gemm_fused_rq_workspace_bytes(M, N, K, fmt)
    if workspace is None:
        workspace = torch.empty(max(wsb, 16), dtype=torch.uint8, device=A_bf16.device)
    st = qfp4_gemm_fused_rq_ex(_ptr(A_bf16), M, K, int(rotate), int(four6), fmt, _ptr(A_amax_in), _ptr(A_amax_out),
                               _ptr(B["codes"]), _ptr(B["scales"]), _ptr(B.get("tscale")), N, _ptr(workspace), wsb,
                               F32 if out.dtype == torch.float32 else BF16, _ptr(out), _stream(stream))
    _check(st, "qfp4_gemm_fused_rq_ex")
    return out


def linear_forward(X, W, fmt=NVFP4, four6=False, out_dtype=None, out=None, workspace=None, stream=None):
    """Y = X W^T through rotated FP4 operands (qfp4_linear_forward); X (M, K)
    and W (N, K) bf16 CUDA tensors."""
    torch = _torch()
    _input(X, "X")
    _input(W, "W")
    M, K = X.shape
    N = W.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32 if out_dtype is None else out_dtype, device=X.device)
    wsb = qfp4_linear_forward_workspace_bytes(M, N, K, fmt)
    if workspace is None:
        workspace = torch.empty(max(wsb, 16), dtype=torch.uint8, device=X.device)
    st = qfp4_linear_forward(_ptr(X), _ptr(W), M, N, K, fmt, int(four6), F32 if out.dtype == torch.float32 else BF16,
                             _ptr(out), _ptr(workspace), wsb, _stream(stream))
    _check(st, "qfp4_linear_forward")
    return out


def linear_backward(G, X, W, fmt=NVFP4, seed=0, out_dtype=None, want_dx=True, want_dw=True, out=None,
                    workspace=None, stream=None):
    """(dX, dW) = (G W, G^T X) through quantized operands
    (qfp4_linear_backward); G (M, N), X (M, K), W (N, K) bf16 CUDA tensors."""
    torch = _torch()
    _input(G, "G")
    for t, name in ((X, "X"), (W, "W")):
        if t is not None:
            _input(t, name)
    M, N = G.shape
    K = X.shape[1] if X is not None else W.shape[1]
    dt = torch.float32 if out_dtype is None else out_dtype
    o = dict(out) if out is not None else {}
    if want_dx and "dX" not in o:
        o["dX"] = torch.empty((M, K), dtype=dt, device=G.device)
    if want_dw and "dW" not in o:
        o["dW"] = torch.empty((N, K), dtype=dt, device=G.device)
    wsb = qfp4_linear_backward_workspace_bytes(M, N, K, fmt)
    if workspace is None:
        workspace = torch.empty(max(wsb, 16), dtype=torch.uint8, device=G.device)
    st = qfp4_linear_backward(_ptr(G), _ptr(X), _ptr(W), M, N, K, fmt, seed, F32 if dt == torch.float32 else BF16,
                              _ptr(o.get("dX")), _ptr(o.get("dW")), _ptr(workspace), wsb, _stream(stream))
    _check(st, "qfp4_linear_backward")
    return o.get("dX"), o.get("dW")


def kl_calibrate(x, bins=2048, levels=8, grid=0, stream=None, out=None):
    """KL-divergence clip point of a CUDA tensor (qfp4_kl_calibrate); returns
    dict(clip (1,) float32, best (1,) int32, kl (bins - first + 1,) float64,
    hist (bins,) int64 holding the uint64 counts)."""
    torch = _torch()
    _input(x, "x", dims=None)
    dev = x.device
    first = 8 if grid else levels
    o = dict(out) if out is not None else {
        "clip": torch.empty(1, dtype=torch.float32, device=dev), "best": torch.empty(1, dtype=torch.int32, device=dev),
        "kl": torch.empty(bins - first + 1, dtype=torch.float64, device=dev),
        "hist": torch.empty(bins, dtype=torch.int64, device=dev)}
    wsb = qfp4_kl_calibrate_workspace_bytes(bins, levels, grid)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)
    st = qfp4_kl_calibrate(_ptr(x), _xdt(x), x.numel(), bins, levels, grid, _ptr(o["clip"]), _ptr(o["best"]),
                           _ptr(o["kl"]), _ptr(o["hist"]), _ptr(ws), wsb, _stream(stream))
    _check(st, "qfp4_kl_calibrate")
    return o

