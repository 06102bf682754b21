"""CPU oracle for FP4 microscaling quantization and the block-scaled FP4 GEMM.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
benchmark's ``cpu_baseline`` / ``--impl reference`` legs may import this
package; the product path (``bit_fwht_hadamard_b200``) never does.

The arithmetic lives in ``qfp4_oracle.c`` (plain single-threaded C, each
routine citing the page it follows); this module only compiles it and
marshals numpy arrays through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from ctypes import POINTER, c_double, c_float, c_int, c_int64, c_uint8, c_uint16, c_uint32, c_uint64, c_void_p

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qfp4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

MXFP4, NVFP4, MXFP8 = 0, 1, 2
RULE_DEFAULT, RULE_OCP_FLOOR, RULE_E4M3_UP = 0, 1, 2
RNE, SR = 0, 1
BF16, F32 = 0, 1
GRAN_TENSOR, GRAN_ROW, GRAN_GROUP16, GRAN_GROUP32 = 0, 1, 2, 3
OK, ERR_ARG, ERR_SHAPE, ERR_UNSUPPORTED = 0, -1, -2, -3


def build(force: bool = False) -> str:
    """Compile the oracle with plain IEEE semantics (no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "qfp4_oracle.h"))
    ):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
             "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        L = _lib
        L.or_e2m1_value.restype = c_float
        L.or_e2m1_value.argtypes = [c_uint8]
        L.or_e2m1_rne.restype = c_uint8
        L.or_e2m1_rne.argtypes = [c_float]
        L.or_e2m1_sr.restype = c_uint8
        L.or_e2m1_sr.argtypes = [c_float, c_uint32]
        L.or_e4m3_value.restype = c_float
        L.or_e4m3_value.argtypes = [c_uint8]
        L.or_e4m3_rne.restype = c_uint8
        L.or_e4m3_rne.argtypes = [c_float]
        L.or_e4m3_sr.restype = c_uint8
        L.or_e4m3_sr.argtypes = [c_float, c_uint32]
        L.or_e8m0_value.restype = c_double
        L.or_e8m0_value.argtypes = [c_uint8]
        L.or_scale_exp.restype = c_int
        L.or_scale_exp.argtypes = [c_float, c_double]
        L.or_philox4x32_10.restype = None
        L.or_philox4x32_10.argtypes = [POINTER(c_uint32), POINTER(c_uint32), POINTER(c_uint32)]
        L.or_sr_word.restype = c_uint32
        L.or_sr_word.argtypes = [c_uint64, c_uint64]
        L.or_fwht128.restype = None
        L.or_fwht128.argtypes = [POINTER(c_float)]
        L.or_quantize.restype = c_int
        L.or_quantize.argtypes = [c_void_p, c_int, c_int64, c_int64, c_int, c_int, c_int, c_int, c_int,
                                  c_uint64, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]
        L.or_scale_exp_floor.restype = c_int
        L.or_scale_exp_floor.argtypes = [c_float, c_int]
        L.or_e4m3_up.restype = c_uint8
        L.or_e4m3_up.argtypes = [c_float]
        L.or_quantize_ex.restype = c_int
        L.or_quantize_ex.argtypes = [c_void_p, c_int, c_int64, c_int64, c_int, c_int, c_int, c_int, c_int, c_int,
                                     c_uint64, c_int64, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                     c_void_p, c_void_p]
        L.or_tensor_amax.restype = c_float
        L.or_tensor_amax.argtypes = [c_void_p, c_int, c_int64, c_int64, c_int]
        L.or_mxfp4_group.restype = c_int
        L.or_mxfp4_group.argtypes = [c_void_p, c_void_p, c_int, c_int, c_int, c_uint64, c_void_p, c_void_p]
        L.or_abs_histogram.restype = c_int
        L.or_abs_histogram.argtypes = [c_void_p, c_int, c_int64, c_int, c_float, c_void_p]
        L.or_e2m1_level_of_bin.restype = c_int
        L.or_e2m1_level_of_bin.argtypes = [c_int64, c_int64]
        L.or_kl_calibrate.restype = c_int
        L.or_kl_calibrate.argtypes = [c_void_p, c_int, c_int, c_int, c_void_p, c_void_p]
        L.or_kl_threshold.restype = c_float
        L.or_kl_threshold.argtypes = [c_float, c_int, c_int]
        L.or_four6_pick.restype = c_int
        L.or_four6_pick.argtypes = [c_void_p, c_float, c_void_p, c_void_p]
        L.or_quantize_mxfp8.restype = c_int
        L.or_quantize_mxfp8.argtypes = [c_void_p, c_int, c_int64, c_int64, c_int, c_uint64,
                                        c_void_p, c_void_p, c_void_p, c_void_p]
        L.or_quantize_fp32scale.restype = c_int
        L.or_quantize_fp32scale.argtypes = [c_void_p, c_int, c_int64, c_int64, c_int, c_void_p, c_void_p]
        L.or_dequantize.restype = c_int
        L.or_dequantize.argtypes = [c_void_p, c_void_p, c_void_p, c_int64, c_int64, c_int, c_void_p]
        L.or_dequantize_mxfp8.restype = c_int
        L.or_dequantize_mxfp8.argtypes = [c_void_p, c_void_p, c_int64, c_int64, c_void_p]
        L.or_f64_to_bf16.restype = c_uint16
        L.or_f64_to_bf16.argtypes = [c_double]
        L.or_f64_to_f32.restype = c_float
        L.or_f64_to_f32.argtypes = [c_double]
        L.or_gemm_sampled.restype = c_int
        L.or_gemm_sampled.argtypes = [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                      c_int64, c_int64, c_int64, c_int, c_void_p, c_void_p, c_int64,
                                      c_void_p, c_void_p]
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data


def _xdt(x: np.ndarray) -> int:
    if x.dtype == np.uint16:
        return BF16
    if x.dtype == np.float32:
        return F32
    raise TypeError("x must be uint16 (bfloat16 bits) or float32")


class OracleError(RuntimeError):
    def __init__(self, status: int):
        super().__init__(f"oracle status {status}")
        self.status = status


def _check(st: int) -> None:
    if st != OK:
        raise OracleError(st)


# ---------------------------------------------------------------- scalars
def e2m1_value(code: int) -> float:
    return lib().or_e2m1_value(code)


def e2m1_rne(v: float) -> int:
    return lib().or_e2m1_rne(v)


def e2m1_sr(v: float, r: int) -> int:
    return lib().or_e2m1_sr(v, r)


def e4m3_value(b: int) -> float:
    return lib().or_e4m3_value(b)


def e4m3_rne(v: float) -> int:
    return lib().or_e4m3_rne(v)


def e4m3_sr(v: float, r: int) -> int:
    return lib().or_e4m3_sr(v, r)


def e8m0_value(b: int) -> float:
    return lib().or_e8m0_value(b)


def scale_exp(amax: float, top: float) -> int:
    return lib().or_scale_exp(amax, top)


def philox4x32_10(ctr, key):
    c = (c_uint32 * 4)(*ctr)
    k = (c_uint32 * 2)(*key)
    o = (c_uint32 * 4)()
    lib().or_philox4x32_10(c, k, o)
    return list(o)


def sr_word(seed: int, e: int) -> int:
    return lib().or_sr_word(seed, e)


def fwht128(x: np.ndarray) -> np.ndarray:
    y = np.ascontiguousarray(x, dtype=np.float32).copy()
    assert y.shape == (128,)
    lib().or_fwht128(y.ctypes.data_as(POINTER(c_float)))
    return y


def f64_to_bf16(v: float) -> int:
    return lib().or_f64_to_bf16(v)


# ---------------------------------------------------------------- arrays
def quantize(x: np.ndarray, fmt: int, rounding: int = RNE, rotate: bool = False, block2d: bool = False,
             four6: bool = False, seed: int = 0, transposed: bool = False):
    """Returns dict(codes, scales, [codesT, scalesT], [tscale])."""
    x = np.ascontiguousarray(x)
    M, K = x.shape
    g = 32 if fmt == MXFP4 else 16
    codes = np.zeros((M, K // 2), np.uint8)
    scales = np.zeros((M, K // g), np.uint8)
    codesT = scalesT = None
    if transposed:
        codesT = np.zeros((K, M // 2), np.uint8)
        scalesT = np.zeros((K, M // g), np.uint8)
    tscale = np.zeros(1, np.float32)
    _check(lib().or_quantize(_p(x), _xdt(x), M, K, fmt, rounding, int(rotate), int(block2d), int(four6),
                             seed, _p(codes), _p(scales), _p(codesT), _p(scalesT), _p(tscale)))
    out = {"codes": codes, "scales": scales}
    if transposed:
        out["codesT"], out["scalesT"] = codesT, scalesT
    if fmt == NVFP4:
        out["tscale"] = tscale
    return out


def quantize_status(x, fmt, rounding=RNE, rotate=False, block2d=False, four6=False, seed=0,
                    transposed=False, M=None, K=None) -> int:
    """Status code only (argument validation pins)."""
    x = np.ascontiguousarray(x)
    M = x.shape[0] if M is None else M
    K = x.shape[1] if K is None else K
    g = 32 if fmt == MXFP4 else 16
    n = max(M * K, 2)
    codes = np.zeros(n, np.uint8)
    scales = np.zeros(n, np.uint8)
    codesT = np.zeros(n, np.uint8) if transposed else None
    scalesT = np.zeros(n, np.uint8) if transposed else None
    tscale = np.zeros(1, np.float32)
    return lib().or_quantize(_p(x), _xdt(x), M, K, fmt, rounding, int(rotate), int(block2d), int(four6), seed,
                             _p(codes), _p(scales), _p(codesT), _p(scalesT), _p(tscale))


def scale_exp_floor(amax: float, emax: int = 2) -> int:
    return lib().or_scale_exp_floor(amax, emax)


def e4m3_up(v: float) -> int:
    return lib().or_e4m3_up(v)


def quantize_ex(x: np.ndarray, fmt: int, rounding: int = RNE, rotate: bool = False, block2d: bool = False,
                four6: bool = False, rule: int = RULE_DEFAULT, seed: int = 0, row0: int = 0, amax_in=None,
                want_amax: bool = False, transposed: bool = False):
    """or_quantize_ex: scale-rule variants, a given tensor amax (NVFP4) and
    a first-row offset.  Returns dict(codes, scales, [codesT, scalesT],
    [tscale], [amax])."""
    x = np.ascontiguousarray(x)
    M, K = x.shape
    g = 32 if fmt == MXFP4 else 16
    codes = np.zeros((M, K // 2), np.uint8)
    scales = np.zeros((M, K // g), np.uint8)
    codesT = scalesT = None
    if transposed:
        codesT = np.zeros((K, M // 2), np.uint8)
        scalesT = np.zeros((K, M // g), np.uint8)
    tscale = np.zeros(1, np.float32)
    ain = None if amax_in is None else np.asarray([amax_in], np.float32)
    aout = np.zeros(1, np.float32) if want_amax else None
    _check(lib().or_quantize_ex(_p(x), _xdt(x), M, K, fmt, rounding, int(rotate), int(block2d), int(four6), rule,
                                seed, row0, _p(ain), _p(codes), _p(scales), _p(codesT), _p(scalesT), _p(tscale),
                                _p(aout)))
    out = {"codes": codes, "scales": scales}
    if transposed:
        out["codesT"], out["scalesT"] = codesT, scalesT
    if fmt == NVFP4:
        out["tscale"] = tscale
    if want_amax:
        out["amax"] = aout
    return out


def quantize_ex_status(x, fmt, rounding=RNE, rotate=False, block2d=False, four6=False, rule=RULE_DEFAULT, seed=0,
                       row0=0, amax_in=None, transposed=False) -> int:
    x = np.ascontiguousarray(x)
    M, K = x.shape
    n = max(M * K, 2)
    bufs = [np.zeros(n, np.uint8) for _ in range(4)]
    tscale = np.zeros(1, np.float32)
    ain = None if amax_in is None else np.asarray([amax_in], np.float32)
    return lib().or_quantize_ex(_p(x), _xdt(x), M, K, fmt, rounding, int(rotate), int(block2d), int(four6), rule,
                                seed, row0, _p(ain), _p(bufs[0]), _p(bufs[1]),
                                _p(bufs[2]) if transposed else None, _p(bufs[3]) if transposed else None,
                                _p(tscale), None)


def tensor_amax(x: np.ndarray, rotate: bool = False) -> float:
    x = np.ascontiguousarray(x)
    return float(lib().or_tensor_amax(_p(x), _xdt(x), x.shape[0], x.shape[1], int(rotate)))


def mxfp4_group(x32: np.ndarray, rounding: int = RNE, four6: bool = False, rule: int = RULE_DEFAULT,
                seed: int = 0, e=None):
    x32 = np.ascontiguousarray(x32, dtype=np.float32)
    e = np.ascontiguousarray(np.arange(32, dtype=np.uint64) if e is None else e, dtype=np.uint64)
    sb = np.zeros(1, np.uint8)
    codes = np.zeros(32, np.uint8)
    pick = lib().or_mxfp4_group(_p(x32), _p(e), rounding, int(four6), rule, seed, _p(sb), _p(codes))
    return pick, int(sb[0]), codes


def four6_pick(x16: np.ndarray, s_t: float):
    x16 = np.ascontiguousarray(x16, dtype=np.float32)
    enc = np.zeros(1, np.uint8)
    codes = np.zeros(16, np.uint8)
    pick = lib().or_four6_pick(_p(x16), s_t, _p(enc), _p(codes))
    return pick, int(enc[0]), codes


def quantize_mxfp8(x: np.ndarray, rounding: int = RNE, seed: int = 0, transposed: bool = False):
    x = np.ascontiguousarray(x)
    M, K = x.shape
    codes = np.zeros((M, K), np.uint8)
    scales = np.zeros((M, K // 32), np.uint8)
    codesT = scalesT = None
    if transposed:
        codesT = np.zeros((K, M), np.uint8)
        scalesT = np.zeros((K, M // 32), np.uint8)
    _check(lib().or_quantize_mxfp8(_p(x), _xdt(x), M, K, rounding, seed, _p(codes), _p(scales),
                                   _p(codesT), _p(scalesT)))
    out = {"codes": codes, "scales": scales}
    if transposed:
        out["codesT"], out["scalesT"] = codesT, scalesT
    return out


def quantize_fp32scale(x: np.ndarray, gran: int):
    x = np.ascontiguousarray(x)
    M, K = x.shape
    n_scales = {GRAN_TENSOR: 1, GRAN_ROW: M, GRAN_GROUP16: M * K // 16, GRAN_GROUP32: M * K // 32}[gran]
    codes = np.zeros((M, K // 2), np.uint8)
    scales = np.zeros(n_scales, np.float32)
    _check(lib().or_quantize_fp32scale(_p(x), _xdt(x), M, K, gran, _p(codes), _p(scales)))
    return {"codes": codes, "scales": scales}


def dequantize(codes: np.ndarray, scales: np.ndarray, tscale, M: int, K: int, fmt: int) -> np.ndarray:
    out = np.zeros((M, K), np.float64)
    ts = None if tscale is None else np.ascontiguousarray(np.asarray(tscale, np.float32).reshape(1))
    _check(lib().or_dequantize(_p(np.ascontiguousarray(codes)), _p(np.ascontiguousarray(scales)), _p(ts),
                               M, K, fmt, _p(out)))
    return out


def dequantize_mxfp8(codes: np.ndarray, scales: np.ndarray, M: int, K: int) -> np.ndarray:
    out = np.zeros((M, K), np.float64)
    _check(lib().or_dequantize_mxfp8(_p(np.ascontiguousarray(codes)), _p(np.ascontiguousarray(scales)),
                                     M, K, _p(out)))
    return out


def gemm_sampled(A: dict, B: dict, M: int, N: int, K: int, fmt: int, rows, cols):
    """Reference Y[rows[t], cols[t]] and sum_k |a||b| for each sampled pair."""
    rows = np.ascontiguousarray(rows, np.int64)
    cols = np.ascontiguousarray(cols, np.int64)
    out = np.zeros(rows.shape[0], np.float64)
    mag = np.zeros(rows.shape[0], np.float64)
    tA = None if fmt != NVFP4 else np.ascontiguousarray(np.asarray(A["tscale"], np.float32).reshape(1))
    tB = None if fmt != NVFP4 else np.ascontiguousarray(np.asarray(B["tscale"], np.float32).reshape(1))
    _check(lib().or_gemm_sampled(_p(np.ascontiguousarray(A["codes"])), _p(np.ascontiguousarray(A["scales"])),
                                 _p(tA), _p(np.ascontiguousarray(B["codes"])), _p(np.ascontiguousarray(B["scales"])),
                                 _p(tB), M, N, K, fmt, _p(rows), _p(cols), rows.shape[0], _p(out), _p(mag)))
    return out, mag


def f64_to_f32_array(v: np.ndarray) -> np.ndarray:
    """binary64 -> binary32, round to nearest even (numpy's IEEE cast)."""
    return np.asarray(v, np.float64).astype(np.float32)


def f64_to_bf16_array(v: np.ndarray) -> np.ndarray:
    L = lib()
    flat = np.asarray(v, np.float64).ravel()
    return np.array([L.or_f64_to_bf16(float(t)) for t in flat], np.uint16).reshape(np.shape(v))


# ---------------------------------------------------------------- KL calibration
def abs_histogram(x: np.ndarray, bins: int, amax: float) -> np.ndarray:
    x = np.ascontiguousarray(x)
    h = np.zeros(bins, np.uint64)
    _check(lib().or_abs_histogram(_p(x), _xdt(x), x.size, bins, amax, _p(h)))
    return h


def e2m1_level_of_bin(b: int, i: int) -> int:
    return lib().or_e2m1_level_of_bin(b, i)


def kl_calibrate(hist: np.ndarray, levels: int = 8, grid: int = 0):
    """(best i, kl array over candidates first .. bins)."""
    hist = np.ascontiguousarray(hist, np.uint64)
    bins = hist.size
    first = 8 if grid else levels
    kl = np.zeros(bins - first + 1, np.float64)
    best = np.zeros(1, np.int32)
    _check(lib().or_kl_calibrate(_p(hist), bins, levels, grid, _p(kl), _p(best)))
    return int(best[0]), kl


def kl_threshold(amax: float, bins: int, i: int) -> float:
    return float(np.float32(lib().or_kl_threshold(amax, bins, i)))

