"""Multi-threaded use of the CPU oracle for full-size parity tests.

The oracle itself is single-threaded; its ctypes calls release the GIL, so
row slices run in parallel threads.  Slices are quantized with their
logical first row (the random words stay keyed on the whole tensor's
element index) and, for NVFP4, with the whole tensor's amax, which
reassembles the whole-tensor result bit for bit
(tests/test_oracle_variants.py::test_row_slices_with_row_offsets_reassemble_the_whole).
Nothing here does any of the method's arithmetic."""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

import oracle


def threads() -> int:
    return max(1, min(64, os.cpu_count() or 1))


def _slices(M: int, n: int, align: int = 1):
    step = max(align, -(-M // n))
    step = -(-step // align) * align
    return [(a, min(M, a + step)) for a in range(0, M, step)]


def tensor_amax(x: np.ndarray, rotate: bool = False) -> float:
    with ThreadPoolExecutor(threads()) as ex:
        parts = list(ex.map(lambda s: oracle.tensor_amax(x[s[0]:s[1]], rotate), _slices(x.shape[0], threads())))
    return max(parts)


def quantize(x: np.ndarray, fmt: int, rounding: int = oracle.RNE, rotate: bool = False, four6: bool = False,
             seed: int = 0, rule: int = oracle.RULE_DEFAULT, amax_in=None) -> dict:
    """1D quantize of x (rows independent) as oracle.quantize / quantize_ex."""
    M = x.shape[0]
    amax = amax_in
    if fmt == oracle.NVFP4 and amax is None:
        amax = tensor_amax(x, rotate)

    def run(s):
        return oracle.quantize_ex(x[s[0]:s[1]], fmt, rounding, rotate=rotate, four6=four6, rule=rule, seed=seed,
                                  row0=s[0], amax_in=amax if fmt == oracle.NVFP4 else None)

    with ThreadPoolExecutor(threads()) as ex:
        parts = list(ex.map(run, _slices(M, 4 * threads())))
    out = {k: np.concatenate([p[k] for p in parts]) for k in ("codes", "scales")}
    if fmt == oracle.NVFP4:
        out["tscale"] = parts[0]["tscale"]
        if amax_in is None:
            out["amax"] = np.asarray([amax], np.float32)
    return out


def gemm_sampled(A: dict, B: dict, M: int, N: int, K: int, fmt: int, rows, cols):
    """oracle.gemm_sampled over chunks of the sample list in parallel."""
    rows = np.asarray(rows, np.int64)
    cols = np.asarray(cols, np.int64)
    chunks = _slices(len(rows), 4 * threads())

    def run(s):
        return oracle.gemm_sampled(A, B, M, N, K, fmt, rows[s[0]:s[1]], cols[s[0]:s[1]])

    with ThreadPoolExecutor(threads()) as ex:
        parts = list(ex.map(run, chunks))
    return np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts])
