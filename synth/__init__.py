"""Seeded synthetic inputs shared by the tests, the oracle checks and the benchmark.

This module holds no arithmetic of the quantization method: it only draws
random numbers and builds the input tensors of the workloads (bfloat16 bits
or binary32).  Both the CUDA path and the CPU oracle are fed the same bytes.

Recipe (reproducible across machines; no library RNG stream is relied on):
  * raw 64-bit words: the splitmix64 sequence started at a per-(seed, stream)
    key, word i = splitmix64(key + i * 0x9E3779B97F4A7C15);
  * uniforms in (0, 1): ((w >> 11) + 0.5) * 2^-53;
  * normals: Box-Muller on consecutive uniform pairs, in binary64;
  * tensors: binary64 value * std (* outlier factor) -> binary32 (round to
    nearest) -> bfloat16 (round to nearest even on the binary32 bits).
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_CHUNK = 1 << 22


def _splitmix64(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
    return z ^ (z >> np.uint64(31))


def _key(seed: int, stream: int) -> np.uint64:
    with np.errstate(over="ignore"):
        k = _splitmix64(np.array([(seed * 0x100000001B3 + stream * 0xC2B2AE3D27D4EB4F) & ((1 << 64) - 1)],
                                 np.uint64))
    return k[0]


def _words(key: np.uint64, start: int, n: int) -> np.ndarray:
    with np.errstate(over="ignore"):
        i = np.arange(start, start + n, dtype=np.uint64)
        return _splitmix64(key + (i + np.uint64(1)) * _GAMMA)


def _uniform(key, start, n):
    w = _words(key, start, n)
    return ((w >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)


def _normal_chunk(key, start, n):
    """normals for indices [start, start+n); index 2t, 2t+1 share a pair."""
    p0, p1 = start // 2, (start + n + 1) // 2
    u = _uniform(key, 2 * p0, 2 * (p1 - p0)).reshape(-1, 2)
    r = np.sqrt(-2.0 * np.log(u[:, 0]))
    th = 2.0 * np.pi * u[:, 1]
    z = np.empty((p1 - p0) * 2, np.float64)
    z[0::2] = r * np.cos(th)
    z[1::2] = r * np.sin(th)
    off = start - 2 * p0
    return z[off:off + n]


def _parallel(n: int, fn):
    """fn(start, count) -> ndarray; concatenated over chunks on all cores."""
    starts = list(range(0, n, _CHUNK))
    if len(starts) <= 1:
        return fn(0, n)
    with ThreadPoolExecutor(max_workers=min(len(starts), os.cpu_count() or 1)) as ex:
        parts = list(ex.map(lambda s: fn(s, min(_CHUNK, n - s)), starts))
    return np.concatenate(parts)


def normal(n: int, seed: int, stream: int = 0) -> np.ndarray:
    """n standard normals (binary64)."""
    key = _key(seed, stream)
    return _parallel(n, lambda s, c: _normal_chunk(key, s, c))


def uniform(n: int, seed: int, stream: int = 0) -> np.ndarray:
    key = _key(seed, stream)
    return _parallel(n, lambda s, c: _uniform(key, s, c))


def permutation_prefix(n: int, k: int, seed: int, stream: int = 0) -> np.ndarray:
    """first k entries of a seeded Fisher-Yates shuffle of range(n)."""
    k = min(k, n)
    a = np.arange(n, dtype=np.int64)
    w = _words(_key(seed, stream), 0, k)
    for t in range(k):
        j = t + int(w[t] % np.uint64(n - t))
        a[t], a[j] = a[j], a[t]
    return np.sort(a[:k])


def f32_to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """binary32 -> bfloat16 bits, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x32, np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.asarray(h, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def to_bf16(z: np.ndarray, shape) -> np.ndarray:
    def conv(s, c):
        return f32_to_bf16_bits(z[s:s + c].astype(np.float32))
    return _parallel(z.size, conv).reshape(shape)


# ---------------------------------------------------------------- workloads
def gaussian_bf16(M: int, K: int, seed: int, std: float = 1.0, stream: int = 0,
                  outlier_cols=None, outlier_factor: float = 1.0) -> np.ndarray:
    z = normal(M * K, seed, stream) * std
    if outlier_cols is not None and len(outlier_cols):
        z = z.reshape(M, K)
        z[:, outlier_cols] *= outlier_factor
        z = z.reshape(-1)
    return to_bf16(z, (M, K))


def student_t3_bf16(M: int, K: int, seed: int, scale: float = 0.5, stream: int = 0) -> np.ndarray:
    """scale * t, t = Z / sqrt(chi2_3 / 3), chi2_3 from three more normals."""
    n = M * K
    z = normal(n, seed, stream)
    chi = normal(n, seed, stream + 1) ** 2 + normal(n, seed, stream + 2) ** 2 + normal(n, seed, stream + 3) ** 2
    return to_bf16(scale * z / np.sqrt(chi / 3.0), (M, K))


def outlier_columns(K: int, count: int, seed: int, stream: int = 99) -> np.ndarray:
    return permutation_prefix(K, count, seed, stream)


# Workload recipes (sizes and distributions of the five configurations).
def cfg1_W(seed: int = 1001) -> np.ndarray:
    """MLP fc1-sized weight 256 x 784, N(0, 0.04^2), binary32."""
    return (normal(256 * 784, seed, 0) * 0.04).astype(np.float32).reshape(256, 784)


def cfg1_X(seed: int = 1001) -> np.ndarray:
    """input 64 x 784, N(0,1), binary32."""
    return normal(64 * 784, seed, 1).astype(np.float32).reshape(64, 784)


def cfg2_X(M: int = 4096, K: int = 4096, seed: int = 1002) -> np.ndarray:
    """bf16 N(0,1) with 40 seeded channels (columns) scaled x20."""
    return gaussian_bf16(M, K, seed, 1.0, 0, outlier_columns(K, 40, seed), 20.0)


def cfg3_X(M: int = 8192, K: int = 4096, seed: int = 1003) -> np.ndarray:
    return student_t3_bf16(M, K, seed, 0.5, 0)


def cfg3_W(N: int = 11008, K: int = 4096, seed: int = 1003) -> np.ndarray:
    return gaussian_bf16(N, K, seed, 0.02, 10)


def cfg4_G(M: int = 8192, K: int = 4096, seed: int = 1004) -> np.ndarray:
    """bf16 N(0, 1e-3^2), each entry x100 with probability 0.001."""
    z = normal(M * K, seed, 0) * 1e-3
    hit = uniform(M * K, seed, 1) < 0.001
    z[hit] *= 100.0
    return to_bf16(z, (M, K))


def cfg4_X(M: int = 8192, K: int = 4096, seed: int = 1004) -> np.ndarray:
    return gaussian_bf16(M, K, seed, 1.0, 20, outlier_columns(K, 40, seed, 98), 20.0)


def cfg4_W(N: int = 4096, K: int = 4096, seed: int = 1004) -> np.ndarray:
    return gaussian_bf16(N, K, seed, 0.02, 30)


def cfg5_A(M: int, K: int, seed: int = 1005) -> np.ndarray:
    """bf16 N(0,1) with round(0.005*K) outlier channels x30."""
    return gaussian_bf16(M, K, seed, 1.0, 0, outlier_columns(K, int(round(0.005 * K)), seed), 30.0)


def cfg5_B(N: int, K: int, seed: int = 1005) -> np.ndarray:
    return gaussian_bf16(N, K, seed, 1.0, 40)


def relu_activation(M: int, K: int, seed: int = 1006) -> np.ndarray:
    """bf16 ReLU-like activation: max(0, z1 + 0.3 * t3), z1 ~ N(0,1) and t3 a
    Student-t(3) draw (z2 / sqrt(chi2_3 / 3)), so most mass sits near zero and
    a thin tail reaches far out (the activation shape of the low-bit blog's
    KL clipping section)."""
    n = M * K
    z = normal(n, seed, 0)
    zz = normal(n, seed, 1)
    c = normal(3 * n, seed, 2).reshape(3, n)
    t3 = zz / np.sqrt((c * c).sum(0) / 3.0)
    return to_bf16(np.maximum(0.0, z + 0.3 * t3), (M, K))

