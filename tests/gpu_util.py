"""Helpers shared by the GPU parity tests (marshalling only)."""
import numpy as np
import torch


def to_dev(x: np.ndarray) -> torch.Tensor:
    """numpy bf16 bits (uint16) or float32 -> CUDA tensor of the same bytes."""
    if x.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    torch.cuda.synchronize()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def mismatch_report(got: np.ndarray, ref: np.ndarray, name: str) -> str:
    bad = np.argwhere(got != ref)
    return f"{name}: {len(bad)} mismatches of {ref.size}; first at {bad[:5].tolist()}: got {got[tuple(bad[0])] if len(bad) else None} want {ref[tuple(bad[0])] if len(bad) else None}"


# ------------------------------------------------------------------ rounding-boundary inputs
E2M1_MIDPOINTS = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)
E4M3_MIDPOINTS = (1.0625, 1.1875, 1.3125, 1.4375, 1.5625, 1.6875, 1.8125, 1.9375)


def nvfp4_boundary_blocks(kind: str) -> np.ndarray:
    """(n, 16) float64 blocks that put NVFP4 quotients on rounding boundaries.

    Block 0 holds the tensor maximum alone.  kind 'bf16': the maximum is 168,
    so s_t = 168 / 2688 = 2^-4 exactly, each block's scale is S = d 2^-4 for
    a power of two d (the block holds 6 S), and its other values are
    +-m S for the E2M1 midpoints m: exact ties of x / S.  kind 'f32': the
    maximum is 168 + 3 * 2^-16, so s_t has a long significand, and the
    values sit 0, 1, 2 or 3 ulps (steps of 2^-23 relative) either side of
    m S.  Further blocks put (amax / 6) / s_t on (or next to) the E4M3
    midpoints, normal and subnormal, with filler values below their maximum."""
    f32 = kind == "f32"
    amax_t = np.float32(168.0 + (3 * 2.0 ** -16 if f32 else 0.0))
    s_t = float(np.float32(amax_t / np.float32(2688.0)))
    ks = (0, 1, -1, 2, -2, 3, -3) if f32 else (0,)
    pairs = [(m, k) for m in E2M1_MIDPOINTS for k in ks]
    blocks = [[float(amax_t)] + [0.0] * 15]
    for j in range(-9, 8):
        S = float(np.float32(np.float32(2.0 ** j) * np.float32(s_t)))
        for start in range(0, len(pairs), 15):
            row = [float(np.float32(6.0 * S))]
            for t, (m, k) in enumerate(pairs[start:start + 15]):
                row.append((-1.0 if (t + start) % 2 else 1.0) * m * S * (1.0 + k * 2.0 ** -23))
            blocks.append(row + [0.0] * (16 - len(row)))
    tops = [(t, j) for t in E4M3_MIDPOINTS for j in (-3, 0, 4)] + [(t * 2.0 ** 6, -15) for t in (0.5, 1.5, 2.5, 6.5)]
    for t, j in tops:
        for k in ks:
            amax = 6.0 * t * 2.0 ** j * s_t * (1.0 + k * 2.0 ** -23)
            blocks.append([amax] + [(-1.0) ** i * amax * i / 16.0 for i in range(1, 16)])
    return np.asarray(blocks, np.float64)


def encode_input(v: np.ndarray, kind: str) -> np.ndarray:
    """float64 values -> the kernel's input array: float32, or bf16 bits
    (the 'bf16' blocks above are exact in bf16 except filler values, which
    round toward values still below their block maximum)."""
    f = np.asarray(v, np.float64).astype(np.float32)
    if kind == "f32":
        return f
    import synth
    return synth.f32_to_bf16_bits(f)


def blocks_to_rows(blocks: np.ndarray, K: int = 128) -> np.ndarray:
    """Blocks of 16 laid along K, K // 16 per row, zero blocks as padding."""
    per = K // 16
    n = -(-len(blocks) // per) * per
    out = np.zeros((n, 16), np.float64)
    out[:len(blocks)] = blocks
    return out.reshape(n // per, K)


def blocks_to_tiles(blocks: np.ndarray, tiles_per_row: int = 4) -> np.ndarray:
    """Each block repeated over the 16 rows of a 16 x 16 tile; tiles laid
    out row-major, zero tiles as padding."""
    n = -(-len(blocks) // tiles_per_row) * tiles_per_row
    b = np.zeros((n, 16), np.float64)
    b[:len(blocks)] = blocks
    tiles = np.repeat(b[:, None, :], 16, axis=1)                  # (n, 16, 16)
    R = n // tiles_per_row
    return tiles.reshape(R, tiles_per_row, 16, 16).transpose(0, 2, 1, 3).reshape(R * 16, tiles_per_row * 16)


# ------------------------------------------------------------------ guarded outputs
# Every output a GPU test hands to the library sits between two 256-byte
# guard bands filled with a pattern; after each test (an autouse fixture in
# conftest.py) the bands must be intact, so a kernel that writes past either
# end of an output buffer fails the test that made it.  The output itself
# starts out holding the pattern too, so elements a kernel forgets to write
# differ from the oracle.
GUARD_BYTES = 256
GUARD_PATTERN = 0xA5
_guards = []


def guarded(shape, dtype, device="cuda"):
    shape = tuple(int(s) for s in shape)
    n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
    raw = torch.full((n + 2 * GUARD_BYTES,), GUARD_PATTERN, dtype=torch.uint8, device=device)
    _guards.append((raw, n))
    return raw[GUARD_BYTES:GUARD_BYTES + n].view(dtype).view(shape)


def check_guards():
    """Assert every guard band since the last check is intact, then forget them."""
    if not _guards:
        return
    torch.cuda.synchronize()
    bad = []
    for raw, n in _guards:
        pre, post = raw[:GUARD_BYTES], raw[GUARD_BYTES + n:]
        if not bool((pre == GUARD_PATTERN).all()) or not bool((post == GUARD_PATTERN).all()):
            bad.append((n, int((pre != GUARD_PATTERN).sum()), int((post != GUARD_PATTERN).sum())))
    _guards.clear()
    assert not bad, f"writes outside output buffers (bytes, bytes changed before, after): {bad}"


def _fmt_g(fmt):
    import bit_fwht_hadamard_b200 as q
    return 32 if fmt == q.MXFP4 else 16


def quantize(x, fmt, rounding=0, rotate=False, block2d=False, four6=False, seed=0, transposed=False, rule=0,
             amax_in=None, amax_out=None):
    """q.quantize with every output in a guarded buffer."""
    import bit_fwht_hadamard_b200 as q
    M, K = x.shape
    g = _fmt_g(fmt)
    o = {"codes": guarded((M, K // 2), torch.uint8), "scales": guarded((M, K // g), torch.uint8)}
    if transposed:
        o["codesT"] = guarded((K, M // 2), torch.uint8)
        o["scalesT"] = guarded((K, M // g), torch.uint8)
    if fmt == q.NVFP4:
        o["tscale"] = guarded((1,), torch.float32)
    return q.quantize(x, fmt, rounding, rotate=rotate, block2d=block2d, four6=four6, seed=seed,
                      transposed=transposed, out=o, rule=rule, amax_in=amax_in, amax_out=amax_out)


def quantize_mxfp8(x, rounding=0, seed=0, transposed=False):
    import bit_fwht_hadamard_b200 as q
    M, K = x.shape
    o = {"codes": guarded((M, K), torch.uint8), "scales": guarded((M, K // 32), torch.uint8)}
    if transposed:
        o["codesT"] = guarded((K, M), torch.uint8)
        o["scalesT"] = guarded((K, M // 32), torch.uint8)
    return q.quantize_mxfp8(x, rounding, seed=seed, transposed=transposed, out=o)


def quantize_fp32scale(x, gran):
    import bit_fwht_hadamard_b200 as q
    M, K = x.shape
    n = {q.GRAN_TENSOR: 1, q.GRAN_ROW: M, q.GRAN_GROUP16: M * K // 16, q.GRAN_GROUP32: M * K // 32}[gran]
    return q.quantize_fp32scale(x, gran, out={"codes": guarded((M, K // 2), torch.uint8),
                                              "scales": guarded((n,), torch.float32)})


def dequantize(qd, M, K, fmt, out_dtype=None):
    import bit_fwht_hadamard_b200 as q
    return q.dequantize(qd, M, K, fmt, out=guarded((M, K), out_dtype or torch.float32))


def gemm(A, B, M, N, K, fmt, out_dtype=None):
    import bit_fwht_hadamard_b200 as q
    return q.gemm(A, B, M, N, K, fmt, out=guarded((M, N), out_dtype or torch.float32))


def gemm_fused_rq(A_bf16, B, N, fmt, rotate=True, four6=False, out_dtype=None, A_amax_in=None, A_amax_out=None):
    import bit_fwht_hadamard_b200 as q
    return q.gemm_fused_rq(A_bf16, B, N, fmt=fmt, rotate=rotate, four6=four6,
                           out=guarded((A_bf16.shape[0], N), out_dtype or torch.float32), A_amax_in=A_amax_in,
                           A_amax_out=A_amax_out)
