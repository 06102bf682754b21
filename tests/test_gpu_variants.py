"""GPU parity of qfp4_quantize_ex: the scale-rule variants (OCP floor E8M0 for
MXFP4, E4M3 rounded up for NVFP4), four-over-six on MXFP4 groups, 32 x 32
MXFP4 tiles, and the caller-supplied tensor amax (delayed scaling), against
the oracle element by element (codes, scales, tensor scale and the reported
amax bit for bit)."""
import numpy as np
import pytest
import torch

import bit_fwht_hadamard_b200 as q
import gpu_util as G
import oracle
import oracle_par
import synth
from gpu_util import host, mismatch_report, to_dev

pytestmark = pytest.mark.gpu


def _cmp(got: dict, ref: dict):
    for k in ("codes", "scales", "codesT", "scalesT", "tscale"):
        if k in ref:
            g = host(got[k]).reshape(ref[k].shape)
            assert np.array_equal(g.view(np.uint8), np.asarray(ref[k]).view(np.uint8)), mismatch_report(
                g.view(np.uint8), np.asarray(ref[k]).view(np.uint8), k)


def _f32(v):
    return torch.tensor([v], dtype=torch.float32, device="cuda")


SHAPES = [(1, 128), (37, 384), (600, 512), (7, 96), (64, 256)]


@pytest.mark.parametrize("M,K", SHAPES)
@pytest.mark.parametrize("rounding", [q.RNE, q.SR], ids=["rne", "sr"])
@pytest.mark.parametrize("rotate", [False, True], ids=["plain", "rot"])
def test_mxfp4_ocp_floor_rule(M, K, rounding, rotate):
    if rotate and K % 128:
        pytest.skip()
    x = synth.cfg2_X(M, K, seed=M + 7 * K)
    got = G.quantize(to_dev(x), q.MXFP4, rounding, rotate=rotate, seed=71, rule=q.SCALE_OCP_FLOOR)
    ref = oracle.quantize_ex(x, oracle.MXFP4, rounding, rotate=rotate, seed=71, rule=oracle.RULE_OCP_FLOOR)
    _cmp(got, ref)


@pytest.mark.parametrize("M,K", SHAPES)
@pytest.mark.parametrize("mode", ["rne", "sr", "four6"])
@pytest.mark.parametrize("rotate", [False, True], ids=["plain", "rot"])
def test_nvfp4_e4m3_round_up_rule(M, K, mode, rotate):
    if rotate and K % 128:
        pytest.skip()
    x = synth.cfg3_X(M, K, seed=M + 11 * K)
    r = q.SR if mode == "sr" else q.RNE
    got = G.quantize(to_dev(x), q.NVFP4, r, rotate=rotate, four6=mode == "four6", seed=72, rule=q.SCALE_E4M3_UP)
    ref = oracle.quantize_ex(x, oracle.NVFP4, r, rotate=rotate, four6=mode == "four6", seed=72,
                             rule=oracle.RULE_E4M3_UP)
    _cmp(got, ref)


@pytest.mark.parametrize("M,K", SHAPES)
@pytest.mark.parametrize("rule", [q.SCALE_DEFAULT, q.SCALE_OCP_FLOOR], ids=["truncfree", "ocpfloor"])
@pytest.mark.parametrize("rotate", [False, True], ids=["plain", "rot"])
def test_mxfp4_four_over_six(M, K, rule, rotate):
    if rotate and K % 128:
        pytest.skip()
    x = synth.cfg3_X(M, K, seed=M + 13 * K)
    got = G.quantize(to_dev(x), q.MXFP4, q.RNE, rotate=rotate, four6=True, rule=rule)
    ref = oracle.quantize_ex(x, oracle.MXFP4, oracle.RNE, rotate=rotate, four6=True, rule=rule)
    _cmp(got, ref)


def test_mxfp4_four_over_six_float32_input():
    x = (np.random.default_rng(5).standard_normal((96, 256)) * 3).astype(np.float32)
    x[4, :32] *= np.float32(7.9 / 6)
    for rule in (q.SCALE_DEFAULT, q.SCALE_OCP_FLOOR):
        _cmp(G.quantize(to_dev(x), q.MXFP4, q.RNE, four6=True, rule=rule),
             oracle.quantize_ex(x, oracle.MXFP4, oracle.RNE, four6=True, rule=rule))


@pytest.mark.parametrize("M,K", [(32, 32), (64, 96), (160, 256), (96, 4096)])
@pytest.mark.parametrize("rounding", [q.RNE, q.SR], ids=["rne", "sr"])
@pytest.mark.parametrize("rule", [q.SCALE_DEFAULT, q.SCALE_OCP_FLOOR], ids=["truncfree", "ocpfloor"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_mxfp4_2d_tiles(M, K, rounding, rule, dtype):
    x = synth.cfg4_G(M, K, seed=M * 3 + K)
    if dtype == "f32":
        x = synth.bf16_bits_to_f32(x) * np.float32(1.0 + 2.0 ** -12)
    got = G.quantize(to_dev(x), q.MXFP4, rounding, block2d=True, seed=1004, transposed=True, rule=rule)
    ref = oracle.quantize_ex(x, oracle.MXFP4, rounding, block2d=True, seed=1004, rule=rule, transposed=True)
    _cmp(got, ref)


def test_mxfp4_2d_full_size_gradient():
    g = synth.cfg4_G()
    for rounding in (q.RNE, q.SR):
        got = G.quantize(to_dev(g), q.MXFP4, rounding, block2d=True, seed=1004, transposed=True)
        ref = oracle.quantize_ex(g, oracle.MXFP4, rounding, block2d=True, seed=1004, transposed=True)
        _cmp(got, ref)


@pytest.mark.parametrize("rounding", [q.RNE, q.SR], ids=["rne", "sr"])
def test_nvfp4_2d_round_up_and_given_amax(rounding):
    x = synth.cfg4_G(64, 128, seed=77)
    own = oracle.tensor_amax(x)
    for rule in (q.SCALE_DEFAULT, q.SCALE_E4M3_UP):
        for amax in (None, own * 0.25):
            got = G.quantize(to_dev(x), q.NVFP4, rounding, block2d=True, seed=3, transposed=True, rule=rule,
                             amax_in=None if amax is None else _f32(amax))
            ref = oracle.quantize_ex(x, oracle.NVFP4, rounding, block2d=True, seed=3, rule=rule, amax_in=amax,
                                     transposed=True)
            _cmp(got, ref)


@pytest.mark.parametrize("M,K", SHAPES)
@pytest.mark.parametrize("rounding", [q.RNE, q.SR], ids=["rne", "sr"])
@pytest.mark.parametrize("rotate", [False, True], ids=["plain", "rot"])
def test_given_amax_and_reported_amax(M, K, rounding, rotate):
    """Given the tensor's own amax the result equals the plain call; given a
    stale amax (x 0.3: top blocks saturate; x 1e-30: every quotient
    overflows and saturates) the result follows the oracle; the amax the
    call reports equals the oracle's own (rotated) amax bit for bit."""
    if rotate and K % 128:
        pytest.skip()
    x = synth.cfg3_X(M, K, seed=M + 17 * K)
    own = oracle.tensor_amax(x, rotate=rotate)
    for amax in (own, own * 0.3, 1e-30, own * 8.0):
        out_amax = G.guarded((1,), torch.float32)
        got = G.quantize(to_dev(x), q.NVFP4, rounding, rotate=rotate, seed=73, amax_in=_f32(amax),
                         amax_out=out_amax)
        ref = oracle.quantize_ex(x, oracle.NVFP4, rounding, rotate=rotate, seed=73, amax_in=amax, want_amax=True)
        _cmp(got, ref)
        assert host(out_amax)[0] == ref["amax"][0] == np.float32(own)
    # only the reported amax, the tensor scale from the call's own pass
    out_amax = G.guarded((1,), torch.float32)
    got = G.quantize(to_dev(x), q.NVFP4, rounding, rotate=rotate, seed=73, amax_out=out_amax)
    _cmp(got, oracle.quantize_ex(x, oracle.NVFP4, rounding, rotate=rotate, seed=73))
    assert host(out_amax)[0] == np.float32(own)


def test_given_amax_with_column_wise_output():
    x = synth.cfg3_X(64, 256, seed=19)
    amax = oracle.tensor_amax(x) * 0.5
    got = G.quantize(to_dev(x), q.NVFP4, q.SR, seed=5, transposed=True, amax_in=_f32(amax))
    _cmp(got, oracle.quantize_ex(x, oracle.NVFP4, oracle.SR, seed=5, amax_in=amax, transposed=True))


def test_given_amax_full_size_single_pass():
    """The cfg3 activation X 8192 x 4096 under the amax of a previous step
    (the tensor's own amax x 0.9): one read of X, bit for bit."""
    x = synth.cfg3_X()
    amax = float(np.float32(oracle_par.tensor_amax(x) * 0.9))
    for four6 in (False, True):
        got = G.quantize(to_dev(x), q.NVFP4, q.RNE, four6=four6, amax_in=_f32(amax))
        ref = oracle_par.quantize(x, oracle.NVFP4, oracle.RNE, four6=four6, amax_in=amax)
        _cmp(got, ref)
    assert q.qfp4_last_device_error() == 0


def test_empty_tensor_with_given_amax():
    e = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    out_amax = G.guarded((1,), torch.float32)
    got = G.quantize(e, q.NVFP4, amax_in=_f32(5376.0), amax_out=out_amax)
    assert host(got["tscale"])[0] == np.float32(2.0) and host(out_amax)[0] == 0.0
