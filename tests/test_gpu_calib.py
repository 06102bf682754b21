"""GPU parity of qfp4_kl_calibrate (low-bit blog §5: KL-divergence clip
calibration) against the oracle: the histogram bit for bit, every
candidate's KL within 1e-12 relative (both sides sum the same binary64 terms
in the same order; only the last ulp of log may differ), the same winning
candidate (or one whose KL ties the oracle's minimum to that tolerance), the
clip point bit for bit, and NVFP4 quantization under the clip as its tensor
amax."""
import numpy as np
import pytest
import torch

import bit_fwht_hadamard_b200 as q
import gpu_util as GU
import oracle
import synth
from gpu_util import host, to_dev

pytestmark = pytest.mark.gpu


def _check(x_host, got, bins, levels, grid):
    xf = synth.bf16_bits_to_f32(x_host) if x_host.dtype == np.uint16 else x_host
    amax = float(np.float32(np.abs(xf).max()))
    h = oracle.abs_histogram(x_host, bins, amax)
    assert np.array_equal(host(got["hist"]).view(np.uint64), h)
    best, kl = oracle.kl_calibrate(h, levels, grid)
    gkl = host(got["kl"])
    assert np.array_equal(np.isinf(gkl), np.isinf(kl))
    f = np.isfinite(kl)
    assert np.allclose(gkl[f], kl[f], rtol=1e-12, atol=1e-300)
    gbest = int(host(got["best"])[0])
    first = 8 if grid else levels
    assert gbest == best or abs(kl[gbest - first] - kl[best - first]) <= 1e-12 * abs(kl[best - first])
    assert host(got["clip"])[0] == np.float32(oracle.kl_threshold(amax, bins, gbest))
    return amax, gbest


@pytest.mark.parametrize("grid,levels", [(0, 8), (0, 128), (1, 8)], ids=["uniform8", "uniform128", "e2m1"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_kl_calibrate_matches_oracle(grid, levels, dtype):
    x = synth.relu_activation(256, 4096, seed=60 + grid + levels)
    if dtype == "f32":
        x = synth.bf16_bits_to_f32(x) * np.float32(1.0 + 2.0 ** -10)
    got = q.kl_calibrate(to_dev(x), bins=2048, levels=levels, grid=grid)
    amax, best = _check(x, got, 2048, levels, grid)
    assert float(host(got["clip"])[0]) < 0.6 * amax          # clipped inside the tail, as the page finds


@pytest.mark.parametrize("n", [1, 7, 4099, 65536])
def test_kl_calibrate_small_and_ragged(n):
    x = synth.relu_activation(1, n, seed=n)
    got = q.kl_calibrate(to_dev(x), bins=256, levels=4, grid=0)
    _check(x, got, 256, 4, 0)


def test_kl_calibrate_all_zero():
    x = np.zeros((4, 64), np.uint16)
    got = q.kl_calibrate(to_dev(x), bins=64, levels=8)
    assert host(got["hist"])[0] == 256 and host(got["clip"])[0] == 0.0


def test_kl_clip_feeds_the_nvfp4_tensor_scale():
    """Calibrate, then quantize NVFP4 with the clip as the tensor amax: one
    pass over X, and the codes follow the oracle under the same amax."""
    x = synth.relu_activation(512, 4096, seed=66)
    got = q.kl_calibrate(to_dev(x), bins=2048, levels=8, grid=1)
    clip = float(host(got["clip"])[0])
    qd = GU.quantize(to_dev(x), q.NVFP4, q.RNE, amax_in=got["clip"])
    ref = oracle.quantize_ex(x, oracle.NVFP4, oracle.RNE, amax_in=clip)
    for k in ("codes", "scales", "tscale"):
        assert np.array_equal(host(qd[k]).view(np.uint8), ref[k].view(np.uint8)), k
    assert q.qfp4_last_device_error() == 0
