"""Failure detection without a GPU fault: every wait inside the library's
kernels is bounded, and a wait that runs out records an error word that the
host reads with qfp4_last_device_error() while the context stays usable.

The self-test entry point launches one thread that waits on a barrier
nothing completes (no copy or MMA in flight) with a 1 ms limit; that is the
give-up path all the kernels share."""
import numpy as np
import pytest
import torch

import bit_fwht_hadamard_b200 as q
import gpu_util as G
import oracle
import synth
from gpu_util import host, to_dev

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_the_host_reads_the_code():
    assert q.qfp4_last_device_error() == 0
    st = q.qfp4_selftest_wait_timeout(1000, torch.cuda.current_stream().cuda_stream)
    assert st == q.OK
    assert q.qfp4_last_device_error() == q.DEV_ERR_TIMEOUT
    assert q.qfp4_last_device_error() == 0                    # cleared by the read
    # the context is still usable: a quantize afterwards matches the oracle
    x = synth.cfg2_X(64, 256, seed=17)
    got = G.quantize(to_dev(x), q.MXFP4, q.SR, rotate=True, seed=5)
    ref = oracle.quantize(x, oracle.MXFP4, oracle.SR, rotate=True, seed=5)
    assert np.array_equal(host(got["codes"]), ref["codes"])
    assert np.array_equal(host(got["scales"]), ref["scales"])
    assert q.qfp4_last_device_error() == 0
