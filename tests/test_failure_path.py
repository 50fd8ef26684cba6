"""The bounded-wait failure path on the GPU, without a fault.

* The library's own wait helpers (the grid barrier and the mbarrier wait the
  prepare and linear kernels call) run into a 10 ms limit: a grid barrier
  that one block never arrives at, an mbarrier phase nothing completes.
* The shipped prepare kernel itself, launched with one block that never
  arrives at its two grid barriers and a 10 ms limit per wait: the other
  blocks give up, record the timeout and run to their end.
In both cases the host reads SHARQ_ERR_TIMEOUT from the status word (then
OK once it is cleared), and the context keeps working: a prepare afterwards
is still bit-exact against the oracle."""
import time

import numpy as np
import pytest
import torch

import activation_sparsity_prep_b200 as sq
from activation_sparsity_prep_b200 import workloads as wl
import oracle
from tests.sharq_testlib import to_dev, to_np

pytestmark = pytest.mark.gpu

TIMEOUT = 4     # SHARQ_ERR_TIMEOUT


def _prepare_still_bit_exact(seed):
    X = wl.activation("laplace_outlier", seed, 0, 33, 512)
    P = sq.prepare(to_dev(X), None, 1e-6)
    torch.cuda.synchronize()
    assert sq.last_device_status() == 0
    R = oracle.prepare(X, None, 1e-6)
    assert np.array_equal(to_np(P.bb_codes), R.bb.codes)
    assert np.array_equal(to_np(P.rs_codes), R.rs.codes)


def test_wait_helpers_time_out_and_the_context_survives():
    sq.last_device_status()                      # start from a cleared status word
    sq.selftest_wait_timeout(10000)
    assert sq.last_device_status() == TIMEOUT
    assert sq.last_device_status() == 0          # read and cleared
    _prepare_still_bit_exact(61)


@pytest.mark.parametrize("M,K", [(33, 512), (4096, 4096)])
def test_prepare_with_a_lost_block_times_out(M, K):
    """A real prepare launch (one block, or a full grid of 296) whose block 0
    skips both barrier arrivals: bounded by two 10 ms waits, not a hang."""
    X = to_dev(wl.activation("laplace_outlier", 62, M, M, K))
    sq.last_device_status()
    t0 = time.perf_counter()
    sq.selftest_prepare_timeout(X, 10000)
    assert sq.last_device_status() == TIMEOUT
    assert time.perf_counter() - t0 < 5.0
    assert sq.last_device_status() == 0
    _prepare_still_bit_exact(63)
