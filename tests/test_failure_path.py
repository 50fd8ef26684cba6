"""The bounded-wait failure path on the GPU, without a fault: a grid wait
that one block never joins gives up after 10 ms, the host reads
SHARQ_ERR_TIMEOUT from the status word (then OK once it is cleared), and
the context keeps working (a prepare afterwards is still bit-exact)."""
import numpy as np
import pytest
import torch

import activation_sparsity_prep_b200 as sq
from activation_sparsity_prep_b200 import workloads as wl
import oracle
from tests.sharq_testlib import to_dev, to_np

pytestmark = pytest.mark.gpu

TIMEOUT = 4     # SHARQ_ERR_TIMEOUT


def test_lost_block_times_out_and_the_context_survives():
    sq.last_device_status()                      # start from a cleared status word
    sq.selftest_wait_timeout(10000)
    assert sq.last_device_status() == TIMEOUT
    assert sq.last_device_status() == 0          # read and cleared
    X = wl.activation("laplace_outlier", 61, 0, 33, 512)
    P = sq.prepare(to_dev(X), None, 1e-6)
    torch.cuda.synchronize()
    assert sq.last_device_status() == 0
    R = oracle.prepare(X, None, 1e-6)
    assert np.array_equal(to_np(P.bb_codes), R.bb.codes)
    assert np.array_equal(to_np(P.rs_codes), R.rs.codes)
