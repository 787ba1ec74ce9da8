"""Failure detection on the GPU without a fault: a bounded mbarrier wait that
nothing satisfies gives up after a short limit, reports
BNN_ERR_DEVICE_TIMEOUT through the device-side flag, and leaves the CUDA
context usable (a product computed afterwards is still exact)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import xnor_popcount_gemm_bnn_b200 as bnn
from gpu_util import dev

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    assert bnn.bnn_device_error() == 0                    # clean start (and clears any stale flag)
    assert bnn.bnn_selftest_wait_timeout(20_000_000)      # 20 ms limit: the wait must run out
    assert bnn.bnn_device_error() == bnn.BNN_ERR_DEVICE_TIMEOUT
    assert bnn.bnn_device_error() == 0                    # reading clears the flag
    # The context still works: a small product after the time-out is exact.
    X = workloads.normal((70, 300), 1.0, 5)
    W = workloads.normal((90, 300), 1.0, 6)
    A_p = bnn.empty_packed(70, 300, dev())
    W_p = bnn.empty_packed(90, 300, dev())
    bnn.bnn_pack_sign(X.to(dev()), A_p)
    bnn.bnn_pack_sign(W.to(dev()), W_p)
    C = torch.empty(70, 90, dtype=torch.int32, device=dev())
    bnn.bnn_xnor_gemm(A_p, W_p, 300, None, C)
    s_ref, _ = oracle.binary_linear(X, W)
    assert np.array_equal(C.cpu().numpy(), s_ref)
    assert bnn.bnn_device_error() == 0


def test_selftest_rejects_bad_limits():
    with pytest.raises(bnn.BnnError):
        bnn.bnn_selftest_wait_timeout(0)
