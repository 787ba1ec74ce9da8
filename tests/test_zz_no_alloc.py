"""The allocation-free ternary pack, bnn_ternary_pack_noalloc.

Some callers of this library cannot allocate device memory: code that only
receives input and output pointers from a host framework (a plugin or custom
operator of another runtime) and latency-critical paths that must not call
cudaMalloc.  bnn_ternary_pack needs a scratch workspace for gamma's row sums;
its no-alloc twin keeps that scratch in a device array owned by the library.
These tests call it through the C ABI and check that it gives exactly what the
workspace entry point gives (the codes bit for bit, gamma to the same fp32
value): twice in a row on the same inputs, then on a different matrix, since
the shared array keeps the previous call's contents.

This file is named so that pytest collects it last."""
import ctypes

import numpy as np
import pytest
import torch

import workloads
import xnor_popcount_gemm_bnn_b200 as bnn


def test_noalloc_rejects_too_many_rows_on_the_host():
    """Beyond the array's capacity the call fails before touching the GPU."""
    fake = ctypes.c_void_p(0x10000)
    rows = bnn.BNN_TERNARY_PACK_NOALLOC_MAX_ROWS + 1
    st = bnn.lib.bnn_ternary_pack_noalloc(fake, bnn.BNN_F32, rows, 64, 64, -1.0, fake, 4, None, None)
    assert st == bnn.BNN_ERR_UNSUPPORTED


def _reference(Wd, delta):
    codes = bnn.empty_ternary(Wd.shape[0], Wd.shape[1], Wd.device)
    g = torch.empty(1, dtype=torch.float32, device=Wd.device)
    bnn.bnn_ternary_pack(Wd, codes, gamma_out=g, delta=delta)
    return codes, g


@pytest.mark.gpu
@pytest.mark.parametrize("delta", [None, 0.01])
def test_noalloc_matches_workspace_entry_point(delta):
    d = torch.device("cuda", 0)
    W1 = workloads.normal((1000, 4096), 0.02, 71).to(d)
    W2 = workloads.normal((37, 1000), 1.0, 72).to(torch.bfloat16).to(d)
    ref1 = _reference(W1, delta)
    ref2 = _reference(W2, delta)
    torch.cuda.synchronize()
    for W, (rc, rg) in ((W1, ref1), (W1, ref1), (W2, ref2)):
        codes = torch.full_like(rc, 0x2468ACE)
        g = torch.full((1,), float("nan"), dtype=torch.float32, device=d)
        bnn.bnn_ternary_pack_noalloc(W, codes, gamma_out=g, delta=delta)
        torch.cuda.synchronize()
        assert torch.equal(codes, rc)
        assert np.float32(g.item()) == np.float32(rg.item())
    assert bnn.bnn_device_error() == bnn.BNN_OK
