"""Batch-1 binary GEMV (x packed inside the kernel) against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import xnor_popcount_gemm_bnn_b200 as bnn
from gpu_util import assert_no_device_error, assert_scaled_close, dev

pytestmark = pytest.mark.gpu


def run_gemv(W, x, with_f32=True):
    d = dev()
    N, K = W.shape
    W_p = bnn.empty_packed(N, K, d)
    alpha = torch.empty(N, dtype=torch.float32, device=d)
    bnn.bnn_pack_sign(W.to(d), W_p, alpha)
    y_i = torch.empty(N, dtype=torch.int32, device=d)
    y_f = torch.empty(N, dtype=torch.float32, device=d) if with_f32 else None
    bnn.bnn_xnor_gemv(W_p, x.to(d), K, alpha, y_i, y_f)
    return y_i, y_f


def reference(W, x):
    s = oracle.gemv_pm1(oracle.sign_pm1(W), oracle.sign_pm1(x))
    return s, oracle.scaled(s, oracle.alpha(W))


def test_llm_decode_workload():
    """W [11008, 4096] packed from N(0, 0.02), x bf16 [4096] N(0, 1)."""
    g = workloads.gemv()
    y_i, y_f = run_gemv(g.W, g.x)
    s_ref, y_ref = reference(g.W, g.x)
    assert np.array_equal(y_i.cpu().numpy(), s_ref)
    assert_scaled_close(y_f, y_ref)
    assert_no_device_error()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("N,K", [(1, 1), (7, 31), (33, 100), (1000, 1000), (300, 4095),
                                 (257, 4097), (130, 8192), (64, 12345), (5, 129), (100, 576)])
def test_ragged_shapes(N, K, dtype):
    W = workloads.normal((N, K), 0.02, N + K)
    x = workloads.random_with_edges(1, K, seed=K, dtype=dtype)[0]
    y_i, y_f = run_gemv(W, x)
    s_ref, y_ref = reference(W, x)
    assert np.array_equal(y_i.cpu().numpy(), s_ref)
    assert_scaled_close(y_f, y_ref)


def test_int32_only_and_f32_only():
    W = workloads.normal((500, 2048), 1.0, 1)
    x = workloads.normal((2048,), 1.0, 2)
    d = dev()
    W_p = bnn.empty_packed(500, 2048, d)
    alpha = torch.empty(500, dtype=torch.float32, device=d)
    bnn.bnn_pack_sign(W.to(d), W_p, alpha)
    s_ref, y_ref = reference(W, x)
    y_i = torch.empty(500, dtype=torch.int32, device=d)
    bnn.bnn_xnor_gemv(W_p, x.to(d), 2048, None, y_i, None)
    assert np.array_equal(y_i.cpu().numpy(), s_ref)
    y_f = torch.empty(500, dtype=torch.float32, device=d)
    bnn.bnn_xnor_gemv(W_p, x.to(d), 2048, alpha, None, y_f)
    assert_scaled_close(y_f, y_ref)


def test_gemv_equals_gemm_row():
    """The GEMV of x equals the GEMM row of the same packed x."""
    N, K = 777, 3000
    W = workloads.normal((N, K), 1.0, 9)
    x = workloads.normal((K,), 1.0, 10)
    d = dev()
    W_p = bnn.empty_packed(N, K, d)
    bnn.bnn_pack_sign(W.to(d), W_p)
    x_p = bnn.empty_packed(1, K, d)
    bnn.bnn_pack_sign(x.to(d).view(1, -1), x_p)
    y_g = torch.empty(1, N, dtype=torch.int32, device=d)
    bnn.bnn_xnor_gemm(x_p, W_p, K, None, y_g)
    y_v = torch.empty(N, dtype=torch.int32, device=d)
    bnn.bnn_xnor_gemv(W_p, x.to(d), K, None, y_v)
    assert torch.equal(y_g[0], y_v)
