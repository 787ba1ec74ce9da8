"""Binary weights x real activations GEMV ("Extreme Quantization ...", Binary
Neural Networks, eq. (1)-(2)) against the oracle's float64 add/sub sum.

Tolerance, derived from the kernel's fp32 arithmetic (u = 2^-24): a table
entry +-x0 +-x1 +-x2 +-x3 takes 3 roundings; a lane sums the 32 groups of
each of its P = ceil(kw/128) chunks on 4 accumulators (8P - 1 roundings
each), the 4 meet in a 2-level tree, and the lanes of a row meet in a
butterfly of at most 5 levels; alpha*s is one multiplication.  That is at
most 8P + 10 roundings on the path of every term, which the bound below,
(ceil(K/256) + 20) roundings of alpha * sum|x|, covers at every K (P = 1 for
K <= 4096, where the bound's count is at least 21; P = 2 needs K > 4096, count
>= 37; P = 3 needs K > 8192, count >= 53).  So |y - y_ref| <= alpha *
(ceil(K/256) + 20) * u * sum|x| + 2u * |y_ref| (the second term also covers
alpha rounded to fp32)."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
import xnor_popcount_gemm_bnn_b200 as bnn
from gpu_util import assert_no_device_error, dev

pytestmark = pytest.mark.gpu

U = 2.0 ** -24


def check(y, W, x, K):
    a, y_ref = oracle.binary_weight_gemv(W, x)
    sx = np.abs(oracle._f32(x).astype(np.float64)).sum()
    tol = a * (math.ceil(K / 256) + 20) * U * sx * 1.05 + 2 * U * np.abs(y_ref) * 1.05
    err = np.abs(y.detach().cpu().numpy().astype(np.float64) - y_ref)
    bad = np.nonzero(err > tol)[0]
    assert bad.size == 0, f"{bad.size} rows outside the bound, first {bad[:5]}: err {err[bad[:5]]} tol {tol[bad[:5]]}"


def run(W, x, K, flags=0):
    d = dev()
    N = W.shape[0]
    Wp = bnn.empty_packed(N, K, d)
    al = torch.empty(N, dtype=torch.float32, device=d)
    bnn.bnn_pack_sign(W.to(d), Wp, al)
    y = torch.full((N,), float("nan"), dtype=torch.float32, device=d)
    bnn.bnn_binary_weight_gemv(Wp, x.to(d), K, al, y, flags=flags)
    torch.cuda.synchronize()
    return y


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("N,K", [(1, 1), (5, 31), (64, 1000), (65, 33), (300, 4096), (100, 4100),
                                 (129, 8192), (33, 12288)])
@pytest.mark.parametrize("flags", [0, 3, 7])
def test_bw_gemv_shapes(N, K, dtype, flags):
    W = workloads.normal((N, K), 1.0, N + K)
    x = workloads.normal((K,), 1.0, K + 7, dtype=dtype)
    y = run(W, x, K, flags)
    check(y, W, x, K)
    assert_no_device_error()


def test_bw_gemv_decode_workload():
    """The decode shape: W [11008, 4096] ~ N(0, 0.02) (the GEMV workload's
    weights), x bf16 [4096] ~ N(0, 1) used as a real activation."""
    g = workloads.gemv()
    y = run(g.W, g.x, g.K, flags=bnn.BNN_GEMV_WEIGHTS_STATIC)
    check(y, g.W, g.x, g.K)
    assert_no_device_error()


def test_bw_gemv_special_values():
    """Signed zeros and exact halves of x: every term is exact, and a +1/-1 x
    reduces to the binary product (K - 2 popcount)."""
    K, N = 256, 40
    W = workloads.normal((N, K), 1.0, 5)
    xb = torch.where(workloads.normal((K,), 1.0, 6) < 0, -1.0, 1.0)
    y = run(W, xb, K)
    s_ref = oracle.gemv_pm1(oracle.sign_pm1(W), oracle.sign_pm1(xb))
    a = oracle.alpha(W)
    assert np.allclose(y.cpu().numpy(), a * s_ref, rtol=4 * U, atol=0)
    x0 = torch.zeros(K)
    x0[::2] = -0.0
    y0 = run(W, x0, K)
    assert torch.count_nonzero(y0) == 0


def test_bw_gemv_store_order_and_independent_calls():
    """BNN_GEMV_WEIGHTS_STATIC | BNN_GEMV_INPUTS_STATIC: consecutive calls
    that write one y keep stream order; with all three flags, calls over
    separate outputs are each exact."""
    d = dev()
    N, K, L = 500, 2048, 5
    Ws = [workloads.normal((N, K), 1.0, 40 + l) for l in range(L)]
    xs = [workloads.normal((K,), 1.0, 50 + l, dtype=torch.bfloat16) for l in range(L)]
    Wp, al = [], []
    for W in Ws:
        p = bnn.empty_packed(N, K, d)
        a = torch.empty(N, dtype=torch.float32, device=d)
        bnn.bnn_pack_sign(W.to(d), p, a)
        Wp.append(p)
        al.append(a)
    xd = [x.to(d) for x in xs]
    ys = [torch.empty(N, dtype=torch.float32, device=d) for _ in range(L)]
    shared = torch.empty(N, dtype=torch.float32, device=d)
    torch.cuda.synchronize()
    for l in range(L):
        bnn.bnn_binary_weight_gemv(Wp[l], xd[l], K, al[l], ys[l], flags=7)
    for l in range(L):
        bnn.bnn_binary_weight_gemv(Wp[l], xd[l], K, al[l], shared, flags=3)
    torch.cuda.synchronize()
    for l in range(L):
        check(ys[l], Ws[l], xs[l], K)
    assert torch.equal(shared, ys[L - 1])
    assert_no_device_error()


# ---------------------------------------------------------------------------
# binary weights x INT8 activations (BitNet section: INT8 activations; eq. (1)
# per-row alpha, eq. (8) one alpha for the matrix).  acc is exact; y_f32 takes
# three roundings: fp32(alpha), fp32(alpha * x_scale), the product with
# fp32(acc) -- |y - y_ref| <= 4u |y_ref| covers them with the fp32 alpha used.
# ---------------------------------------------------------------------------

def run_i8(W, xq, K, per_row=True, flags=0, x_scale=0.03125, x_dev=None):
    d = dev()
    N = W.shape[0]
    Wp = bnn.empty_packed(N, K, d)
    al = torch.empty(N, dtype=torch.float32, device=d)
    bnn.bnn_pack_sign(W.to(d), Wp, al)
    if not per_row:
        al = torch.tensor([oracle.ternary_gamma(W)], dtype=torch.float32, device=d)
    xs = torch.tensor([x_scale], dtype=torch.float32, device=d)
    yi = torch.full((N,), -7, dtype=torch.int32, device=d)
    yf = torch.full((N,), float("nan"), dtype=torch.float32, device=d)
    bnn.bnn_binary_weight_gemv_i8(Wp, xq.to(d) if x_dev is None else x_dev, K, al, xs, yi, yf, flags=flags)
    torch.cuda.synchronize()
    return yi, yf, al.cpu().numpy().astype(np.float64)


def check_i8(yi, yf, W, xq, alpha_used, x_scale=0.03125):
    acc = oracle.binary_weight_product(oracle.sign_pm1(W), xq.numpy().astype(np.float64))
    assert np.array_equal(yi.cpu().numpy().astype(np.float64), acc)
    a = alpha_used if alpha_used.size == acc.size else np.full(acc.size, alpha_used[0])
    y_ref = a * x_scale * acc
    err = np.abs(yf.cpu().numpy().astype(np.float64) - y_ref)
    assert np.all(err <= 4 * U * np.abs(y_ref)), f"max rel err {np.max(err / np.maximum(np.abs(y_ref), 1e-300))}"


@pytest.mark.parametrize("N,K", [(1, 1), (5, 31), (64, 1000), (65, 33), (300, 4096), (100, 4100), (129, 8192),
                                 (33, 12288), (7, 49152), (1000, 2100)])
@pytest.mark.parametrize("flags", [0, 1, 3, 7])
def test_bw_gemv_i8_shapes(N, K, flags):
    W = workloads.normal((N, K), 1.0, 3 * N + K)
    xq = workloads.int8_uniform((K,), K + 11)
    yi, yf, a = run_i8(W, xq, K, flags=flags)
    check_i8(yi, yf, W, xq, a)
    assert_no_device_error()


def test_bw_gemv_i8_decode_workload():
    """The decode shape: packed W [11008, 4096] from N(0, 0.02), x int8 [4096]."""
    g, t = workloads.gemv(), workloads.ternary()
    yi, yf, a = run_i8(g.W, t.x, g.K, flags=bnn.BNN_GEMV_WEIGHTS_STATIC)
    check_i8(yi, yf, g.W, t.x, a)
    assert_no_device_error()


def test_bw_gemv_i8_one_alpha_for_the_matrix():
    """eq. (8): one scale ||W||_1 / (n m) for every row."""
    N, K = 777, 3000
    W = workloads.normal((N, K), 0.5, 91)
    xq = workloads.int8_uniform((K,), 92)
    yi, yf, a = run_i8(W, xq, K, per_row=False)
    assert a.size == 1
    check_i8(yi, yf, W, xq, a)


def test_bw_gemv_i8_extremes_and_unaligned_x():
    """x = -128 everywhere and W all +1 / all -1 rows: |acc| = 128 K; x read
    from an unaligned address takes the byte path."""
    N, K = 64, 4096
    W = torch.ones(N, K)
    W[1::2] = -1.0
    xq = torch.full((K,), -128, dtype=torch.int8)
    yi, yf, a = run_i8(W, xq, K)
    check_i8(yi, yf, W, xq, a)
    assert int(yi[0]) == -128 * K and int(yi[1]) == 128 * K
    xq2 = workloads.int8_uniform((K,), 5)
    buf = torch.zeros(K + 1, dtype=torch.int8, device=dev())
    buf[1:] = xq2.to(dev())
    W2 = workloads.normal((N, K), 1.0, 6)
    yi2, yf2, a2 = run_i8(W2, xq2, K, x_dev=buf[1:])
    check_i8(yi2, yf2, W2, xq2, a2)
    assert_no_device_error()
