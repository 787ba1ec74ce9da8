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
                                 (257, 4097), (130, 8192), (64, 12345), (5, 129), (100, 576),
                                 (300, 2100), (301, 2400), (77, 3100)])
def test_ragged_shapes(N, K, dtype):
    W = workloads.normal((N, K), 0.02, N + K)
    x = workloads.random_with_edges(1, K, seed=K, dtype=dtype)[0]
    y_i, y_f = run_gemv(W, x)
    s_ref, y_ref = reference(W, x)
    assert np.array_equal(y_i.cpu().numpy(), s_ref)
    assert_scaled_close(y_f, y_ref)


@pytest.mark.parametrize("flags", [0, 1, 3, 7])
@pytest.mark.parametrize("K", [2100, 2400, 3100, 4096])
def test_row128_kernel_every_block_shape(K, flags):
    """The one-chunk-per-lane kernel takes rows of 68..128 words; with bf16 x
    its pack covers 4 vectors per word, so kw * 4 vectors need not fill whole
    warps (K = 2100, 2400, 3100).  Every dependency mode (each has its own
    block shape) must give the exact product there."""
    N = 1234
    d = dev()
    W = workloads.normal((N, K), 0.02, 3 * K + flags)
    x = workloads.random_with_edges(1, K, seed=K + 1, dtype=torch.bfloat16)[0]
    W_p = bnn.empty_packed(N, K, d)
    alpha = torch.empty(N, dtype=torch.float32, device=d)
    bnn.bnn_pack_sign(W.to(d), W_p, alpha)
    y_i = torch.empty(N, dtype=torch.int32, device=d)
    y_f = torch.empty(N, dtype=torch.float32, device=d)
    bnn.bnn_xnor_gemv_ex(W_p, x.to(d), K, alpha, y_i, y_f, flags=flags)
    torch.cuda.synchronize()
    s_ref, y_ref = reference(W, x)
    assert np.array_equal(y_i.cpu().numpy(), s_ref)
    assert_scaled_close(y_f, y_ref)
    assert_no_device_error()


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


def _chain_reference(Ws, x0):
    """Oracle chain: x_{l+1} = alpha_l * s_l (float64), s_l from sign(W_l), sign(x_l)."""
    x = np.asarray(x0, dtype=np.float64)
    out = []
    for W in Ws:
        s = oracle.gemv_pm1(oracle.sign_pm1(W), oracle.sign_pm1(x.astype(np.float32)))
        y = oracle.scaled(s, oracle.alpha(W))
        out.append((s, y))
        x = y
    return out


@pytest.mark.parametrize("use_graph", [False, True])
def test_static_weights_chain_orders_dependent_gemvs(use_graph):
    """Eight GEMVs back to back on one stream with BNN_GEMV_WEIGHTS_STATIC,
    each reading the previous one's fp32 output as its x: the dependency wait
    must order every read of x after the previous kernel's writes."""
    D, L = 4096, 8
    d = dev()
    Ws = [workloads.normal((D, D), 1.0, 500 + l) for l in range(L)]
    x0 = workloads.normal((D,), 1.0, 499)
    Wp, al = [], []
    for W in Ws:
        p = bnn.empty_packed(D, D, d)
        a = torch.empty(D, dtype=torch.float32, device=d)
        bnn.bnn_pack_sign(W.to(d), p, a)
        Wp.append(p)
        al.append(a)
    xs = [x0.to(d)] + [torch.empty(D, dtype=torch.float32, device=d) for _ in range(L)]
    ys = [torch.empty(D, dtype=torch.int32, device=d) for _ in range(L)]
    torch.cuda.synchronize()

    def chain():
        for l in range(L):
            bnn.bnn_xnor_gemv_ex(Wp[l], xs[l], D, al[l], ys[l], xs[l + 1], flags=bnn.BNN_GEMV_WEIGHTS_STATIC)

    if use_graph:
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            chain()
        torch.cuda.current_stream().wait_stream(s)
        for t in xs[1:]:
            t.fill_(float("nan"))
        with torch.cuda.graph(g):
            chain()
        for t in xs[1:]:
            t.fill_(float("nan"))
        g.replay()
    else:
        chain()
    torch.cuda.synchronize()
    ref = _chain_reference(Ws, x0.numpy())
    for l in range(L):
        assert np.array_equal(ys[l].cpu().numpy(), ref[l][0]), f"layer {l}"
        assert_scaled_close(xs[l + 1], ref[l][1])
    assert_no_device_error()


def test_gemv_ex_rejects_unknown_flags():
    W = bnn.empty_packed(8, 64, dev())
    x = torch.zeros(64, device=dev())
    y = torch.empty(8, dtype=torch.int32, device=dev())
    with pytest.raises(bnn.BnnError):
        bnn.bnn_xnor_gemv_ex(W, x, 64, None, y, None, flags=8)


@pytest.mark.parametrize("use_graph", [False, True])
def test_static_inputs_independent_gemvs(use_graph):
    """BNN_GEMV_WEIGHTS_STATIC | BNN_GEMV_INPUTS_STATIC on independent GEMVs
    over resident inputs: each result exact; consecutive calls that write the
    same y keep stream order (the last call's values remain)."""
    N, K, L = 1000, 4000, 6
    d = dev()
    Ws = [workloads.normal((N, K), 1.0, 700 + l) for l in range(L)]
    xs = [workloads.normal((K,), 1.0, 800 + l, dtype=torch.bfloat16) for l in range(L)]
    Wp, al = [], []
    for W in Ws:
        p = bnn.empty_packed(N, K, d)
        a = torch.empty(N, dtype=torch.float32, device=d)
        bnn.bnn_pack_sign(W.to(d), p, a)
        Wp.append(p)
        al.append(a)
    xd = [x.to(d) for x in xs]
    ys = [torch.empty(N, dtype=torch.int32, device=d) for _ in range(L)]
    y_shared = torch.empty(N, dtype=torch.int32, device=d)
    flags = bnn.BNN_GEMV_WEIGHTS_STATIC | bnn.BNN_GEMV_INPUTS_STATIC
    torch.cuda.synchronize()

    def run():
        for l in range(L):
            bnn.bnn_xnor_gemv_ex(Wp[l], xd[l], K, al[l], ys[l], None, flags=flags)
        for l in range(L):
            bnn.bnn_xnor_gemv_ex(Wp[l], xd[l], K, al[l], y_shared, None, flags=flags)

    if use_graph:
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            run()
        torch.cuda.current_stream().wait_stream(s)
        with torch.cuda.graph(g):
            run()
        for t in ys + [y_shared]:
            t.fill_(-7)
        g.replay()
    else:
        run()
    torch.cuda.synchronize()
    for l in range(L):
        ref = oracle.gemv_pm1(oracle.sign_pm1(Ws[l]), oracle.sign_pm1(xs[l]))
        assert np.array_equal(ys[l].cpu().numpy(), ref), f"gemv {l}"
    assert torch.equal(y_shared, ys[L - 1])
    assert_no_device_error()


@pytest.mark.parametrize("use_graph", [False, True])
def test_independent_gemvs_all_flags(use_graph):
    """All three flags on GEMVs over distinct resident inputs and distinct
    outputs: they may run concurrently; every result exact, and a kernel
    queued after them (a torch copy) sees all of them finished."""
    N, K, L = 777, 4096, 8
    d = dev()
    Ws = [workloads.normal((N, K), 1.0, 900 + l) for l in range(L)]
    xs = [workloads.normal((K,), 1.0, 950 + l, dtype=torch.bfloat16) for l in range(L)]
    Wp, al = [], []
    for W in Ws:
        p = bnn.empty_packed(N, K, d)
        a = torch.empty(N, dtype=torch.float32, device=d)
        bnn.bnn_pack_sign(W.to(d), p, a)
        Wp.append(p)
        al.append(a)
    xd = [x.to(d) for x in xs]
    ys = [torch.empty(N, dtype=torch.int32, device=d) for _ in range(L)]
    yf = [torch.empty(N, dtype=torch.float32, device=d) for _ in range(L)]
    flags = bnn.BNN_GEMV_WEIGHTS_STATIC | bnn.BNN_GEMV_INPUTS_STATIC | bnn.BNN_GEMV_OUTPUT_FREE
    torch.cuda.synchronize()

    def run():
        for l in range(L):
            bnn.bnn_xnor_gemv_ex(Wp[l], xd[l], K, al[l], ys[l], yf[l], flags=flags)
        return torch.stack(ys)

    if use_graph:
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            run()
        torch.cuda.current_stream().wait_stream(s)
        with torch.cuda.graph(g):
            stacked = run()
        for t in ys:
            t.fill_(-7)
        g.replay()
    else:
        stacked = run()
    torch.cuda.synchronize()
    for l in range(L):
        wb, xb = oracle.sign_pm1(Ws[l]), oracle.sign_pm1(xs[l])
        ref = oracle.gemv_pm1(wb, xb)
        assert np.array_equal(ys[l].cpu().numpy(), ref), f"gemv {l}"
        assert np.array_equal(stacked[l].cpu().numpy(), ref), f"stacked {l}"
        assert_scaled_close(yf[l], oracle.scaled(ref, oracle.alpha(Ws[l])))
    assert_no_device_error()


@pytest.mark.parametrize("pin_x,pin_y", [(True, True), (False, False), (True, False), (False, True)],
                         ids=["pinned", "pageable", "pinned_x", "pinned_y"])
@pytest.mark.parametrize("N,K,x_dt", [(3000, 4096, torch.bfloat16), (3001, 4095, torch.bfloat16),
                                      (11008, 4096, torch.bfloat16), (517, 1000, torch.float32)])
@pytest.mark.parametrize("flags", [bnn.BNN_GEMV_WEIGHTS_STATIC,
                                   bnn.BNN_GEMV_WEIGHTS_STATIC | bnn.BNN_GEMV_INPUTS_STATIC], ids=["w", "wx"])
def test_host_buffer_entry_matches_device_gemv(pin_x, pin_y, N, K, x_dt, flags):
    """bnn_xnor_gemv_host (x and y in host memory, copies inside the call)
    gives the same y as bnn_xnor_gemv on device buffers, bit for bit, on two
    calls in a row with different x.  Pinned x and y with 16-byte multiples
    take the kernel copies over PCIe; pageable buffers, odd byte counts
    (K = 4095 bf16, N = 3001 or 517) take the copy engines."""
    d = dev()
    W = workloads.normal((N, K), 0.02, 91)
    W_p = bnn.empty_packed(N, K, d)
    alpha = torch.empty(N, dtype=torch.float32, device=d)
    bnn.bnn_pack_sign(W.to(d), W_p, alpha)
    x_dev = torch.empty(K, dtype=x_dt, device=d)
    y_dev = torch.empty(N, dtype=torch.float32, device=d)
    for seed in (92, 93):
        x = workloads.normal((K,), 1.0, seed, dtype=x_dt)
        x_host = x.pin_memory() if pin_x else x.clone()
        y_host = torch.full((N,), float("nan"), dtype=torch.float32)
        if pin_y:
            y_host = y_host.pin_memory()
        bnn.bnn_xnor_gemv_host(W_p, x_host, K, alpha, x_dev, y_dev, y_host, flags=flags)
        torch.cuda.synchronize()
        y_ref = torch.empty(N, dtype=torch.float32, device=d)
        bnn.bnn_xnor_gemv(W_p, x.to(d), K, alpha, None, y_ref)
        assert torch.equal(y_host, y_ref.cpu())
    assert_no_device_error()


@pytest.mark.parametrize("flags", [bnn.BNN_GEMV_WEIGHTS_STATIC,
                                   bnn.BNN_GEMV_WEIGHTS_STATIC | bnn.BNN_GEMV_INPUTS_STATIC], ids=["w", "wx"])
def test_host_buffer_entry_chained_steps(flags):
    """Twelve host-buffer calls enqueued back to back with no host
    synchronisation (the kernel copies chained by programmatic dependent
    launch), each with its own pinned x and y and the shared device scratch:
    every y equals the device GEMV of its own x, so no step's copy overtook
    the previous step's use of the scratch."""
    N, K, steps = 11008, 4096, 12
    d = dev()
    W = workloads.normal((N, K), 0.02, 95)
    W_p = bnn.empty_packed(N, K, d)
    alpha = torch.empty(N, dtype=torch.float32, device=d)
    bnn.bnn_pack_sign(W.to(d), W_p, alpha)
    xs = [workloads.normal((K,), 1.0, 200 + i, dtype=torch.bfloat16) for i in range(steps)]
    x_hosts = [x.pin_memory() for x in xs]
    y_hosts = [torch.full((N,), float("nan"), dtype=torch.float32).pin_memory() for _ in range(steps)]
    x_dev = torch.empty(K, dtype=torch.bfloat16, device=d)
    y_dev = torch.empty(N, dtype=torch.float32, device=d)
    torch.cuda.synchronize()
    for i in range(steps):
        bnn.bnn_xnor_gemv_host(W_p, x_hosts[i], K, alpha, x_dev, y_dev, y_hosts[i], flags=flags)
    torch.cuda.synchronize()
    for i in range(steps):
        y_ref = torch.empty(N, dtype=torch.float32, device=d)
        bnn.bnn_xnor_gemv(W_p, xs[i].to(d), K, alpha, None, y_ref)
        assert torch.equal(y_hosts[i], y_ref.cpu()), f"step {i}"
    assert_no_device_error()
