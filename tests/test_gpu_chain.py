"""The batch-1 binary layer chain in one launch (bnn_xnor_gemv_chain) against
the oracle's fully binary MLP forward at batch 1 (sign, +1/-1 products,
BatchNorm evaluated directly in double, alpha * s at the end): every hidden
layer's packed bits bit-exact, the last layer's int32 s exact and alpha * s
within 1e-6 relative."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import xnor_popcount_gemm_bnn_b200 as bnn
from gpu_util import assert_no_device_error, assert_scaled_close, dev, u32

pytestmark = pytest.mark.gpu


def gpu_layers(c: workloads.Chain):
    """Pack every layer's weights (alpha from the pack) and fold each hidden
    layer's BatchNorm into popcount thresholds on the host."""
    d = dev()
    layers = []
    L = len(c.Ws)
    for l, W in enumerate(c.Ws):
        N, K = W.shape
        Wp = bnn.empty_packed(N, K, d)
        alpha = torch.empty(N, dtype=torch.float32, device=d)
        bnn.bnn_pack_sign(W.to(d), Wp, alpha)
        if l < L - 1:
            bn = c.bns[l]
            thr, mode = bnn.bnn_fold_bn_threshold(alpha.cpu(), bn.gamma, bn.beta, bn.mean, bn.var, bn.eps, K)
            layers.append({"W": Wp, "popc_thresh": thr.to(d), "thresh_mode": mode.to(d)})
        else:
            layers.append({"W": Wp, "alpha": alpha})
    return layers


def run_chain(c: workloads.Chain, layers=None, ws=None, x=None):
    d = dev()
    layers = gpu_layers(c) if layers is None else layers
    ws = bnn.gemv_chain_workspace(d) if ws is None else ws
    x = c.x0.to(d) if x is None else x
    hidden = [w.shape[0] for w in c.Ws[:-1]]
    acts = None
    if hidden:
        ld = max(bnn.bnn_packed_ld_words(n) for n in hidden)
        acts = torch.full((len(hidden), ld), -1, dtype=torch.int32, device=d)
    n_out = c.Ws[-1].shape[0]
    y_i32 = torch.full((n_out,), 12345, dtype=torch.int32, device=d)
    y_f32 = torch.full((n_out,), float("nan"), dtype=torch.float32, device=d)
    bnn.bnn_xnor_gemv_chain(layers, x, ws, y_i32=y_i32, y_f32=y_f32, acts=acts)
    torch.cuda.synchronize()
    return acts, y_i32, y_f32


def oracle_chain(c: workloads.Chain):
    bns = [(b.gamma.numpy(), b.beta.numpy(), b.mean.numpy(), b.var.numpy(), b.eps) for b in c.bns]
    acts, logits = oracle.mlp_forward(c.x0, c.Ws, bns)
    s_last = oracle.matmul_pm1(acts[-1], oracle.sign_pm1(c.Ws[-1]))[0]
    return acts, s_last, logits[0]


def check(c: workloads.Chain, acts, y_i32, y_f32):
    acts_ref, s_ref, logits_ref = oracle_chain(c)
    for l in range(1, len(acts_ref)):
        ref = oracle.pack_pm1(acts_ref[l])[0]
        got = u32(acts[l - 1])[: ref.size]
        assert np.array_equal(got, ref), f"layer {l} input bits"
    assert np.array_equal(y_i32.cpu().numpy(), s_ref.astype(np.int32))
    assert_scaled_close(y_f32, logits_ref)
    assert_no_device_error()


CASES = [
    # K0, widths, x dtype
    (1000, (256, 300, 77, 33), torch.bfloat16),          # ragged words everywhere
    (1000, (256, 300, 77, 33), torch.float32),
    (1000, (300,), torch.float32),                       # one layer: a plain GEMV
    (4096, (11008, 4096), torch.bfloat16),               # one up / down pair
    (100, (64, 96, 33, 200, 64, 500, 31, 40, 70, 130, 65, 17), torch.bfloat16),  # slot buffers reused
    (16384, (1000, 16384, 50), torch.float32),           # rows of 512 words (4 vectors per lane)
    (33, (100, 33, 64), torch.float32),                  # one 16-byte vector per row: 32 rows per warp load
    (512, (4096, 100000), torch.bfloat16),               # last layer of several batches per warp
    (8192, (16384, 8192, 16384, 100), torch.bfloat16),   # hidden layers of several batches per warp
]


@pytest.mark.parametrize("K0,widths,xdt", CASES, ids=[f"K{c[0]}-L{len(c[1])}-{str(c[2])[6:]}" for c in CASES])
def test_chain_matches_oracle(K0, widths, xdt):
    c = workloads.chain(widths=widths, K0=K0, x_dtype=xdt)
    check(c, *run_chain(c))


def test_chain_decode_workload():
    """The decode-shaped chain: 8 layers alternating [11008, 4096] and
    [4096, 11008], bf16 x; every hidden activation and all outputs."""
    c = workloads.chain()
    check(c, *run_chain(c))


def test_chain_workspace_reuse():
    """Each call leaves the workspace zero: calls on one workspace repeat and
    interleave with another chain."""
    d = dev()
    a = workloads.chain(widths=(11008, 4096, 11008, 4096, 1000), K0=4096)
    b = workloads.chain(widths=(300, 77, 500, 64, 33, 128), K0=1000, x_seed=33, w_seed0=60, bn_seed0=80)
    la, lb = gpu_layers(a), gpu_layers(b)
    ws = bnn.gemv_chain_workspace(d)
    first = run_chain(a, la, ws)
    check(a, *first)
    for _ in range(3):
        check(b, *run_chain(b, lb, ws))
        again = run_chain(a, la, ws)
        for t0, t1 in zip(first, again):
            assert torch.equal(t0, t1)
    assert int(ws.abs().sum()) == 0


def test_chain_unaligned_input():
    """x not 16-byte aligned: the input pack reads element by element."""
    c = workloads.chain(widths=(513, 4096, 77), K0=1003, x_dtype=torch.float32)
    buf = torch.zeros(1004, dtype=torch.float32, device=dev())
    buf[1:].copy_(c.x0.to(dev()))
    x = buf[1:]
    assert x.data_ptr() % 16 != 0
    check(c, *run_chain(c, x=x))


def test_chain_in_a_cuda_graph():
    """The cooperative launch captured in a graph and replayed."""
    d = dev()
    c = workloads.chain(widths=(11008, 4096, 1000), K0=4096)
    layers = bnn.chain_layers(gpu_layers(c))
    ws = bnn.gemv_chain_workspace(d)
    x = c.x0.to(d)
    y_i32 = torch.zeros(1000, dtype=torch.int32, device=d)
    y_f32 = torch.zeros(1000, dtype=torch.float32, device=d)
    acts = torch.zeros(2, bnn.bnn_packed_ld_words(11008), dtype=torch.int32, device=d)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        bnn.bnn_xnor_gemv_chain(layers, x, ws, y_i32=y_i32, y_f32=y_f32, acts=acts, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        bnn.bnn_xnor_gemv_chain(layers, x, ws, y_i32=y_i32, y_f32=y_f32, acts=acts)
    for _ in range(5):
        y_i32.fill_(0)
        g.replay()
    torch.cuda.synchronize()
    check(c, acts, y_i32, y_f32)


def test_chain_wait_gives_up_on_a_corrupt_workspace():
    """Slots whose row counts can never match make the second layer's wait
    run out: the call returns, the device error flag reads TIMEOUT, and the
    workspace is zero again for the next call."""
    d = dev()
    c = workloads.chain(widths=(256, 300, 77), K0=1000)
    layers = gpu_layers(c)
    ws = bnn.gemv_chain_workspace(d)
    slots = ws[16:].view(torch.int64)
    slots.fill_(0x7FFFFFF0 << 32)         # counts far above 32: never complete
    run_chain(c, layers, ws)
    assert bnn.bnn_device_error() == bnn.BNN_ERR_DEVICE_TIMEOUT
    assert int(ws.abs().sum()) == 0
    check(c, *run_chain(c, layers, ws))
