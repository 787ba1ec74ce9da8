"""Fully binary MLP forward: layers chained through the THRESHOLD_PACK epilogue
(each layer's packed output is the next layer's packed A), last layer alpha*s.
Bits bit-exact, logits within 1e-6 relative."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import xnor_popcount_gemm_bnn_b200 as bnn
from gpu_util import assert_no_device_error, assert_scaled_close, dev, u32

pytestmark = pytest.mark.gpu


@pytest.fixture(params=[bnn.BNN_GEMM_ENGINE_POPCOUNT, bnn.BNN_GEMM_ENGINE_TENSOR, bnn.BNN_GEMM_ENGINE_TENSOR_I8],
                ids=["popcount", "tensor", "tensor_i8"])
def engine(request):
    with bnn.gemm_engine(request.param):
        yield request.param


def gpu_mlp(m: workloads.Mlp):
    """Pack input and weights, fold BN on the host once, run the layers."""
    d = dev()
    B, D = m.X0.shape
    A = bnn.empty_packed(B, D, d)
    bnn.bnn_pack_sign(m.X0.to(d), A)
    acts = [A]
    logits = None
    L = len(m.Ws)
    for l, W in enumerate(m.Ws):
        N, K = W.shape
        W_p = bnn.empty_packed(N, K, d)
        alpha = torch.empty(N, dtype=torch.float32, device=d)
        bnn.bnn_pack_sign(W.to(d), W_p, alpha)
        if l < L - 1:
            bn = m.bns[l]
            thr, mode = bnn.bnn_fold_bn_threshold(alpha.cpu(), bn.gamma, bn.beta, bn.mean, bn.var, bn.eps, K)
            out = bnn.empty_packed(B, N, d)
            ep = bnn.make_epilogue(bnn.BNN_OUT_THRESHOLD_PACK, popc_thresh=thr.to(d), thresh_mode=mode.to(d))
            bnn.bnn_binary_linear_fused(A, W_p, K, ep, out)
            A = out
            acts.append(A)
        else:
            logits = torch.empty(B, N, dtype=torch.float32, device=d)
            bnn.bnn_binary_linear_fused(A, W_p, K, bnn.make_epilogue(bnn.BNN_OUT_SCALED_F32, alpha=alpha), logits)
    return acts, logits


def oracle_mlp(m: workloads.Mlp, rows=None):
    X0 = m.X0 if rows is None else m.X0[rows]
    bns = [(b.gamma.numpy(), b.beta.numpy(), b.mean.numpy(), b.var.numpy(), b.eps) for b in m.bns]
    return oracle.mlp_forward(X0, m.Ws, bns)


@pytest.mark.parametrize("batch,width", [(64, 256), (100, 300), (33, 4096)])
def test_small_mlp_all_rows(batch, width, engine):
    m = workloads.mlp(batch=batch, width=width)
    acts, logits = gpu_mlp(m)
    acts_ref, logits_ref = oracle_mlp(m)
    for l in range(len(acts)):
        assert np.array_equal(u32(acts[l]), oracle.pack_pm1(acts_ref[l])), f"layer {l} bits"
    assert_scaled_close(logits, logits_ref)
    assert_no_device_error()


def test_mlp_workload_sampled_rows(engine):
    """Batch 4096, width 4096, 4 layers; rows are independent, so 24 sampled
    rows are checked through all layers against the oracle."""
    m = workloads.mlp()
    acts, logits = gpu_mlp(m)
    rows = np.sort(np.random.default_rng(4096).choice(4096, 24, replace=False))
    acts_ref, logits_ref = oracle_mlp(m, rows)
    ridx = torch.from_numpy(rows).to(dev())
    for l in range(len(acts)):
        assert np.array_equal(u32(acts[l][ridx]), oracle.pack_pm1(acts_ref[l])), f"layer {l} bits"
    assert_scaled_close(logits[ridx], logits_ref)
    assert_no_device_error()


def test_threshold_layer_engines_agree_repeated():
    """One 4096 x 4096 x 4096 BN-threshold layer, 4 launches on the tensor
    engine, every packed output word compared with the popcount engine's."""
    m = workloads.mlp()
    d = dev()
    B, D = m.X0.shape
    A = bnn.empty_packed(B, D, d)
    bnn.bnn_pack_sign(m.X0.to(d), A)
    W_p = bnn.empty_packed(D, D, d)
    alpha = torch.empty(D, dtype=torch.float32, device=d)
    bnn.bnn_pack_sign(m.Ws[0].to(d), W_p, alpha)
    bn = m.bns[0]
    thr, mode = bnn.bnn_fold_bn_threshold(alpha.cpu(), bn.gamma, bn.beta, bn.mean, bn.var, bn.eps, D)
    ep = bnn.make_epilogue(bnn.BNN_OUT_THRESHOLD_PACK, popc_thresh=thr.to(d), thresh_mode=mode.to(d))
    ref = bnn.empty_packed(B, D, d)
    with bnn.gemm_engine(bnn.BNN_GEMM_ENGINE_POPCOUNT):
        bnn.bnn_binary_linear_fused(A, W_p, D, ep, ref)
    out = bnn.empty_packed(B, D, d)
    with bnn.gemm_engine(bnn.BNN_GEMM_ENGINE_TENSOR):
        for r in range(4):
            out.fill_(0x5A5A5A5A)
            bnn.bnn_binary_linear_fused(A, W_p, D, ep, out)
            torch.cuda.synchronize()
            assert torch.equal(out, ref), f"launch {r}: {int((out != ref).sum())} words differ"
    assert_no_device_error()
