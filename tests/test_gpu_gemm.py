"""Packed XOR-popcount GEMM and its fused epilogues against the oracle.

int32 products and packed output bits: bit-exact.  fp32: within 1e-6 relative
(alpha*s) or relative to the magnitude of the terms (affine)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import xnor_popcount_gemm_bnn_b200 as bnn
from gpu_util import assert_affine_close, assert_no_device_error, assert_scaled_close, dev, u32

pytestmark = pytest.mark.gpu

ENGINES = [bnn.BNN_GEMM_ENGINE_POPCOUNT, bnn.BNN_GEMM_ENGINE_TENSOR, bnn.BNN_GEMM_ENGINE_TENSOR_I8]
ENGINE_IDS = ["popcount", "tensor", "tensor_i8"]


@pytest.fixture(params=ENGINES, ids=ENGINE_IDS)
def engine(request):
    """Run the test body with one GEMM engine forced (both must agree with the oracle)."""
    with bnn.gemm_engine(request.param):
        yield request.param


def packed_operands(X, W):
    d = dev()
    M, K = X.shape
    N = W.shape[0]
    A_p = bnn.empty_packed(M, K, d)
    W_p = bnn.empty_packed(N, K, d)
    alpha = torch.empty(N, dtype=torch.float32, device=d)
    bnn.bnn_pack_sign(X.to(d), A_p)
    bnn.bnn_pack_sign(W.to(d), W_p, alpha)
    return A_p, W_p, alpha


def test_tiny_workload(engine):
    """X [64, 1000], W [256, 1000] N(0, 1): K not a multiple of 32."""
    t = workloads.tiny()
    A_p, W_p, alpha = packed_operands(t.X, t.W)
    C_i32 = torch.empty(t.M, t.N, dtype=torch.int32, device=dev())
    C_f32 = torch.empty(t.M, t.N, dtype=torch.float32, device=dev())
    bnn.bnn_xnor_gemm(A_p, W_p, t.K, alpha, C_i32, C_f32)
    s_ref, a_ref = oracle.binary_linear(t.X, t.W)
    assert np.array_equal(C_i32.cpu().numpy(), s_ref)
    assert_scaled_close(C_f32, oracle.scaled(s_ref, a_ref))
    assert_no_device_error()


RAGGED = [(1, 1, 1), (3, 5, 7), (129, 130, 1000), (200, 300, 65), (128, 128, 4096),
          (77, 255, 2049), (256, 384, 1024), (130, 129, 8192), (513, 33, 31), (64, 1000, 97),
          (300, 520, 700), (1000, 257, 5000)]


@pytest.mark.parametrize("M,N,K", RAGGED)
def test_ragged_shapes(M, N, K, engine):
    X = workloads.normal((M, K), 1.0, M * 31 + K)
    W = workloads.normal((N, K), 1.0, N * 37 + K + 1)
    A_p, W_p, alpha = packed_operands(X, W)
    C_i32 = torch.empty(M, N, dtype=torch.int32, device=dev())
    C_f32 = torch.empty(M, N, dtype=torch.float32, device=dev())
    bnn.bnn_xnor_gemm(A_p, W_p, K, alpha, C_i32, C_f32)
    s_ref, a_ref = oracle.binary_linear(X, W)
    assert np.array_equal(C_i32.cpu().numpy(), s_ref)
    assert_scaled_close(C_f32, oracle.scaled(s_ref, a_ref))


def test_output_strides_and_single_outputs(engine):
    M, N, K = 70, 90, 300
    X = workloads.normal((M, K), 1.0, 1)
    W = workloads.normal((N, K), 1.0, 2)
    A_p, W_p, alpha = packed_operands(X, W)
    big_i = torch.full((M, N + 13), -7, dtype=torch.int32, device=dev())
    bnn.bnn_xnor_gemm(A_p, W_p, K, None, big_i[:, :N], None)
    s_ref, a_ref = oracle.binary_linear(X, W)
    assert np.array_equal(big_i[:, :N].cpu().numpy(), s_ref)
    assert torch.all(big_i[:, N:] == -7)
    big_f = torch.full((M, N + 3), 5.0, dtype=torch.float32, device=dev())
    bnn.bnn_xnor_gemm(A_p, W_p, K, alpha, None, big_f[:, :N])
    assert_scaled_close(big_f[:, :N], oracle.scaled(s_ref, a_ref))
    assert torch.all(big_f[:, N:] == 5.0)


def test_closed_forms_on_gpu(engine):
    """W = X gives K on the diagonal, W = -X gives -K, Sylvester-Hadamard rows
    give 0 off the diagonal (eq. (6) identities with no oracle needed)."""
    K = 4096
    H = torch.ones(1, 1)
    while H.shape[0] < K:
        H = torch.cat([torch.cat([H, H], 1), torch.cat([H, -H], 1)], 0)
    A_p, W_p, _ = packed_operands(H[:256], H[:256])
    C = torch.empty(256, 256, dtype=torch.int32, device=dev())
    bnn.bnn_xnor_gemm(A_p, W_p, K, None, C)
    assert torch.equal(C.cpu(), K * torch.eye(256, dtype=torch.int32))
    A_n, _, _ = packed_operands(-H[:256], H[:8])
    bnn.bnn_xnor_gemm(A_n, W_p, K, None, C)
    assert torch.equal(torch.diagonal(C.cpu()), torch.full((256,), -K, dtype=torch.int32))


def test_affine_epilogue(engine):
    M, N, K = 150, 200, 576
    X = workloads.normal((M, K), 1.0, 3)
    W = workloads.normal((N, K), 0.1, 4)
    g = workloads.uniform((N,), 0.5, 1.5, 5)
    b = workloads.normal((N,), 0.1, 6)
    A_p, W_p, alpha = packed_operands(X, W)
    out = torch.empty(M, N, dtype=torch.float32, device=dev())
    ep = bnn.make_epilogue(bnn.BNN_OUT_AFFINE_F32, alpha=alpha, gamma=g.to(dev()), beta=b.to(dev()))
    bnn.bnn_binary_linear_fused(A_p, W_p, K, ep, out)
    s_ref, a_ref = oracle.binary_linear(X, W)
    y_ref = oracle.affine(s_ref, a_ref, g.numpy(), b.numpy())
    scale = np.abs(g.numpy().astype(np.float64) * a_ref * s_ref) + np.abs(b.numpy())
    assert_affine_close(out, y_ref, scale)
    out_i = torch.empty(M, N, dtype=torch.int32, device=dev())
    bnn.bnn_binary_linear_fused(A_p, W_p, K, bnn.make_epilogue(bnn.BNN_OUT_INT32), out_i)
    assert np.array_equal(out_i.cpu().numpy(), s_ref)
    out_s = torch.empty(M, N, dtype=torch.float32, device=dev())
    bnn.bnn_binary_linear_fused(A_p, W_p, K, bnn.make_epilogue(bnn.BNN_OUT_SCALED_F32, alpha=alpha), out_s)
    assert_scaled_close(out_s, oracle.scaled(s_ref, a_ref))


@pytest.mark.parametrize("M,N,K", [(64, 256, 1000), (130, 100, 4096), (1, 33, 64), (257, 513, 97),
                                   (200, 40, 300), (129, 300, 2000)])
def test_threshold_pack_epilogue(M, N, K, engine):
    """Folded BatchNorm + sign, re-packed along N: bit-exact against the
    oracle's direct float64 BatchNorm decision, pad bits and pad words 0."""
    X = workloads.normal((M, K), 1.0, M + 11)
    W = workloads.normal((N, K), 1.0, N + 12)
    bn = workloads.batchnorm_params(N, K)
    bn.mean.mul_(float(np.sqrt(K)) * 0.3)       # put thresholds inside the reachable range
    A_p, W_p, alpha = packed_operands(X, W)
    thr, mode = bnn.bnn_fold_bn_threshold(alpha.cpu(), bn.gamma, bn.beta, bn.mean, bn.var, bn.eps, K)
    out = torch.full((M, bnn.bnn_packed_ld_words(N)), -1, dtype=torch.int32, device=dev())
    ep = bnn.make_epilogue(bnn.BNN_OUT_THRESHOLD_PACK, popc_thresh=thr.to(dev()), thresh_mode=mode.to(dev()))
    bnn.bnn_binary_linear_fused(A_p, W_p, K, ep, out)
    s_ref, _ = oracle.binary_linear(X, W)
    a_f32 = oracle.alpha_f32(W)
    assert np.array_equal(a_f32, alpha.cpu().numpy())   # same fp32 alpha on both sides
    act = oracle.bn_sign(s_ref, a_f32, bn.gamma.numpy(), bn.beta.numpy(), bn.mean.numpy(),
                         bn.var.numpy(), bn.eps)
    assert np.array_equal(u32(out), oracle.pack_pm1(act))
    assert_no_device_error()


def test_square_workload_sampled_rows(engine):
    """M = N = K = 8192 (the square workload) on the GPU, checked on 48 sampled
    rows against the oracle (every column of those rows)."""
    sq = workloads.square()
    A_p, W_p, alpha = packed_operands(sq.A, sq.W)
    C_i32 = torch.empty(sq.M, sq.N, dtype=torch.int32, device=dev())
    C_f32 = torch.empty(sq.M, sq.N, dtype=torch.float32, device=dev())
    bnn.bnn_xnor_gemm(A_p, W_p, sq.K, alpha, C_i32, C_f32)
    rows = np.sort(np.random.default_rng(8192).choice(sq.M, 48, replace=False))
    rows[-1] = sq.M - 1
    s_ref = oracle.matmul_pm1(oracle.sign_pm1(sq.A[rows]), oracle.sign_pm1(sq.W))
    a_ref = oracle.alpha(sq.W)
    assert np.array_equal(C_i32[torch.from_numpy(rows).to(dev())].cpu().numpy(), s_ref)
    assert_scaled_close(C_f32[torch.from_numpy(rows).to(dev())], oracle.scaled(s_ref, a_ref))
    # properties that hold at any size: parity of s and |s| <= K on the whole output
    C = C_i32.cpu()
    assert bool(((C - sq.K) % 2 == 0).all()) and int(C.abs().max()) <= sq.K
    assert_no_device_error()


def test_engine_setting_roundtrip():
    prev = bnn.bnn_get_gemm_engine()
    for e in (bnn.BNN_GEMM_ENGINE_TENSOR, bnn.BNN_GEMM_ENGINE_TENSOR_I8, bnn.BNN_GEMM_ENGINE_POPCOUNT,
              bnn.BNN_GEMM_ENGINE_AUTO):
        bnn.bnn_set_gemm_engine(e)
        assert bnn.bnn_get_gemm_engine() == e
    with pytest.raises(bnn.BnnError):
        bnn.bnn_set_gemm_engine(7)
    bnn.bnn_set_gemm_engine(prev)


def test_engines_agree_bit_for_bit():
    """Every engine on the same operands: identical int32 and identical fp32."""
    M, N, K = 384, 512, 3000
    X = workloads.normal((M, K), 1.0, 77)
    W = workloads.normal((N, K), 1.0, 78)
    A_p, W_p, alpha = packed_operands(X, W)
    outs = []
    for e in ENGINES:
        with bnn.gemm_engine(e):
            Ci = torch.empty(M, N, dtype=torch.int32, device=dev())
            Cf = torch.empty(M, N, dtype=torch.float32, device=dev())
            bnn.bnn_xnor_gemm(A_p, W_p, K, alpha, Ci, Cf)
            outs.append((Ci.cpu(), Cf.cpu()))
    for o in outs[1:]:
        assert torch.equal(outs[0][0], o[0])
        assert torch.equal(outs[0][1], o[1])
    assert_no_device_error()


@pytest.mark.parametrize("tensor_engine,launches", [(bnn.BNN_GEMM_ENGINE_TENSOR, 8), (bnn.BNN_GEMM_ENGINE_TENSOR_I8, 4)],
                         ids=["tensor", "tensor_i8"])
def test_tensor_engine_full_matrix_repeated(tensor_engine, launches):
    """Races show up as a few wrong tiles in some launches only, so the square
    workload runs several times on a tensor engine and every one of the 67M int32
    outputs is compared with the popcount engine's (two independent kernels;
    the popcount result is itself checked against the oracle above).  Once with
    fp32 alpha outputs too, whose epilogue parameters come from shared memory."""
    sq = workloads.square()
    A_p, W_p, alpha = packed_operands(sq.A, sq.W)
    ref = torch.empty(sq.M, sq.N, dtype=torch.int32, device=dev())
    ref_f = torch.empty(sq.M, sq.N, dtype=torch.float32, device=dev())
    with bnn.gemm_engine(bnn.BNN_GEMM_ENGINE_POPCOUNT):
        bnn.bnn_xnor_gemm(A_p, W_p, sq.K, alpha, ref, ref_f)
    C = torch.empty_like(ref)
    Cf = torch.empty_like(ref_f)
    with bnn.gemm_engine(tensor_engine):
        for r in range(launches):
            C.fill_(0x5A5A5A5A)
            Cf.fill_(float("nan"))
            bnn.bnn_xnor_gemm(A_p, W_p, sq.K, alpha if r == 0 else None, C, Cf if r == 0 else None)
            torch.cuda.synchronize()
            assert torch.equal(C, ref), f"launch {r}: {int((C != ref).sum())} outputs differ"
            if r == 0:
                assert torch.equal(Cf, ref_f)
    assert_no_device_error()


def test_e2m1_engine_exact_at_the_largest_k():
    """The 4-bit tensor engine accumulates in fp32; its partial sums are
    integers of magnitude up to the padded K (2^20 at most), which fp32 holds
    exactly.  K = 1,048,000 (padded 1,048,064, the top of its range): W rows
    0..129 are the A rows with 1 in 64 elements negated, so s[m, m] = K - 2 f_m
    (about 0.97 K, closed form), and every output must equal the popcount
    engine's exact integer."""
    M, N, K = 130, 140, 1_048_000
    d = dev()
    X = workloads.normal((M, K), 1.0, 2024)
    flip = workloads.uniform((M, K), 0.0, 1.0, 2025) < (1.0 / 64)
    Wt = torch.cat([torch.where(flip, -X, X), workloads.normal((N - M, K), 1.0, 2026)])
    # sign(-x) differs from sign(x) unless x == 0 (then both are +1)
    f = (flip & (X != 0)).sum(1)
    A_p, W_p, _ = packed_operands(X, Wt)
    del X, Wt, flip
    out = {}
    for e in (bnn.BNN_GEMM_ENGINE_TENSOR, bnn.BNN_GEMM_ENGINE_POPCOUNT):
        with bnn.gemm_engine(e):
            C = torch.empty(M, N, dtype=torch.int32, device=d)
            bnn.bnn_xnor_gemm(A_p, W_p, K, None, C)
            out[e] = C.cpu()
    diag = torch.diagonal(out[bnn.BNN_GEMM_ENGINE_TENSOR][:, :M])
    assert torch.equal(diag, (K - 2 * f).to(torch.int32))
    assert torch.equal(out[bnn.BNN_GEMM_ENGINE_TENSOR], out[bnn.BNN_GEMM_ENGINE_POPCOUNT])
    assert_no_device_error()
