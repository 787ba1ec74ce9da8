"""Host BatchNorm fold (libbnn.so, no GPU needed) against the oracle's direct
BatchNorm decision, exhaustively over every reachable s = K - 2d.

The fold turns "sign(BN(alpha*s)) = +1" into one integer compare on the
popcount d per channel; the oracle evaluates the BatchNorm value in float64 for
every s directly.  They must agree on every (channel, d)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import xnor_popcount_gemm_bnn_b200 as bnn


def folded_bits(thr, mode, K):
    d = np.arange(K + 1)[None, :]
    thr = thr.numpy().astype(np.int64)[:, None]
    mode = mode.numpy()[:, None]
    return np.where(mode == 0, d > thr, d < thr)          # True = bit 1 = -1


def oracle_bits(alpha_f32, g, b, mu, var, eps, K):
    d = np.arange(K + 1)[:, None]
    s = K - 2 * d                                           # [K+1, 1] broadcast over channels
    return (oracle.bn_sign(s, alpha_f32, g, b, mu, var, eps) == -1).T


def check(alpha, g, b, mu, var, eps, K):
    thr, mode = bnn.bnn_fold_bn_threshold(torch.from_numpy(alpha), torch.from_numpy(g),
                                          torch.from_numpy(b), torch.from_numpy(mu),
                                          torch.from_numpy(var), eps, K)
    got = folded_bits(thr, mode, K)
    want = oracle_bits(alpha, g, b, mu, var, eps, K)
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"fold disagrees at (channel, d) {bad[:5].tolist()}"
    return thr, mode


@pytest.mark.parametrize("K", [1, 2, 7, 64, 1000, 4096])
def test_fold_random_channels(K):
    rng = np.random.default_rng(K)
    N = 512
    alpha = rng.uniform(0.01, 2.0, N).astype(np.float32)
    g = rng.uniform(0.5, 1.5, N).astype(np.float32) * rng.choice([-1, 1], N).astype(np.float32)
    b = (0.1 * rng.standard_normal(N)).astype(np.float32)
    mu = (np.sqrt(K) * rng.standard_normal(N)).astype(np.float32)
    var = rng.uniform(0.5, 2.0, N).astype(np.float32)
    check(alpha, g, b, mu, var, 1e-5, K)


def test_fold_degenerate_channels():
    K = 33
    # gamma = 0 (constant sign(beta)), alpha = 0 (constant), thresholds beyond both ends,
    # a tie exactly at zero, negative gamma.
    alpha = np.array([1, 1, 0, 1, 1, 0.5, 1, 1], np.float32)
    g = np.array([0, 0, 1, 1, 1, 1, -1, -2], np.float32)
    b = np.array([0.5, -0.5, 0.3, 0, 0, 0, 0.25, 0], np.float32)
    mu = np.array([0, 0, 0, 1e6, -1e6, 2.5, 3, -7], np.float32)
    var = np.array([1, 1, 1, 1, 1, 1 - 1e-5, 1, 1], np.float32)
    thr, mode = check(alpha, g, b, mu, var, 1e-5, K)
    assert (int(thr[0]), int(mode[0])) == (K, 0)     # always +1
    assert (int(thr[1]), int(mode[1])) == (-1, 0)    # always -1
    assert (int(thr[3]), int(mode[3])) == (-1, 0)    # mean far above every alpha*s
    assert (int(thr[4]), int(mode[4])) == (K, 0)     # mean far below


def test_fold_mlp_workload_parameters():
    """The BatchNorm parameters of the 4-layer binary MLP workload (width 4096),
    with alpha from its weights: every channel, every d."""
    m = workloads.mlp(batch=1, width=4096)
    for l, bn in enumerate(m.bns):
        a = oracle.alpha_f32(m.Ws[l])
        check(a, bn.gamma.numpy(), bn.beta.numpy(), bn.mean.numpy(), bn.var.numpy(), bn.eps, 4096)
