"""Binary 1x1 convolution with stride (the downsampling projection of a
ResNet-class block) against the oracle's literal convolution, through the C
ABI: int32 exact, alpha-scaled and affine fp32 within the tolerances of the
3x3 convolution."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import xnor_popcount_gemm_bnn_b200 as bnn
from gpu_util import assert_affine_close, assert_no_device_error, assert_scaled_close, dev

pytestmark = pytest.mark.gpu


def run_conv1x1(X, Wt, gamma, beta, stride, mode, rsign_beta=None):
    d = dev()
    n, c, h, w = X.shape
    cout = Wt.shape[0]
    Xb = bnn.empty_packed_nhwc(n, c, h, w, d)
    if rsign_beta is None:
        bnn.bnn_pack_sign_nchw(X.to(d).contiguous(), Xb)
    else:
        bnn.bnn_pack_sign_nchw_rsign(X.to(d).contiguous(), rsign_beta.to(d), Xb)
    Wp = bnn.empty_packed(cout, c, d)
    alpha = torch.empty(cout, dtype=torch.float32, device=d)
    bnn.bnn_pack_sign(Wt.reshape(cout, c).to(d).contiguous(), Wp, alpha)
    oh, ow = (h - 1) // stride + 1, (w - 1) // stride + 1
    dt = torch.int32 if mode == bnn.BNN_OUT_INT32 else torch.float32
    out = torch.full((n, cout, oh, ow), -7, dtype=dt, device=d)
    ep = bnn.make_epilogue(mode, alpha=alpha, gamma=None if gamma is None else gamma.to(d),
                           beta=None if beta is None else beta.to(d))
    bnn.bnn_binary_conv1x1_fused(Xb, c, Wp, ep, out, stride=stride)
    torch.cuda.synchronize()
    return out


# (n, c, h, w, cout, stride): the ResNet-18 downsampling shapes (64 -> 128 at
# 56x56, 128 -> 256, 256 -> 512), ragged channel words, odd sizes, stride 1
# and 3, one channel and one pixel.
CASES = [(2, 64, 56, 56, 128, 2), (2, 128, 28, 28, 256, 2), (1, 256, 14, 14, 512, 2), (3, 40, 9, 7, 5, 2),
         (1, 130, 8, 8, 16, 2), (2, 512, 7, 7, 8, 2), (2, 33, 5, 5, 3, 1), (1, 1, 1, 1, 1, 3), (2, 96, 11, 13, 20, 3),
         (1, 300, 6, 5, 33, 2)]


@pytest.mark.parametrize("n,c,h,w,cout,stride", CASES)
def test_conv1x1_modes(n, c, h, w, cout, stride):
    X = workloads.normal((n, c, h, w), 1.0, n + c + h + 1, dtype=torch.bfloat16)
    Wt = workloads.normal((cout, c, 1, 1), 0.1, cout + c + 1)
    g = workloads.uniform((cout,), 0.5, 1.5, cout + 2)
    b = workloads.normal((cout,), 0.1, cout + 3)
    s_ref = oracle.conv2d_pm1(oracle.sign_pm1(X), oracle.sign_pm1(Wt), stride, 0)
    a_ref = oracle.alpha(Wt.reshape(cout, -1))
    out_i = run_conv1x1(X, Wt, None, None, stride, bnn.BNN_OUT_INT32)
    assert np.array_equal(out_i.cpu().numpy(), s_ref)
    out_s = run_conv1x1(X, Wt, None, None, stride, bnn.BNN_OUT_SCALED_F32)
    assert_scaled_close(out_s, np.moveaxis(oracle.scaled(np.moveaxis(s_ref, 1, -1), a_ref), -1, 1))
    out_a = run_conv1x1(X, Wt, g, b, stride, bnn.BNN_OUT_AFFINE_F32)
    s2, y_a = oracle.conv_affine(X, Wt, g.numpy(), b.numpy(), stride, 0)
    assert np.array_equal(s2, s_ref)
    scale = (np.abs(g.numpy().astype(np.float64)[None, :, None, None] * a_ref[None, :, None, None] * s_ref)
             + np.abs(b.numpy().astype(np.float64))[None, :, None, None])
    assert_affine_close(out_a, y_a, scale)
    assert_no_device_error()


def test_conv1x1_after_rsign_pack():
    """The vision path with a learned activation threshold: RSign pack, then
    the downsampling 1x1 convolution, against the oracle's rsign + conv."""
    n, c, h, w, cout = 2, 64, 16, 16, 32
    X = workloads.normal((n, c, h, w), 1.0, 91)
    Wt = workloads.normal((cout, c, 1, 1), 0.1, 92)
    beta = workloads.normal((c,), 0.5, 93)
    out = run_conv1x1(X, Wt, None, None, 2, bnn.BNN_OUT_INT32, rsign_beta=beta)
    s_ref = oracle.conv2d_pm1(oracle.rsign_pm1(X, beta, axis=1), oracle.sign_pm1(Wt), 2, 0)
    assert np.array_equal(out.cpu().numpy(), s_ref)
    assert_no_device_error()
