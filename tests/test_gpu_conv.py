"""Binary 3x3 convolution (implicit GEMM on packed channel words) against the
oracle's literal 7-loop convolution."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import xnor_popcount_gemm_bnn_b200 as bnn
from gpu_util import assert_affine_close, assert_no_device_error, assert_scaled_close, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(params=[bnn.BNN_GEMM_ENGINE_POPCOUNT, bnn.BNN_GEMM_ENGINE_TENSOR, bnn.BNN_GEMM_ENGINE_TENSOR_I8],
                ids=["popcount", "tensor", "tensor_i8"])
def engine(request):
    """TENSOR runs the tcgen05 convolution where it applies (c <= 64,
    cout <= 256); other shapes stay on the popcount kernel."""
    with bnn.gemm_engine(request.param):
        yield request.param


def run_conv(X, Wt, gamma, beta, stride, pad, mode):
    d = dev()
    n, c, h, w = X.shape
    cout = Wt.shape[0]
    Xb = bnn.empty_packed_nhwc(n, c, h, w, d)
    bnn.bnn_pack_sign_nchw(X.to(d).contiguous(), Xb)
    Wp = bnn.empty_conv3x3_weights(cout, c, d)
    alpha = torch.empty(cout, dtype=torch.float32, device=d)
    bnn.bnn_pack_conv3x3_weights(Wt.to(d).contiguous(), Wp, alpha)
    oh = (h + 2 * pad - 3) // stride + 1
    ow = (w + 2 * pad - 3) // stride + 1
    dt = torch.int32 if mode == bnn.BNN_OUT_INT32 else torch.float32
    out = torch.empty(n, cout, oh, ow, dtype=dt, device=d)
    ep = bnn.make_epilogue(mode, alpha=alpha, gamma=None if gamma is None else gamma.to(d),
                           beta=None if beta is None else beta.to(d))
    bnn.bnn_binary_conv3x3_fused(Xb, c, Wp, ep, out, stride=stride, pad=pad)
    return out


CASES = [(2, 64, 9, 7, 5, 1, 1), (1, 3, 5, 6, 4, 1, 1), (2, 33, 8, 8, 3, 2, 1), (1, 2, 4, 4, 2, 1, 0),
         (3, 100, 7, 9, 17, 1, 1), (1, 128, 6, 6, 8, 1, 1), (2, 64, 56, 56, 64, 1, 1), (1, 40, 11, 13, 6, 2, 0),
         # tensor-core shapes: filter counts off the 16/32 grid, 256 filters, ragged last tile
         (3, 50, 19, 17, 40, 1, 1), (1, 20, 9, 9, 48, 1, 1), (2, 32, 12, 12, 256, 1, 1), (1, 64, 10, 10, 200, 1, 1),
         (1, 1, 5, 5, 1, 1, 1), (5, 64, 33, 31, 96, 2, 1), (1, 16, 6, 7, 8, 1, 2)]


@pytest.mark.parametrize("n,c,h,w,cout,stride,pad", CASES)
def test_conv_modes(n, c, h, w, cout, stride, pad, engine):
    X = workloads.normal((n, c, h, w), 1.0, n + c + h, dtype=torch.bfloat16)
    Wt = workloads.normal((cout, c, 3, 3), 0.1, cout + c)
    g = workloads.uniform((cout,), 0.5, 1.5, cout)
    b = workloads.normal((cout,), 0.1, cout + 1)
    xb = oracle.sign_pm1(X)
    fb = oracle.sign_pm1(Wt)
    s_ref = oracle.conv2d_pm1(xb, fb, stride, pad)
    a_ref = oracle.alpha(Wt.reshape(cout, -1))
    out_i = run_conv(X, Wt, None, None, stride, pad, bnn.BNN_OUT_INT32)
    assert np.array_equal(out_i.cpu().numpy(), s_ref)
    out_s = run_conv(X, Wt, None, None, stride, pad, bnn.BNN_OUT_SCALED_F32)
    y_s = np.moveaxis(oracle.scaled(np.moveaxis(s_ref, 1, -1), a_ref), -1, 1)
    assert_scaled_close(out_s, y_s)
    out_a = run_conv(X, Wt, g, b, stride, pad, bnn.BNN_OUT_AFFINE_F32)
    _, y_a = oracle.conv3x3_affine(X, Wt, g.numpy(), b.numpy(), stride, pad)
    scale = (np.abs(g.numpy().astype(np.float64)[None, :, None, None] * a_ref[None, :, None, None] * s_ref)
             + np.abs(b.numpy().astype(np.float64))[None, :, None, None])
    assert_affine_close(out_a, y_a, scale)
    assert_no_device_error()


def test_resnet_layer_workload_sampled_images(engine):
    """The ResNet-18-class layer: input bf16 [64, 64, 56, 56], filters
    [64, 64, 3, 3], stride 1, pad 1, affine epilogue; images 0, 31 and 63
    checked against the oracle (each image is independent)."""
    cv = workloads.conv()
    out = run_conv(cv.X, cv.W, cv.gamma, cv.beta, 1, 1, bnn.BNN_OUT_AFFINE_F32)
    imgs = [0, 31, 63]
    s_ref, y_ref = oracle.conv3x3_affine(cv.X[imgs], cv.W, cv.gamma.numpy(), cv.beta.numpy(), 1, 1)
    a_ref = oracle.alpha(cv.W.reshape(64, -1))
    scale = (np.abs(cv.gamma.numpy().astype(np.float64)[None, :, None, None] * a_ref[None, :, None, None]
                    * s_ref) + np.abs(cv.beta.numpy().astype(np.float64))[None, :, None, None])
    assert_affine_close(out[imgs], y_ref, scale)
    assert_no_device_error()


@pytest.mark.parametrize("n,c,h,w,cout", [(1, 128, 170, 340, 16), (1, 20, 40, 1680, 16)])
def test_conv_window_segments(n, c, h, w, cout):
    """Wide images: the 2*(w+2)+2 halo leaves room for one 128-position tile
    per shared-memory buffer, so the stride-1 tensor-core kernel walks each
    CTA's 3-4 tiles as separate segments and reuses both buffers.  INT32 and
    affine outputs against the oracle, and the popcount engine bit for bit."""
    X = workloads.normal((n, c, h, w), 1.0, w, dtype=torch.bfloat16)
    Wt = workloads.normal((cout, c, 3, 3), 0.1, c)
    g = workloads.uniform((cout,), 0.5, 1.5, cout)
    b = workloads.normal((cout,), 0.1, cout + 1)
    with bnn.gemm_engine(bnn.BNN_GEMM_ENGINE_TENSOR):
        out_i = run_conv(X, Wt, None, None, 1, 1, bnn.BNN_OUT_INT32)
        out_a = run_conv(X, Wt, g, b, 1, 1, bnn.BNN_OUT_AFFINE_F32)
    with bnn.gemm_engine(bnn.BNN_GEMM_ENGINE_POPCOUNT):
        out_p = run_conv(X, Wt, None, None, 1, 1, bnn.BNN_OUT_INT32)
    s_ref, y_ref = oracle.conv3x3_affine(X, Wt, g.numpy(), b.numpy(), 1, 1)
    assert np.array_equal(out_i.cpu().numpy(), s_ref)
    assert torch.equal(out_i, out_p)
    a_ref = oracle.alpha(Wt.reshape(cout, -1))
    scale = (np.abs(g.numpy().astype(np.float64)[None, :, None, None] * a_ref[None, :, None, None] * s_ref)
             + np.abs(b.numpy().astype(np.float64))[None, :, None, None])
    assert_affine_close(out_a, y_ref, scale)
    assert_no_device_error()


@pytest.mark.parametrize("tensor_engine", [bnn.BNN_GEMM_ENGINE_TENSOR, bnn.BNN_GEMM_ENGINE_TENSOR_I8],
                         ids=["tensor", "tensor_i8"])
def test_tensor_conv_full_output_repeated(tensor_engine):
    """Races show up as a few wrong tiles in some launches only: the ResNet
    layer runs 4 times on the tensor-core window kernel (e2m1 and int8
    operands; INT32 output) and all 12.8M outputs are compared with the
    popcount kernel's."""
    cv = workloads.conv()
    d = dev()
    n, c, h, w = cv.X.shape
    Xb = bnn.empty_packed_nhwc(n, c, h, w, d)
    bnn.bnn_pack_sign_nchw(cv.X.to(d), Xb)
    Wp = bnn.empty_conv3x3_weights(64, c, d)
    bnn.bnn_pack_conv3x3_weights(cv.W.to(d), Wp, None)
    ep = bnn.make_epilogue(bnn.BNN_OUT_INT32)
    ref = torch.empty(n, 64, h, w, dtype=torch.int32, device=d)
    with bnn.gemm_engine(bnn.BNN_GEMM_ENGINE_POPCOUNT):
        bnn.bnn_binary_conv3x3_fused(Xb, c, Wp, ep, ref, 1, 1)
    out = torch.empty_like(ref)
    with bnn.gemm_engine(tensor_engine):
        for r in range(4):
            out.fill_(0x5A5A5A5A)
            bnn.bnn_binary_conv3x3_fused(Xb, c, Wp, ep, out, 1, 1)
            torch.cuda.synchronize()
            assert torch.equal(out, ref), f"launch {r}: {int((out != ref).sum())} outputs differ"
    assert_no_device_error()
