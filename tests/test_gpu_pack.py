"""Sign-and-pack kernels against the oracle: packed words bit-exact (pad bits
and pad words included), alpha within 1e-6 relative."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import xnor_popcount_gemm_bnn_b200 as bnn
from gpu_util import assert_no_device_error, dev, u32

pytestmark = pytest.mark.gpu

SHAPES = [(1, 1), (5, 31), (7, 32), (3, 33), (2, 65), (9, 129), (64, 1000), (256, 1000),
          (4, 4096), (3, 8192), (33, 4097), (1, 12345)]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("rows,K", SHAPES)
def test_pack_sign_rows(rows, K, dtype):
    x = workloads.random_with_edges(rows, K, seed=rows * 7919 + K, dtype=dtype)
    xd = x.to(dev())
    packed = bnn.empty_packed(rows, K, dev())
    alpha = torch.empty(rows, dtype=torch.float32, device=dev())
    bnn.bnn_pack_sign(xd, packed, alpha)
    assert np.array_equal(u32(packed), oracle.pack_real(x))
    a_ref = oracle.alpha(x)
    a = alpha.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(a - a_ref) <= 1e-6 * np.abs(a_ref))
    assert_no_device_error()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_pack_sign_nonfinite_and_signed_zero(dtype):
    edges = workloads.sign_edge_values(dtype)
    x = edges.repeat(3, 11)[:, :150].contiguous()          # NaN, +-inf, -0.0, denormals ...
    packed = bnn.empty_packed(x.shape[0], x.shape[1], dev())
    bnn.bnn_pack_sign(x.to(dev()), packed)                   # no alpha
    assert np.array_equal(u32(packed), oracle.pack_real(x))


def test_pack_sign_strided_and_wide_ld():
    """Row stride ld_x > K that breaks 16-byte alignment (scalar path), and an
    output stride wider than needed: words past the padded row stay untouched."""
    rows, K, ldx = 17, 999, 1003
    base = workloads.normal((rows, ldx), 1.0, 42)
    x = base[:, :K]
    packed = torch.full((rows, bnn.bnn_packed_ld_words(K) + 8), -1, dtype=torch.int32, device=dev())
    alpha = torch.empty(rows, dtype=torch.float32, device=dev())
    bnn.bnn_pack_sign(base.to(dev())[:, :K], packed, alpha)
    got = u32(packed)
    kw = bnn.bnn_packed_ld_words(K)
    assert np.array_equal(got[:, :kw], oracle.pack_real(x))
    assert np.all(got[:, kw:] == 0xFFFFFFFF)
    a_ref = oracle.alpha(x)
    assert np.all(np.abs(alpha.cpu().numpy() - a_ref) <= 1e-6 * a_ref)


def test_pack_sign_alpha_closed_form():
    rows, K = 8, 1000
    c = 0.375
    sgn = torch.where(workloads.normal((rows, K), 1.0, 5) < 0, -1.0, 1.0)
    x = (c * sgn).to(torch.float32)
    packed = bnn.empty_packed(rows, K, dev())
    alpha = torch.empty(rows, dtype=torch.float32, device=dev())
    bnn.bnn_pack_sign(x.to(dev()), packed, alpha)
    assert torch.all(alpha.cpu() == c)


def test_pack_sign_gemv_weights_full_size():
    """The LLM-decode weight matrix [11008, 4096] fp32 N(0, 0.02)."""
    g = workloads.gemv()
    packed = bnn.empty_packed(g.N, g.K, dev())
    alpha = torch.empty(g.N, dtype=torch.float32, device=dev())
    bnn.bnn_pack_sign(g.W.to(dev()), packed, alpha)
    assert np.array_equal(u32(packed), oracle.pack_real(g.W))
    a_ref = oracle.alpha(g.W)
    assert np.all(np.abs(alpha.cpu().numpy() - a_ref) <= 1e-6 * a_ref)
    assert_no_device_error()


def expected_nhwc(x):
    """Oracle words per pixel: sign of the channel vector, packed (first cw words)."""
    n, c, h, w = x.shape
    cw = (c + 31) // 32
    xs = x.float().permute(0, 2, 3, 1).reshape(-1, c)
    return oracle.pack_real(xs)[:, :cw].reshape(n, h, w, cw)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", [(2, 64, 5, 7), (2, 33, 8, 8), (1, 1, 3, 3), (3, 100, 4, 6),
                                   (2, 64, 56, 56), (2, 48, 6, 4), (1, 17, 4, 4), (3, 70, 5, 9),
                                   (2, 300, 9, 16), (1, 520, 4, 8), (3, 32, 40, 40), (1, 5, 1, 8)])
def test_pack_sign_nchw(shape, dtype):
    n, c, h, w = shape
    x = workloads.random_with_edges(n * c, h * w, seed=sum(shape), dtype=dtype).reshape(shape).contiguous()
    out = bnn.empty_packed_nhwc(n, c, h, w, dev())
    bnn.bnn_pack_sign_nchw(x.to(dev()), out)
    assert np.array_equal(u32(out), expected_nhwc(x))


def expected_conv_weights(wt):
    """Oracle rows in (kh, kw, c) order, channels padded to whole words per tap."""
    cout, cin = wt.shape[:2]
    cw = (cin + 31) // 32
    t = wt.float().permute(0, 2, 3, 1)                                 # co, kh, kw, c
    tp = torch.zeros(cout, 3, 3, 32 * cw)
    tp[..., :cin] = t
    packed = oracle.pack_real(tp.reshape(cout, -1))                    # zeros pack as +1
    ldk = bnn.bnn_conv3x3_ld_words(cin)
    out = np.zeros((cout, ldk), np.uint32)
    out[:, :9 * cw] = packed[:, :9 * cw]
    return out


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("cout,cin", [(64, 64), (5, 3), (7, 33), (16, 128)])
def test_pack_conv3x3_weights(cout, cin, dtype):
    wt = workloads.normal((cout, cin, 3, 3), 0.1, cout * 100 + cin).to(dtype)
    packed = bnn.empty_conv3x3_weights(cout, cin, dev())
    alpha = torch.empty(cout, dtype=torch.float32, device=dev())
    bnn.bnn_pack_conv3x3_weights(wt.to(dev()).contiguous(), packed, alpha)
    assert np.array_equal(u32(packed), expected_conv_weights(wt))
    a_ref = oracle.alpha(wt.float().reshape(cout, -1))
    assert np.all(np.abs(alpha.cpu().numpy() - a_ref) <= 1e-6 * a_ref)


# ---------------------------------------------------------------------------
# per-channel threshold (RSign): sign(x - beta_c)
# ---------------------------------------------------------------------------

def _beta(n, seed):
    b = workloads.normal((n,), 0.5, seed)
    b[:3] = torch.tensor([0.0, float("inf"), -float("inf")])[: min(3, n)]
    return b


@pytest.mark.parametrize("rows,K", [(1, 1), (7, 33), (64, 1000), (300, 4096), (5, 4100)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_pack_sign_rsign_rows(rows, K, dtype):
    d = dev()
    x = workloads.normal((rows, K), 1.0, rows + 3 * K).to(dtype)
    x[0, : min(K, 4)] = torch.tensor([0.0, -0.0, float("nan"), 1.0])[: min(K, 4)].to(dtype)
    beta = _beta(K, K + 5)
    if K > 4:
        x[0, 4] = beta[4].to(dtype)                                   # a tie where bf16 holds beta exactly or not
    packed = torch.full((rows, bnn.bnn_packed_ld_words(K)), -1, dtype=torch.int32, device=d)
    bnn.bnn_pack_sign_rsign(x.to(d), beta.to(d), packed)
    torch.cuda.synchronize()
    want = oracle.pack_pm1(oracle.rsign_pm1(x, beta, axis=1))
    assert np.array_equal(u32(packed), want)
    assert_no_device_error()


@pytest.mark.parametrize("shape", [(2, 64, 56, 56), (3, 40, 7, 9), (1, 130, 5, 5), (2, 32, 1, 1)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_pack_sign_nchw_rsign(shape, dtype):
    d = dev()
    n, c, h, w = shape
    x = workloads.normal(shape, 1.0, n * c + h * w).to(dtype)
    beta = _beta(c, c + 11)
    x[0, 3, 0, 0] = beta[3].to(dtype)
    packed = bnn.empty_packed_nhwc(n, c, h, w, d)
    bnn.bnn_pack_sign_nchw_rsign(x.to(d), beta.to(d), packed)
    torch.cuda.synchronize()
    cw = (c + 31) // 32
    r = oracle.rsign_pm1(x, beta, axis=1)                               # [n, c, h, w]
    want = oracle.pack_pm1(np.ascontiguousarray(r.transpose(0, 2, 3, 1)).reshape(-1, c))[:, :cw]
    assert np.array_equal(u32(packed).reshape(-1, cw), want)
    assert_no_device_error()


def test_pack_sign_rsign_zero_threshold_is_sign():
    """beta = 0 gives exactly bnn_pack_sign's bits (both layouts)."""
    d = dev()
    x = workloads.normal((4, 64, 9, 9), 1.0, 77).to(d)
    a = bnn.empty_packed_nhwc(4, 64, 9, 9, d)
    b = bnn.empty_packed_nhwc(4, 64, 9, 9, d)
    bnn.bnn_pack_sign_nchw(x, a)
    bnn.bnn_pack_sign_nchw_rsign(x, torch.zeros(64, device=d), b)
    m = x.reshape(36, -1)
    pa = bnn.empty_packed(36, m.shape[1], d)
    pb = bnn.empty_packed(36, m.shape[1], d)
    bnn.bnn_pack_sign(m, pa)
    bnn.bnn_pack_sign_rsign(m, torch.zeros(m.shape[1], device=d), pb)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(pa, pb)
    assert_no_device_error()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_pack_sign_nchw_many_tiles_per_warp(dtype):
    """A tensor of more 4 KiB tiles than the grid's warps x stages, so every
    warp of the TMA-streamed pack refills its stages; checked against the
    oracle and against the register kernel (taken for an unaligned view)."""
    d = dev()
    n, c, h, w = 96, 64, 56, 56
    x = workloads.normal((n, c, h, w), 1.0, 4242).to(dtype)
    xd = x.to(d)
    out = bnn.empty_packed_nhwc(n, c, h, w, d)
    bnn.bnn_pack_sign_nchw(xd, out)
    buf = torch.empty(xd.numel() + 8, dtype=dtype, device=d)
    xu = buf[1:1 + xd.numel()].view(n, c, h, w)                      # 2 or 4 bytes off: the other kernel
    xu.copy_(xd)
    out_u = bnn.empty_packed_nhwc(n, c, h, w, d)
    bnn.bnn_pack_sign_nchw(xu, out_u)
    torch.cuda.synchronize()
    assert torch.equal(out, out_u)
    assert np.array_equal(u32(out), expected_nhwc(x))
    assert_no_device_error()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_pack_sign_nchw_rsign_ragged_channels_streamed(dtype):
    """RSign on the TMA-streamed pack: 40 channels (the second word holds 8),
    72 pixels per image (whole 16-byte rows for both dtypes)."""
    d = dev()
    shape = (3, 40, 8, 9)
    n, c, h, w = shape
    x = workloads.normal(shape, 1.0, 977).to(dtype)
    beta = _beta(c, 131)
    x[1, 3, 0, 0] = beta[3].to(dtype)
    packed = bnn.empty_packed_nhwc(n, c, h, w, d)
    bnn.bnn_pack_sign_nchw_rsign(x.to(d), beta.to(d), packed)
    torch.cuda.synchronize()
    cw = (c + 31) // 32
    r = oracle.rsign_pm1(x, beta, axis=1)
    want = oracle.pack_pm1(np.ascontiguousarray(r.transpose(0, 2, 3, 1)).reshape(-1, c))[:, :cw]
    assert np.array_equal(u32(packed).reshape(-1, cw), want)
    assert_no_device_error()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", [(2, 64, 8, 8), (3, 40, 6, 6), (1, 33, 5, 7)])
def test_pack_sign_nchw_nonfinite(shape, dtype):
    """NaN -> +1, +inf -> +1, -inf -> -1, signed zeros and subnormals, on the
    streamed pack (whole 16-byte rows) and the register kernel (the rest)."""
    n, c, h, w = shape
    x = workloads.random_with_edges(n * c, h * w, seed=7 * sum(shape), dtype=dtype, edge_fraction=0.3,
                                    finite=False).reshape(shape).contiguous()
    out = bnn.empty_packed_nhwc(n, c, h, w, dev())
    bnn.bnn_pack_sign_nchw(x.to(dev()), out)
    assert np.array_equal(u32(out), expected_nhwc(x))
