"""Ternary weights ("Extreme Quantization: Binary, Ternary & 1-bit LLMs",
eq. (7) and BitNet b1.58 eq. (9)) and their product with int8 activations,
through the C ABI, against the oracle.

Bars: the packed codes bit-exact (eq. (9) keeps +-1 exactly where
|w| > gamma / 2: the kernel decides it as w >= the smallest fp32 above
gamma / 2, the oracle by RoundClip in fp64; gamma is summed in a different
order on the two sides, so an element within 1e-12 relative of gamma / 2 may
take either code -- none does in these draws, and the test says how many it
exempted); gamma within one fp32 ulp; the int32
product exact; y_f32 = fp32(fp32(w_scale * x_scale) * acc) within two
roundings of the float64 product (|err| <= 2^-22 |y|)."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
import xnor_popcount_gemm_bnn_b200 as bnn
from gpu_util import assert_no_device_error, dev, u32

pytestmark = pytest.mark.gpu


def unpack_codes(Q: np.ndarray, K: int) -> np.ndarray:
    """[rows, ld] uint32 -> [rows, ld * 16] 2-bit codes (test-side reader of the layout)."""
    Q = Q.astype(np.uint64)
    sh = (2 * np.arange(16, dtype=np.uint64))[None, None, :]
    return ((Q[:, :, None] >> sh) & np.uint64(3)).reshape(Q.shape[0], -1).astype(np.int64)


def gpu_pack(W: torch.Tensor, delta=None, ldq=None, gamma=True, ld_w=None):
    d = dev()
    rows, K = W.shape
    nw = bnn.bnn_ternary_ld_words(K)
    ldq = nw if ldq is None else ldq
    codes = torch.full((rows, ldq), 0x12345678, dtype=torch.int32, device=d)
    g = torch.full((1,), float("nan"), dtype=torch.float32, device=d) if gamma else None
    if ld_w is None:
        Wd = W.to(d)
    else:
        buf = torch.full((rows, ld_w), float("nan"), dtype=W.dtype, device=d)
        buf[:, :K] = W.to(d)
        Wd = buf[:, :K]
    bnn.bnn_ternary_pack(Wd, codes, gamma_out=g, delta=delta, K=K)
    torch.cuda.synchronize()
    return codes, g


def check_codes(codes: torch.Tensor, W, delta=None):
    rows, K = W.shape
    nw = oracle.ternary_ld_words(K)
    t_ref, g_ref = oracle.ternary_quantize(W, delta)
    want = unpack_codes(oracle.pack_ternary(t_ref), K)
    got_words = u32(codes)
    got = unpack_codes(got_words[:, :nw], K)
    assert want.shape == got.shape
    diff = want != got
    exempt = 0
    if delta is None and diff.any():
        wd = oracle._f32(W).astype(np.float64)
        near = np.zeros_like(diff)
        near[:, :K] = np.abs(np.abs(wd) - g_ref / 2) <= 1e-12 * g_ref
        ok_alt = np.zeros_like(diff)
        ok_alt[:, :K] = (got[:, :K] == 1) | (got[:, :K] == 1 + np.sign(wd).astype(np.int64))
        exempt = int((diff & near & ok_alt).sum())
        diff &= ~(near & ok_alt)
    bad = np.argwhere(diff)
    assert bad.size == 0, f"{len(bad)} codes differ, first {bad[:5].tolist()}"
    if codes.shape[1] > nw:       # words past the packed row are never written
        assert np.all(got_words[:, nw:] == 0x12345678)
    return g_ref, exempt


SHAPES = [(1, 1), (5, 17), (64, 1000), (65, 33), (300, 4096), (33, 12288), (3, 100000)]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("rows,K", SHAPES)
def test_ternary_pack_absmean(rows, K, dtype):
    """eq. (9): codes and gamma."""
    W = workloads.normal((rows, K), 0.02, rows * 7 + K).to(dtype)
    codes, g = gpu_pack(W)
    g_ref, _ = check_codes(codes, W)
    gf = np.float32(g.item())
    assert abs(float(gf) - g_ref) <= float(np.spacing(np.float32(g_ref))), (gf, g_ref)
    assert_no_device_error()


@pytest.mark.parametrize("delta", [0.0, 0.01, 0.5, math.inf])
def test_ternary_pack_threshold(delta):
    """eq. (7) with a given Delta (gamma still reported)."""
    W = workloads.normal((70, 999), 0.02, 31)
    W[0, :5] = torch.tensor([0.01, -0.01, 0.0, -0.0, 0.5])
    codes, g = gpu_pack(W, delta=delta)
    check_codes(codes, W, delta)
    assert abs(g.item() - oracle.ternary_gamma(W)) <= 1e-7 * oracle.ternary_gamma(W)
    codes2, _ = gpu_pack(W, delta=delta, gamma=False)      # no gamma, no workspace
    assert torch.equal(codes, codes2)
    assert_no_device_error()


def test_ternary_pack_strided_and_padded():
    """Row strides larger than K on both sides; words past the row untouched."""
    W = workloads.normal((37, 250), 1.0, 41)
    codes, _ = gpu_pack(W, ldq=bnn.bnn_ternary_ld_words(250) + 8, ld_w=264)
    check_codes(codes, W)
    assert_no_device_error()


def test_ternary_pack_special_values():
    """All-zero W (gamma 0, every weight 0), exact ties at gamma / 2 (round
    half to even: 0), NaN weights (0), infinities."""
    z = torch.zeros(4, 40)
    codes, g = gpu_pack(z)
    assert g.item() == 0.0
    assert np.all(u32(codes) == 0x55555555)
    tie = torch.tensor([[1.0, 3.0, -1.0, -3.0]])     # gamma 2: +-1 are ties -> 0, +-3 -> +-1
    codes, g = gpu_pack(tie)
    assert g.item() == 2.0
    assert unpack_codes(u32(codes), 4)[0, :4].tolist() == [1, 2, 1, 0]
    check_codes(codes, tie)
    nan = workloads.normal((3, 64), 1.0, 43)
    nan[1, 5] = float("nan")
    codes, _ = gpu_pack(nan, delta=0.5)
    check_codes(codes, nan, 0.5)
    assert unpack_codes(u32(codes), 64)[1, 5] == 1
    inf = torch.tensor([[math.inf, -math.inf, 1.0, 0.0]])
    codes, _ = gpu_pack(inf, delta=0.5)
    assert unpack_codes(u32(codes), 4)[0, :4].tolist() == [2, 0, 2, 1]
    assert_no_device_error()


def test_ternary_pack_decode_workload():
    """The decode weights W [11008, 4096] ~ N(0, 0.02), eq. (9), every code."""
    g = workloads.ternary()
    codes, gam = gpu_pack(g.W)
    g_ref, exempt = check_codes(codes, g.W)
    assert abs(gam.item() - g_ref) <= float(np.spacing(np.float32(g_ref)))
    t_ref, _ = oracle.ternary_quantize(g.W)
    zero_frac = float((t_ref == 0).mean())
    assert 0.25 < zero_frac < 0.37, zero_frac       # |w| <= 0.4 sigma for a normal: about 31%
    print(f"exempted near-tie codes: {exempt}")
    assert_no_device_error()


# ---------------------------------------------------------------------------
# product
# ---------------------------------------------------------------------------

def upload_codes(t: np.ndarray, ld=None) -> torch.Tensor:
    Q = oracle.pack_ternary(t, ld)
    return torch.from_numpy(Q.view(np.int32).copy()).to(dev())


def check_product(y_i32, y_f32, t, x, w_scale=1.0, x_scale=1.0):
    acc, y_ref = oracle.ternary_gemv_i8(t, x.numpy(), w_scale, x_scale)
    if y_i32 is not None:
        got = y_i32.cpu().numpy().astype(np.int64)
        bad = np.nonzero(got != acc)[0]
        assert bad.size == 0, f"{bad.size} rows differ, first {bad[:5]}: {got[bad[:5]]} vs {acc[bad[:5]]}"
    if y_f32 is not None:
        got = y_f32.cpu().numpy().astype(np.float64)
        err = np.abs(got - y_ref)
        assert np.all(err <= 2.0 ** -22 * np.abs(y_ref)), float((err / np.maximum(np.abs(y_ref), 1e-300)).max())


def random_ternary(N, K, seed, p_zero=0.3):
    rng = np.random.default_rng(seed)
    return np.where(rng.random((N, K)) < p_zero, 0, np.where(rng.random((N, K)) < 0.5, -1, 1)).astype(np.int8)


# flags 7 launch 4 rows per warp, the other flags 8 rows per warp; both for
# every shape.
@pytest.mark.parametrize("N,K", [(1, 1), (5, 17), (64, 1000), (65, 33), (300, 4096), (100, 4100),
                                 (129, 8192), (33, 12288), (40, 11008), (17, 16384), (300, 16400),
                                 (70, 50000), (3, 98304)])
@pytest.mark.parametrize("flags", [0, 1, 3, 7])
def test_ternary_gemv_shapes(N, K, flags):
    d = dev()
    t = random_ternary(N, K, N * 31 + K)
    x = workloads.int8_uniform((K,), K + 3)
    Q = upload_codes(t)
    yi = torch.full((N,), -7, dtype=torch.int32, device=d)
    yf = torch.full((N,), float("nan"), dtype=torch.float32, device=d)
    ws = torch.tensor([0.0123], device=d)
    xs = torch.tensor([0.5], device=d)
    bnn.bnn_ternary_gemv_i8(Q, x.to(d), K, y_i32=yi, y_f32=yf, w_scale=ws, x_scale=xs, flags=flags)
    torch.cuda.synchronize()
    check_product(yi, yf, t, x, np.float32(0.0123), 0.5)
    assert_no_device_error()


def test_ternary_gemv_unaligned_x_and_strided_codes():
    """x at an odd byte offset (the byte path of the staging), codes with a
    row stride past the packed row."""
    d = dev()
    N, K = 77, 3000
    t = random_ternary(N, K, 5)
    x = workloads.int8_uniform((K,), 6)
    buf = torch.zeros(K + 16, dtype=torch.int8, device=d)
    buf[3:3 + K] = x.to(d)
    Q = upload_codes(t, ld=oracle.ternary_ld_words(K) + 12)
    yi = torch.empty(N, dtype=torch.int32, device=d)
    bnn.bnn_ternary_gemv_i8(Q, buf[3:3 + K], K, y_i32=yi)
    torch.cuda.synchronize()
    check_product(yi, None, t, x)
    assert_no_device_error()


def test_ternary_gemv_extremes():
    """Largest magnitudes: every weight -1 against x = -128 (acc = 128 K) and
    +1 against 127, at K = 65536 (fp32(acc) still exact); all-zero weights."""
    d = dev()
    K = 65536
    for tv, xv in ((-1, -128), (1, 127), (-1, 127), (0, -128)):
        t = np.full((9, K), tv, np.int8)
        x = torch.full((K,), xv, dtype=torch.int8)
        yi = torch.empty(9, dtype=torch.int32, device=d)
        yf = torch.empty(9, dtype=torch.float32, device=d)
        bnn.bnn_ternary_gemv_i8(upload_codes(t), x.to(d), K, y_i32=yi, y_f32=yf)
        torch.cuda.synchronize()
        assert np.all(yi.cpu().numpy() == tv * xv * K)
        assert np.all(yf.cpu().numpy() == np.float32(tv * xv * K))
    assert_no_device_error()


def test_ternary_decode_end_to_end():
    """The decode shape end to end on the GPU: eq. (9) pack of W [11008, 4096]
    then the int8 product with gamma as w_scale, against the oracle's
    quantiser and add/skip/sub sum."""
    d = dev()
    g = workloads.ternary()
    codes, gam = gpu_pack(g.W)
    t_ref, g_ref = oracle.ternary_quantize(g.W)
    xs = torch.tensor([0.031], device=d)
    yi = torch.empty(g.N, dtype=torch.int32, device=d)
    yf = torch.empty(g.N, dtype=torch.float32, device=d)
    bnn.bnn_ternary_gemv_i8(codes, g.x.to(d), g.K, y_i32=yi, y_f32=yf, w_scale=gam, x_scale=xs,
                            flags=bnn.BNN_GEMV_WEIGHTS_STATIC)
    torch.cuda.synchronize()
    check_product(yi, yf, t_ref, g.x, float(np.float32(gam.item())), float(np.float32(0.031)))
    assert_no_device_error()


@pytest.mark.parametrize("use_graph", [False, True])
def test_ternary_gemv_static_weights_chain(use_graph):
    """Six GEMVs with BNN_GEMV_WEIGHTS_STATIC, each x made by a torch kernel
    from the previous GEMV's output: the dependency wait must order every
    read of x after the kernel that wrote it."""
    d = dev()
    N = K = 2048
    L = 6
    ts = [random_ternary(N, K, 900 + l) for l in range(L)]
    Qs = [upload_codes(t) for t in ts]
    x0 = workloads.int8_uniform((K,), 77)
    xs = [x0.to(d)] + [torch.empty(K, dtype=torch.int8, device=d) for _ in range(L)]
    ys = [torch.empty(N, dtype=torch.int32, device=d) for _ in range(L)]
    torch.cuda.synchronize()

    def chain():
        for l in range(L):
            bnn.bnn_ternary_gemv_i8(Qs[l], xs[l], K, y_i32=ys[l], flags=bnn.BNN_GEMV_WEIGHTS_STATIC)
            xs[l + 1].copy_(torch.remainder(ys[l], 256).sub(128).to(torch.int8))

    if use_graph:
        gr = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            chain()
        torch.cuda.current_stream().wait_stream(s)
        for t in xs[1:]:
            t.zero_()
        with torch.cuda.graph(gr):
            chain()
        for t in xs[1:]:
            t.zero_()
        gr.replay()
    else:
        chain()
    torch.cuda.synchronize()
    x = x0.numpy().astype(np.int64)
    for l in range(L):
        acc = oracle.ternary_product(ts[l], x)
        assert np.array_equal(ys[l].cpu().numpy().astype(np.int64), acc), l
        x = np.remainder(acc, 256) - 128
    assert_no_device_error()


def test_ternary_gemv_independent_all_flags():
    """All three flags over independent inputs and outputs: every result
    exact; repeated writes of one y keep stream order (the last call wins)."""
    d = dev()
    N, K, L = 1000, 4096, 6
    ts = [random_ternary(N, K, 950 + l) for l in range(L)]
    Qs = [upload_codes(t) for t in ts]
    xh = [workloads.int8_uniform((K,), 960 + l) for l in range(L)]
    xd = [x.to(d) for x in xh]
    ys = [torch.empty(N, dtype=torch.int32, device=d) for _ in range(L)]
    y_shared = torch.empty(N, dtype=torch.int32, device=d)
    torch.cuda.synchronize()
    for rep in range(3):
        for l in range(L):
            bnn.bnn_ternary_gemv_i8(Qs[l], xd[l], K, y_i32=ys[l], flags=7)
    for l in range(L):
        bnn.bnn_ternary_gemv_i8(Qs[l], xd[l], K, y_i32=y_shared, flags=3)
    torch.cuda.synchronize()
    for l in range(L):
        check_product(ys[l], None, ts[l], xh[l])
    check_product(y_shared, None, ts[-1], xh[-1])
    assert_no_device_error()
