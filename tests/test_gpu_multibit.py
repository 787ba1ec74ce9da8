"""Multi-bit products on bit planes against the oracle ("State of the Art
Survey (2016 -> 2026)", classic CNN BNN table): DoReFa-Net's unsigned low-bit
codes (bit planes, the integer product, bit-exact) and ABC-Net's binary bases
(a weighted sum of +1/-1 products, fp32 within the bound the header derives)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import xnor_popcount_gemm_bnn_b200 as bnn
from gpu_util import assert_no_device_error, assert_scaled_close, dev, u32

pytestmark = pytest.mark.gpu

U = 2.0 ** -24


def _codes(rows, K, bits, seed):
    return workloads.codes((rows, K), bits, seed)


def _planes_ref(codes: np.ndarray, bits: int, ld: int) -> np.ndarray:
    """Plane-interleaved packed planes from the oracle's bit planes and packer:
    a plane bit 1 is packed as bit 1 (the -1 of the +1/-1 encoding)."""
    pl = oracle.bit_planes(codes, bits)                       # [bits, rows, K] of {0, 1}
    rows = codes.shape[0]
    out = np.zeros((rows * bits, ld), dtype=np.uint32)
    for p in range(bits):
        out[p::bits] = oracle.pack_pm1(1 - 2 * pl[p].astype(np.int8), ld)
    return out


def _pack_planes(codes: torch.Tensor, bits: int, K: int):
    rows = codes.shape[0]
    planes = torch.empty(rows * bits, bnn.bnn_packed_ld_words(K), dtype=torch.int32, device=dev())
    bnn.bnn_pack_bit_planes(codes.to(dev()), bits, planes, K)
    return planes


@pytest.mark.parametrize("rows,K,bits", [(1, 1, 1), (3, 31, 2), (17, 100, 3), (64, 1000, 4), (5, 4097, 8),
                                         (40, 513, 2), (9, 16, 1)])
def test_pack_bit_planes(rows, K, bits):
    codes = _codes(rows, K, bits, rows * 7 + K)
    # high bits above `bits` must be ignored: set them in some codes
    if bits < 8:
        noisy = codes | (workloads.codes(codes.shape, 1, K + 3) << 7)
    else:
        noisy = codes
    got = _pack_planes(noisy, bits, K)
    torch.cuda.synchronize()
    ref = _planes_ref(codes.numpy(), bits, bnn.bnn_packed_ld_words(K))
    assert np.array_equal(u32(got), ref)


def test_pack_bit_planes_unaligned_rows():
    """Codes whose rows are not 16-byte aligned take the byte path."""
    rows, K, bits = 11, 300, 3
    big = _codes(rows, K + 5, bits, 99)
    view = big[:, 3:3 + K]                                       # row stride K + 5, offset 3
    d = big.to(dev())[:, 3:3 + K]
    planes = torch.empty(rows * bits, bnn.bnn_packed_ld_words(K), dtype=torch.int32, device=dev())
    bnn.bnn_pack_bit_planes(d, bits, planes, K)
    torch.cuda.synchronize()
    assert np.array_equal(u32(planes), _planes_ref(view.contiguous().numpy(), bits, bnn.bnn_packed_ld_words(K)))


SHAPES = [(1, 1, 1), (7, 5, 33), (130, 300, 1000), (257, 129, 4097), (64, 256, 128), (300, 260, 96)]


@pytest.mark.parametrize("a_bits,w_bits", [(1, 1), (2, 2), (1, 2), (2, 1), (3, 2), (4, 4), (4, 1), (2, 4)])
@pytest.mark.parametrize("M,N,K", SHAPES)
def test_bitserial_gemm(M, N, K, a_bits, w_bits, tc_engine):
    a = _codes(M, K, a_bits, 11 * M + K + a_bits)
    w = _codes(N, K, w_bits, 13 * N + K + w_bits)
    A = _pack_planes(a, a_bits, K)
    W = _pack_planes(w, w_bits, K)
    alpha = workloads.normal((N,), 0.01, N + 5).abs() + 1e-3
    ad = alpha.to(dev())
    Ci = torch.empty(M, N, dtype=torch.int32, device=dev())
    Cf = torch.empty(M, N, dtype=torch.float32, device=dev())
    bnn.bnn_bitserial_gemm(A, a_bits, W, w_bits, K, ad, Ci, Cf)
    torch.cuda.synchronize()
    ref = oracle.bitserial_product(a.numpy(), w.numpy())
    assert np.array_equal(Ci.cpu().numpy().astype(np.int64), ref)
    # two roundings, fp32(acc) then fp32(alpha * acc): within the 1e-6 relative bar
    assert_scaled_close(Cf, oracle.scaled(ref, alpha.numpy().astype(np.float64)))
    assert_no_device_error()


def test_bitserial_gemm_int32_only_and_f32_only():
    M, N, K, ab, wb = 200, 300, 777, 2, 3
    a, w = _codes(M, K, ab, 1), _codes(N, K, wb, 2)
    A, W = _pack_planes(a, ab, K), _pack_planes(w, wb, K)
    ref = oracle.bitserial_product(a.numpy(), w.numpy())
    Ci = torch.empty(M, N, dtype=torch.int32, device=dev())
    bnn.bnn_bitserial_gemm(A, ab, W, wb, K, None, Ci, None)
    alpha = torch.full((N,), 0.5, device=dev())
    Cf = torch.empty(M, N, dtype=torch.float32, device=dev())
    bnn.bnn_bitserial_gemm(A, ab, W, wb, K, alpha, None, Cf)
    torch.cuda.synchronize()
    assert np.array_equal(Ci.cpu().numpy().astype(np.int64), ref)
    assert np.array_equal(Cf.cpu().numpy().astype(np.float64), 0.5 * ref)   # exact: ref < 2^24, alpha a power of 2


def test_bitserial_gemm_full_size_sampled_rows():
    """The bench workload (M = N = K = 4096, 2-bit activations x 2-bit
    weights) on every column of 24 sampled rows spanning all row tiles."""
    M = N = K = 4096
    ab = wb = 2
    a, w = _codes(M, K, ab, 41), _codes(N, K, wb, 42)
    A, W = _pack_planes(a, ab, K), _pack_planes(w, wb, K)
    Ci = torch.empty(M, N, dtype=torch.int32, device=dev())
    bnn.bnn_bitserial_gemm(A, ab, W, wb, K, None, Ci, None)
    torch.cuda.synchronize()
    got = Ci.cpu().numpy()
    rows = sorted(set(np.linspace(0, M - 1, 24).astype(int).tolist()) | {127, 128, 4095})
    an, wn = a.numpy(), w.numpy()
    for m in rows:
        assert np.array_equal(got[m].astype(np.int64), oracle.bitserial_product(an[m:m + 1], wn)[0]), f"row {m}"
    assert_no_device_error()


def test_bitserial_one_plane_equals_and_popcount_identity():
    """With 1-bit codes the product is popcount(a AND w): the DoReFa product of
    {0,1} planes, checked against the binary GEMM of the same bits through
    (K - s)/2 = popcount(a XOR w) and popcount(a) + popcount(w)."""
    M, N, K = 100, 130, 555
    a, w = _codes(M, K, 1, 5), _codes(N, K, 1, 6)
    A, W = _pack_planes(a, 1, K), _pack_planes(w, 1, K)
    Cb = torch.empty(M, N, dtype=torch.int32, device=dev())
    bnn.bnn_bitserial_gemm(A, 1, W, 1, K, None, Cb, None)
    S = torch.empty(M, N, dtype=torch.int32, device=dev())
    bnn.bnn_xnor_gemm(A, W, K, None, S, None)
    torch.cuda.synchronize()
    pa = a.numpy().astype(np.int64).sum(1)[:, None]
    pw = w.numpy().astype(np.int64).sum(1)[None, :]
    d = (K - S.cpu().numpy().astype(np.int64)) // 2
    assert np.array_equal(Cb.cpu().numpy().astype(np.int64), (pa + pw - d) // 2)


def test_bitserial_rejects():
    K = 64
    A = bnn.empty_packed(2 * 5, K, dev())
    W = bnn.empty_packed(3 * 5, K, dev())
    C = torch.empty(2, 3, dtype=torch.int32, device=dev())
    with pytest.raises(bnn.BnnError):
        bnn.bnn_bitserial_gemm(A, 5, W, 5, K, None, C, None)          # 5 planes: more than 4
    with pytest.raises(bnn.BnnError):
        bnn.bnn_bitserial_gemm(A[:8], 4, W[:12], 4, K, None, None, None)   # no output
    with pytest.raises(bnn.BnnError):
        bnn.bnn_bitserial_gemm(A[:8], 4, W[:12], 4, K, None, None, C.float())   # fp32 without alpha


# ---------------------------------------------------------------------------
# ABC-Net binary bases
# ---------------------------------------------------------------------------

def _pack_bases(h_real, J, rows, K):
    """Base j of row r packed at row r * J + j (strided views of one matrix)."""
    out = torch.empty(rows * J, bnn.bnn_packed_ld_words(K), dtype=torch.int32, device=dev())
    for j in range(J):
        bnn.bnn_pack_sign(h_real[j].to(dev()), out[j::J])
    return out


def _bases_case(M, N, K, J, I, seed):
    c = workloads.bases(M, N, K, J, I, seed)
    return c.h_real, c.b_real, c.alpha, c.beta


def _bases_reference(h_real, b_real, alpha, beta):
    h = oracle.sign_pm1(h_real.numpy())
    b = oracle.sign_pm1(b_real.numpy())
    y = oracle.binary_bases_product(h, b, alpha.numpy(), beta.numpy())
    J, I = h.shape[0], b.shape[0]
    mag = np.zeros_like(y)
    for j in range(J):
        for i in range(I):
            s = oracle.matmul_pm1(h[j], b[i]).astype(np.float64)
            mag += np.abs(float(beta[j]) * alpha.numpy()[i].astype(np.float64)[None, :] * s)
    return y, mag


@pytest.fixture(params=[bnn.BNN_GEMM_ENGINE_TENSOR, bnn.BNN_GEMM_ENGINE_TENSOR_I8], ids=["tensor", "tensor_i8"])
def tc_engine(request):
    """TENSOR: the e2m1 kernel in CTA pairs where M allows, else int8;
    TENSOR_I8: the int8 kernel for every shape."""
    with bnn.gemm_engine(request.param):
        yield request.param


@pytest.mark.parametrize("J,I", [(1, 1), (2, 3), (3, 3), (4, 2), (5, 8), (8, 1), (1, 4)])
@pytest.mark.parametrize("M,N,K", [(1, 1, 1), (7, 5, 33), (130, 300, 1000), (70, 129, 4097)])
def test_binary_bases_gemm(M, N, K, J, I, tc_engine):
    h_real, b_real, alpha, beta = _bases_case(M, N, K, J, I, M + N + K + 10 * J + I)
    H = _pack_bases(h_real, J, M, K)
    B = _pack_bases(b_real, I, N, K)
    Y = torch.full((M, N), float("nan"), dtype=torch.float32, device=dev())
    bnn.bnn_binary_bases_gemm(H, J, B, I, K, beta.to(dev()), alpha.to(dev()), Y)
    torch.cuda.synchronize()
    y_ref, mag = _bases_reference(h_real, b_real, alpha, beta)
    got = Y.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got))
    err = np.abs(got - y_ref)
    bound = (I + J + 2) * U * mag
    assert np.all(err <= bound), f"max err/bound {np.max(err / np.maximum(bound, 1e-300))}"
    assert_no_device_error()


_SHAPE_REFS = {}


@pytest.mark.parametrize("J", [1, 2, 4, 8])
@pytest.mark.parametrize("I", [1, 2, 4, 8])
def test_binary_bases_every_combine_shape(J, I, tc_engine):
    """Every (J', I') instance of the epilogue's per-shape combine (powers of
    two up to 8 bases a side), at a shape with several row and column tiles
    and ragged edges, against the oracle (computed once per (J, I))."""
    M, N, K = 200, 160, 300
    h_real, b_real, alpha, beta = _bases_case(M, N, K, J, I, 500 + 10 * J + I)
    H, B = _pack_bases(h_real, J, M, K), _pack_bases(b_real, I, N, K)
    Y = torch.full((M, N), float("nan"), dtype=torch.float32, device=dev())
    bnn.bnn_binary_bases_gemm(H, J, B, I, K, beta.to(dev()), alpha.to(dev()), Y)
    torch.cuda.synchronize()
    if (J, I) not in _SHAPE_REFS:
        _SHAPE_REFS[(J, I)] = _bases_reference(h_real, b_real, alpha, beta)
    y_ref, mag = _SHAPE_REFS[(J, I)]
    got = Y.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got))
    assert np.all(np.abs(got - y_ref) <= (I + J + 2) * U * mag)
    assert_no_device_error()


@pytest.mark.parametrize("col0,ld", [(0, 304), (1, 304), (0, 303), (3, 311)])
def test_binary_bases_strided_output(col0, ld, tc_engine):
    """Y as a column window of a wider buffer: row strides and start columns
    with and without 16-byte alignment (vector and scalar stores), and the
    columns around the window left untouched."""
    M, N, K, J, I = 300, 290, 700, 3, 2
    h_real, b_real, alpha, beta = _bases_case(M, N, K, J, I, 31 + col0 + ld)
    H, B = _pack_bases(h_real, J, M, K), _pack_bases(b_real, I, N, K)
    big = torch.full((M, ld), -7.0, dtype=torch.float32, device=dev())
    Y = big[:, col0:col0 + N]
    bnn.bnn_binary_bases_gemm(H, J, B, I, K, beta.to(dev()), alpha.to(dev()), Y)
    torch.cuda.synchronize()
    y_ref, mag = _bases_reference(h_real, b_real, alpha, beta)
    got = Y.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - y_ref) <= (I + J + 2) * U * mag)
    rest = torch.cat([big[:, :col0].flatten(), big[:, col0 + N:].flatten()])
    assert bool((rest == -7.0).all())
    assert_no_device_error()


def test_binary_bases_one_base_is_the_scaled_binary_product():
    """J = I = 1, beta = 1: the bases product is alpha * s of the binary GEMM."""
    M, N, K = 200, 300, 999
    h_real, b_real, alpha, _ = _bases_case(M, N, K, 1, 1, 77)
    beta = torch.ones(1)
    H, B = _pack_bases(h_real, 1, M, K), _pack_bases(b_real, 1, N, K)
    Y = torch.empty(M, N, dtype=torch.float32, device=dev())
    bnn.bnn_binary_bases_gemm(H, 1, B, 1, K, beta.to(dev()), alpha.to(dev()), Y)
    Yb = torch.empty(M, N, dtype=torch.float32, device=dev())
    bnn.bnn_xnor_gemm(H, B, K, alpha[0].contiguous().to(dev()), None, Yb)
    torch.cuda.synchronize()
    assert torch.equal(Y, Yb)


def test_binary_bases_rejects():
    K = 64
    H = bnn.empty_packed(9 * 2, K, dev())
    Y = torch.empty(2, 2, device=dev())
    with pytest.raises(bnn.BnnError):
        bnn.bnn_binary_bases_gemm(H, 9, H, 9, K, torch.ones(9, device=dev()), torch.ones(9, 2, device=dev()), Y)


# ---------------------------------------------------------------------------
# full outputs, repeated launches (race detectors): the tensor-core kernels
# against the independent popcount engine.  A sampled-row oracle check can
# miss a hand-off race that corrupts a few tiles in some launches; these
# compare every output of several launches.
# ---------------------------------------------------------------------------

def _and_popcount_reference(a, w, A, W, ab, wb, K):
    """sum_{b,b'} 2^(b+b') popcount(a_b AND w_b'), each plane pair from the
    popcount engine's +1/-1 product s: popcount(a_b AND w_b') =
    (popcount(a_b) + popcount(w_b') - (K - s) / 2) / 2."""
    d = dev()
    M, N = a.shape[0], w.shape[0]
    an, wn = a.to(d).to(torch.int64), w.to(d).to(torch.int64)
    ref = torch.zeros(M, N, dtype=torch.int64, device=d)
    S = torch.empty(M, N, dtype=torch.int32, device=d)
    with bnn.gemm_engine(bnn.BNN_GEMM_ENGINE_POPCOUNT):
        for b in range(ab):
            pa = ((an >> b) & 1).sum(1)
            for c in range(wb):
                pw = ((wn >> c) & 1).sum(1)
                bnn.bnn_xnor_gemm(A[b::ab], W[c::wb], K, None, S, None)
                ref += (1 << (b + c)) * ((pa[:, None] + pw[None, :] - (K - S.to(torch.int64)) // 2) // 2)
    return ref


@pytest.mark.parametrize("a_bits,w_bits", [(1, 1), (2, 2), (4, 4)])
def test_bitserial_full_output_repeated(a_bits, w_bits):
    M = N = K = 4096
    a, w = _codes(M, K, a_bits, 141), _codes(N, K, w_bits, 142)
    A, W = _pack_planes(a, a_bits, K), _pack_planes(w, w_bits, K)
    ref = _and_popcount_reference(a, w, A, W, a_bits, w_bits, K)
    C = torch.empty(M, N, dtype=torch.int32, device=dev())
    for rep in range(3):
        C.fill_(-1)
        bnn.bnn_bitserial_gemm(A, a_bits, W, w_bits, K, None, C, None)
        torch.cuda.synchronize()
        bad = int((C.to(torch.int64) != ref).sum())
        assert bad == 0, f"launch {rep}: {bad} outputs differ"
    assert_no_device_error()


@pytest.mark.parametrize("J,I", [(2, 2), (3, 3)])
def test_binary_bases_full_output_repeated(J, I):
    M = N = K = 2048
    h_real, b_real, alpha, beta = _bases_case(M, N, K, J, I, 7 * J + I)
    H, B = _pack_bases(h_real, J, M, K), _pack_bases(b_real, I, N, K)
    d = dev()
    al, be = alpha.to(d), beta.to(d)
    ref = torch.zeros(M, N, dtype=torch.float64, device=d)
    mag = torch.zeros_like(ref)
    S = torch.empty(M, N, dtype=torch.int32, device=d)
    with bnn.gemm_engine(bnn.BNN_GEMM_ENGINE_POPCOUNT):
        for j in range(J):
            for i in range(I):
                bnn.bnn_xnor_gemm(H[j::J], B[i::I], K, None, S, None)
                t = be[j].double() * al[i].double()[None, :] * S.double()
                ref += t
                mag += t.abs()
    Y = torch.empty(M, N, dtype=torch.float32, device=d)
    for rep in range(3):
        Y.fill_(float("nan"))
        bnn.bnn_binary_bases_gemm(H, J, B, I, K, be, al, Y)
        torch.cuda.synchronize()
        bad = int((((Y.double() - ref).abs() > (I + J + 2) * U * mag) | ~torch.isfinite(Y)).sum())
        assert bad == 0, f"launch {rep}: {bad} outputs outside the bound"
    assert_no_device_error()
