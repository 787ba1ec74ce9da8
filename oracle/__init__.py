"""CPU oracle for the binary (+1/-1) matrix product -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA path
(``xnor_popcount_gemm_bnn_b200``) and never imports it.

What it computes is the plain definition of the method, with +1/-1 values
materialised and integers multiplied and added (``bnn_oracle.c``), and the
real-valued epilogues evaluated in float64 here with numpy:

* sign -- "Extreme Quantization: Binary, Ternary & 1-bit LLMs", Notation
  (sign(x) = +1 for x >= 0, -1 for x < 0) and eq. (4) of the XNOR-Net section.
* packed encoding -- "First Principles: Why Binary Ops Can Be Exponentially
  Faster", section "1. Arithmetic: MAC -> XNOR + popcount" (bit 0 is +1,
  bit 1 is -1, pad bits encode +1).
* alpha and the scaled product -- "Extreme Quantization ...", Binary Neural
  Networks section, eq. (1): y = alpha * (w_b^T x), alpha = (1/n) sum |w_i|.
* per-channel sign threshold (RSign) -- "State of the Art Survey (2016 ->
  2026)", classic CNN BNN table (ReActNet): sign(x - beta_c).
* ternary weights -- "Extreme Quantization ...", eq. (7) (threshold Delta)
  and eq. (9) (BitNet b1.58: RoundClip(W / gamma, -1, 1), gamma = mean |W|
  over the matrix); "First Principles ...", the op-per-element table
  (ternary: add / skip / sub), with int8 activations (the BitNet section:
  activations quantised to INT8).
* multi-bit products -- "State of the Art Survey ...", classic CNN BNN table:
  DoReFa-Net bit planes (unsigned k-bit codes, the integer product) and
  ABC-Net binary bases (a weighted sum of +1/-1 products).
* BatchNorm before re-binarisation -- "Binary Neural Network (BNN)" glossary
  page, the BatchNorm paragraph (BN stabilises the inputs to each binarised
  layer; per-filter alpha multiplies the binary product).  The pages give no
  BN formula; the oracle uses standard inference BatchNorm on alpha*s,
  evaluated in float64 in the order ((alpha*s - mean) / sqrt(var + eps)) *
  gamma + beta, and maps a result >= 0 to +1 (the same tie rule as sign).

Readings of the pages made here (all listed with reasons in the design notes):
sign(-0.0) = +1, sign(NaN) = +1, bit j of word w is element 32*w + j, rows
padded to a multiple of 4 words, alpha over the true K from the real weights,
convolution padding value +1, RoundClip rounding halves to even, ternary
codes t + 1 packed 2 bits per weight (16 per word, least significant first,
pad code 1), BN decisions taken with alpha rounded to fp32
(the precision the product stores alpha in).

Parity pins for every function live in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        i64, p = ctypes.c_int64, ctypes.c_void_p
        lib.oracle_ld_words.argtypes = [i64]
        lib.oracle_ld_words.restype = i64
        lib.oracle_sign_f32.argtypes = [p, i64, p]
        lib.oracle_pack_pm1.argtypes = [p, i64, i64, p, i64]
        lib.oracle_alpha_f32.argtypes = [p, i64, i64, p]
        lib.oracle_matmul_pm1.argtypes = [p, p, i64, i64, i64, p]
        lib.oracle_conv2d_pm1.argtypes = [p, i64, i64, i64, i64, p, i64, i64, i64, i64, p]
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
        for name in ("oracle_sign_f32", "oracle_pack_pm1", "oracle_alpha_f32",
                     "oracle_matmul_pm1", "oracle_conv2d_pm1", "oracle_set_num_threads"):
            getattr(lib, name).restype = None
        _LIB = lib
    return _LIB


def _f32(x) -> np.ndarray:
    """Accept numpy arrays or CPU torch tensors (fp32 or bf16; bf16 widens exactly)."""
    if hasattr(x, "detach"):
        import torch
        t = x.detach().cpu()
        if t.dtype != torch.float32:
            t = t.to(torch.float32)
        x = t.numpy()
    return np.ascontiguousarray(x, dtype=np.float32)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(_lib().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Threads for the C loops (timing only; no result depends on it)."""
    _lib().oracle_set_num_threads(int(n))


def ld_words(K: int) -> int:
    """Words per packed row: ceil(K/32) rounded up to a multiple of 4."""
    return int(_lib().oracle_ld_words(int(K)))


def sign_pm1(x) -> np.ndarray:
    """int8 +1/-1 of the same shape: -1 exactly where x < 0 (Notation, eq. (4))."""
    xf = _f32(x)
    out = np.empty(xf.shape, dtype=np.int8)
    _lib().oracle_sign_f32(_ptr(xf), xf.size, _ptr(out))
    return out



def rsign_pm1(x, beta, axis: int = -1) -> np.ndarray:
    """int8 +1/-1: sign(x - beta_c) with a learned threshold beta_c per channel
    (ReActNet's RSign, "State of the Art Survey (2016 -> 2026)", classic CNN
    BNN table: a per-channel reshape of the activation distribution before
    the sign).  beta has one entry per index of x along `axis` and is
    broadcast over the other axes.  The difference is taken in float64 and
    mapped by the Notation rule of "Extreme Quantization ..." (-1 exactly
    where x - beta < 0; so x = beta gives +1, and NaN anywhere gives +1)."""
    xf = _f32(x).astype(np.float64)
    b = _f32(beta).astype(np.float64).reshape(-1)
    ax = axis % xf.ndim
    assert b.size == xf.shape[ax], (b.size, xf.shape, ax)
    shape = [1] * xf.ndim
    shape[ax] = b.size
    with np.errstate(invalid="ignore"):
        v = xf - b.reshape(shape)
        return np.where(v < 0.0, -1, 1).astype(np.int8)

def pack_pm1(b: np.ndarray, ld: int | None = None) -> np.ndarray:
    """Pack a [rows, K] int8 +1/-1 matrix into uint32 [rows, ld] words."""
    b = np.ascontiguousarray(b, dtype=np.int8)
    if b.ndim == 1:
        b = b[None, :]
    rows, K = b.shape
    ld = ld_words(K) if ld is None else int(ld)
    out = np.empty((rows, ld), dtype=np.uint32)
    _lib().oracle_pack_pm1(_ptr(b), rows, K, _ptr(out), ld)
    return out


def pack_real(x, ld: int | None = None) -> np.ndarray:
    """sign() then pack, for a real [rows, K] matrix."""
    return pack_pm1(sign_pm1(x), ld)


def alpha(w) -> np.ndarray:
    """float64 [rows]: mean |w| over each row's true K (eq. (1))."""
    wf = _f32(w)
    if wf.ndim == 1:
        wf = wf[None, :]
    rows, K = wf.shape
    out = np.empty(rows, dtype=np.float64)
    _lib().oracle_alpha_f32(_ptr(wf), rows, K, _ptr(out))
    return out


def alpha_f32(w) -> np.ndarray:
    """alpha rounded once to fp32 (round to nearest)."""
    return alpha(w).astype(np.float32)


def matmul_pm1(a: np.ndarray, w: np.ndarray) -> np.ndarray:
    """int32 [M, N] = a @ w^T for int8 +1/-1 a [M, K] and w [N, K]."""
    a = np.ascontiguousarray(a, dtype=np.int8)
    w = np.ascontiguousarray(w, dtype=np.int8)
    if a.ndim == 1:
        a = a[None, :]
    M, K = a.shape
    N, K2 = w.shape
    assert K == K2, (K, K2)
    s = np.empty((M, N), dtype=np.int32)
    _lib().oracle_matmul_pm1(_ptr(a), _ptr(w), M, N, K, _ptr(s))
    return s


def gemv_pm1(w: np.ndarray, x: np.ndarray) -> np.ndarray:
    """int32 [N] = w @ x for int8 +1/-1 w [N, K] and x [K]."""
    return matmul_pm1(np.asarray(x, dtype=np.int8)[None, :], w)[0]


def binary_weight_product(w: np.ndarray, x) -> np.ndarray:
    """float64 [N]: sum_i sign(w_ni) * x_i for int8 +1/-1 w [N, K] and a real
    x [K] -- "Extreme Quantization: Binary, Ternary & 1-bit LLMs", Binary
    Neural Networks, eq. (1) without alpha, with eq. (2): each term is +x_i
    where the weight is +1 and -x_i where it is -1 (no multiplication).  The
    terms are added in float64."""
    w = np.asarray(w, dtype=np.int8)
    xd = np.asarray(x, dtype=np.float64)
    return np.where(w > 0, xd[None, :], -xd[None, :]).sum(axis=1)


def binary_weight_gemv(w_real, x_real) -> tuple[np.ndarray, np.ndarray]:
    """eq. (1): y = alpha * (w_b^T x) per output row with binary weights and
    real activations; returns (alpha float64, y float64).  x is taken as
    stored (bf16 inputs widened exactly)."""
    wb = sign_pm1(w_real)
    a = alpha(w_real)
    return a, scaled(binary_weight_product(wb, _f32(x_real)), a)



# ---------------------------------------------------------------------------
# ternary weights (BitNet b1.58) times int8 activations
# ---------------------------------------------------------------------------

def ternary_ld_words(K: int) -> int:
    """Words per packed ternary row: 2 bits per weight, 16 weights per uint32
    word, rounded up to a multiple of 4 words (whole 16-byte units, as the
    binary rows)."""
    K = int(K)
    if K < 1:
        return -1
    words = -(-K // 16)
    return -(-words // 4) * 4


def ternary_gamma(w) -> float:
    """eq. (9) of "Extreme Quantization: Binary, Ternary & 1-bit LLMs", BitNet
    b1.58: gamma = ||W||_1 / (n m), the mean absolute value over every entry
    of the matrix (one scale per tensor), in float64."""
    wd = _f32(w).astype(np.float64)
    return float(np.abs(wd).sum() / wd.size)


def round_clip(v, lo: float, hi: float) -> np.ndarray:
    """RoundClip(v, lo, hi) of eq. (9): round to the nearest integer, then
    clip to [lo, hi].  The pages do not say how halves round; this takes
    round half to even (numpy.rint), so +-0.5 go to 0."""
    return np.clip(np.rint(np.asarray(v, dtype=np.float64)), lo, hi)


def ternary_quantize(w, delta: float | None = None) -> tuple[np.ndarray, float]:
    """Ternary weights in {-1, 0, +1} (int8, same shape as w) and gamma.

    delta None -- eq. (9), BitNet b1.58: W_t = RoundClip(W / gamma, -1, 1) with
    gamma = ternary_gamma(W), the division and rounding in float64.  An all-
    zero W has gamma = 0; its weights are all 0.
    delta given -- eq. (7), ternary quantisation with threshold Delta:
    +1 where w > Delta, 0 where |w| <= Delta, -1 where w < -Delta.
    gamma is returned in both cases (the scale of eq. (9))."""
    wd = _f32(w).astype(np.float64)
    g = ternary_gamma(w)
    if delta is None:
        if g == 0.0:
            return np.zeros(wd.shape, dtype=np.int8), g
        return round_clip(wd / g, -1, 1).astype(np.int8), g
    d = float(delta)
    t = np.where(wd > d, 1, np.where(wd < -d, -1, 0))
    return t.astype(np.int8), g


def pack_ternary(t: np.ndarray, ld: int | None = None) -> np.ndarray:
    """Pack a [rows, K] matrix of ternary weights into uint32 [rows, ld].
    Weight k of a row is the 2-bit code t + 1 (0 for -1, 1 for 0, 2 for +1)
    at bits 2k, 2k+1 of the row's bit string, least significant bit first:
    bits 2(k mod 16) of word k // 16.  Positions past K hold code 1 (weight
    0).  The pages give the density (about 0.2 bytes per weight, log2(3) =
    1.58 bits) but no layout; this is the plainest addressable one."""
    t = np.ascontiguousarray(t, dtype=np.int8)
    if t.ndim == 1:
        t = t[None, :]
    rows, K = t.shape
    ld = ternary_ld_words(K) if ld is None else int(ld)
    codes = np.ones((rows, ld * 16), dtype=np.uint64)
    codes[:, :K] = (t.astype(np.int64) + 1).astype(np.uint64)
    shifts = (2 * np.arange(16, dtype=np.uint64))[None, None, :]
    words = (codes.reshape(rows, ld, 16) << shifts).sum(axis=2)
    return words.astype(np.uint32)


def ternary_product(t: np.ndarray, x) -> np.ndarray:
    """int64 [N]: sum_k t_nk * x_k for ternary t [N, K] and integer x [K], by
    the rule of the op-per-element table in "First Principles: Why Binary Ops
    Can Be Exponentially Faster" (ternary: add / skip / sub): x_k is added
    where the weight is +1, skipped where it is 0, subtracted where it is -1."""
    t = np.asarray(t, dtype=np.int8)
    if t.ndim == 1:
        t = t[None, :]
    xi = np.asarray(x, dtype=np.int64)
    terms = np.where(t > 0, xi[None, :], np.where(t < 0, -xi[None, :], 0))
    return terms.sum(axis=1)


def ternary_gemv_i8(t: np.ndarray, x_q, w_scale: float = 1.0, x_scale: float = 1.0):
    """Ternary weights times an int8 activation vector ("Extreme Quantization
    ...", BitNet: activations quantised to INT8; BitNet b1.58: ternary
    weights).  Returns (acc int64 [N], y float64 [N]) with
    y = w_scale * x_scale * acc, the dequantised product (w_scale is gamma of
    eq. (9); x_scale the activation's quantisation step, which the pages
    leave to the caller)."""
    acc = ternary_product(t, x_q)
    return acc, float(w_scale) * float(x_scale) * acc.astype(np.float64)



# ---------------------------------------------------------------------------
# multi-bit products: bit planes (DoReFa-Net) and binary bases (ABC-Net)
# ---------------------------------------------------------------------------

def bit_planes(x_u, k: int) -> np.ndarray:
    """uint8 [k, *shape]: plane b holds bit b of the unsigned k-bit codes
    x_u (0 <= x < 2^k), so x = sum_b 2^b * plane_b ("State of the Art Survey
    (2016 -> 2026)", classic CNN BNN table, DoReFa-Net: low-bit weights and
    activations, bit-convolution)."""
    x = np.asarray(x_u, dtype=np.int64)
    assert k >= 1 and x.min(initial=0) >= 0 and x.max(initial=0) < (1 << k)
    return np.stack([(x >> b) & 1 for b in range(k)]).astype(np.uint8)


def bitserial_product(a_u, w_u) -> np.ndarray:
    """int64 [M, N]: sum_k a[m, k] * w[n, k] for unsigned integer codes
    a [M, K] and w [N, K] -- the product a bit-serial kernel computes as
    sum over plane pairs (b, b') of 2^(b+b') * popcount(a_b AND w_b')
    (DoReFa-Net's bit-convolution, same table).  Written as the plain sum of
    products."""
    a = np.asarray(a_u, dtype=np.int64)
    w = np.asarray(w_u, dtype=np.int64)
    return (a[:, None, :] * w[None, :, :]).sum(axis=2)


def binary_bases_product(h_pm1, b_pm1, alpha, beta) -> np.ndarray:
    """float64 [M, N]: sum_j sum_i beta_j * alpha_i[n] * (H_j B_i^T)[m, n]
    for activations approximated by J binary bases, A ~ sum_j beta_j H_j
    (H_j in {-1, +1}^[M, K]), and weights by I bases, W ~ sum_i alpha_i B_i
    (B_i in {-1, +1}^[N, K], alpha_i per output channel) ("State of the Art
    Survey ...", classic CNN BNN table, ABC-Net: approximate full precision
    with K binary bases).  Each H_j B_i^T is a +1/-1 product (eq. (6))."""
    h = np.asarray(h_pm1, dtype=np.int8)
    b = np.asarray(b_pm1, dtype=np.int8)
    al = np.asarray(alpha, dtype=np.float64)
    be = np.asarray(beta, dtype=np.float64).reshape(-1)
    J, M, K = h.shape
    I, N, K2 = b.shape
    assert K == K2 and al.shape == (I, N) and be.shape == (J,)
    y = np.zeros((M, N), dtype=np.float64)
    for j in range(J):
        for i in range(I):
            y += be[j] * al[i][None, :] * matmul_pm1(h[j], b[i]).astype(np.float64)
    return y

def conv2d_pm1(x: np.ndarray, f: np.ndarray, stride: int = 1, pad: int = 1) -> np.ndarray:
    """int32 NCHW output of a square-kernel convolution on +1/-1 tensors,
    padded taps reading +1."""
    x = np.ascontiguousarray(x, dtype=np.int8)
    f = np.ascontiguousarray(f, dtype=np.int8)
    n, c, h, wd = x.shape
    cout, c2, kk, kk2 = f.shape
    assert c == c2 and kk == kk2
    oh = (h + 2 * pad - kk) // stride + 1
    ow = (wd + 2 * pad - kk) // stride + 1
    out = np.empty((n, cout, oh, ow), dtype=np.int32)
    _lib().oracle_conv2d_pm1(_ptr(x), n, c, h, wd, _ptr(f), cout, kk, stride, pad, _ptr(out))
    return out


# ---------------------------------------------------------------------------
# epilogues, float64
# ---------------------------------------------------------------------------

def scaled(s: np.ndarray, alpha_n: np.ndarray) -> np.ndarray:
    """alpha_n * s_mn in float64; alpha indexes the last axis (output channel)."""
    return np.asarray(alpha_n, dtype=np.float64) * np.asarray(s, dtype=np.float64)


def affine(s: np.ndarray, alpha_n, gamma, beta) -> np.ndarray:
    """gamma_n * (alpha_n * s) + beta_n in float64 (last axis = channel)."""
    a = np.asarray(alpha_n, dtype=np.float64)
    g = np.asarray(gamma, dtype=np.float64)
    b = np.asarray(beta, dtype=np.float64)
    return g * (a * np.asarray(s, dtype=np.float64)) + b


def bn_value(s: np.ndarray, alpha_n_f32, gamma, beta, mean, var, eps: float) -> np.ndarray:
    """Inference BatchNorm of alpha*s in float64: ((alpha*s - mean)/sqrt(var+eps))*gamma + beta."""
    a = np.asarray(alpha_n_f32, dtype=np.float32).astype(np.float64)
    x = a * np.asarray(s, dtype=np.float64)
    mu = np.asarray(mean, dtype=np.float32).astype(np.float64)
    v = np.asarray(var, dtype=np.float32).astype(np.float64)
    g = np.asarray(gamma, dtype=np.float32).astype(np.float64)
    b = np.asarray(beta, dtype=np.float32).astype(np.float64)
    return (x - mu) / np.sqrt(v + float(eps)) * g + b


def bn_sign(s, alpha_n_f32, gamma, beta, mean, var, eps: float) -> np.ndarray:
    """int8 +1/-1: +1 where the BatchNorm value is >= 0 (tie goes to +1, as sign(0))."""
    y = bn_value(s, alpha_n_f32, gamma, beta, mean, var, eps)
    return np.where(y >= 0.0, 1, -1).astype(np.int8)


# ---------------------------------------------------------------------------
# whole layers, composed from the definitions above
# ---------------------------------------------------------------------------

def binary_linear(x_real, w_real):
    """XNOR-Net linear layer: s = sign(x) sign(W)^T, alpha from the real W.

    Returns (s int32 [M, N], alpha float64 [N])."""
    a = sign_pm1(x_real)
    if a.ndim == 1:
        a = a[None, :]
    wb = sign_pm1(w_real)
    return matmul_pm1(a, wb), alpha(w_real)


def conv_affine(x_real, w_real, gamma, beta, stride: int = 1, pad: int = 1):
    """Binary convolution (any square kernel in w_real [cout, cin, k, k]) with
    per-output-channel alpha over the filter's cin*k*k weights and an affine
    epilogue.  Returns (s int32 NCHW, y float64 NCHW)."""
    return conv3x3_affine(x_real, w_real, gamma, beta, stride, pad)


def conv3x3_affine(x_real, w_real, gamma, beta, stride: int = 1, pad: int = 1):
    """Binary 3x3 convolution with per-output-channel alpha and an affine epilogue
    (the code holds for any square kernel size).

    Returns (s int32 NCHW, y float64 NCHW)."""
    xb = sign_pm1(x_real)
    fb = sign_pm1(w_real)
    cout = fb.shape[0]
    s = conv2d_pm1(xb, fb, stride, pad)
    a = alpha(_f32(w_real).reshape(cout, -1))
    y = affine(np.moveaxis(s, 1, -1), a, gamma, beta)
    return s, np.moveaxis(y, -1, 1)


def mlp_forward(x0_real, ws_real, bns):
    """Fully binary MLP: sign the input, then for each layer the +1/-1 product
    with sign(W_l); layers before the last re-binarise through BatchNorm of
    alpha*s; the last layer returns alpha*s in float64.

    ``bns`` is a list of (gamma, beta, mean, var, eps), one per hidden layer.
    Returns (list of int8 +1/-1 activations entering each layer, logits)."""
    a = sign_pm1(x0_real)
    if a.ndim == 1:
        a = a[None, :]
    acts = [a]
    L = len(ws_real)
    logits = None
    for l, w in enumerate(ws_real):
        s = matmul_pm1(a, sign_pm1(w))
        al = alpha(w)
        if l < L - 1:
            g, b, mu, var, eps = bns[l]
            a = bn_sign(s, al.astype(np.float32), g, b, mu, var, eps)
            acts.append(a)
        else:
            logits = scaled(s, al)
    return acts, logits
