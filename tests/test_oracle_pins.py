"""Pins for the CPU oracle: checks against what the pages and the mathematics fix.

None of these compares the oracle with itself.  Each check is one of: a value
the pages fix (or a hand-computed answer to an exercise they pose), a closed
form, an invariant, brute force on tiny inputs, or a special case that reduces
to an independent library routine (torch float64 matmul / conv2d /
batch_norm, numpy mean).

The checks are written as functions of the oracle's functions so that
``test_oracle_mistakes.py`` can run them against oracles with a planted
mistake and show that every plausible slip fails at least one pin.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import workloads


def _popcount_u32(a: np.ndarray) -> np.ndarray:
    """Per-element popcount of a uint32 array (test-side, independent of the oracle)."""
    a = a.astype(np.uint64)
    return np.array([int(v).bit_count() for v in a.ravel()], dtype=np.int64).reshape(a.shape)


def all_pm1_vectors(K: int) -> np.ndarray:
    """All 2^K vectors in {-1, +1}^K as int8 rows."""
    rows = np.array(list(itertools.product([1, -1], repeat=K)), dtype=np.int8)
    return rows


# ---------------------------------------------------------------------------
# pin checks (each returns normally or raises AssertionError)
# ---------------------------------------------------------------------------

def check_identity_bruteforce(o, Ks=range(1, 11)):
    """eq. (6) of 'Extreme Quantization ...' (XNOR-Net) and the identity of
    'First Principles ...', section 1: <w,x> = K - 2 popcount(w xor x),
    over every pair of +1/-1 vectors for K = 1..10."""
    for K in Ks:
        V = all_pm1_vectors(K)
        s = o.matmul_pm1(V, V)                       # plain sum of products
        P = o.pack_pm1(V)                            # packed words
        d = np.zeros((len(V), len(V)), dtype=np.int64)
        for w in range(P.shape[1]):
            x = P[:, w][:, None] ^ P[:, w][None, :]
            d += _popcount_u32(x)
        assert np.array_equal(s.astype(np.int64), K - 2 * d), f"identity fails at K={K}"


def check_elementwise_xnor_form(o):
    """eq. (5): w_b x_b = 2 XNOR(w~, x~) - 1 with w~ = (w_b + 1)/2, all four cases."""
    for wb, xb in itertools.product([1, -1], repeat=2):
        s = o.matmul_pm1(np.array([[xb]], np.int8), np.array([[wb]], np.int8))[0, 0]
        wt, xt = (wb + 1) // 2, (xb + 1) // 2
        xnor = 1 if wt == xt else 0
        assert s == 2 * xnor - 1, (wb, xb, s)


def check_exercise1(o, golden):
    """Exercise 1 of 'Extreme Quantization ...' (hand-computed answer)."""
    g = json.load(open(os.path.join(golden, "exercise1.json")))
    w = np.array(g["w_b"], np.int8)
    x = np.array(g["x_b"], np.int8)
    assert o.matmul_pm1(x[None, :], w[None, :])[0, 0] == g["dot"]
    pw, px = o.pack_pm1(w[None, :]), o.pack_pm1(x[None, :])
    assert int(pw[0, 0]) == g["w_word"] and int(px[0, 0]) == g["x_word"]
    assert int(pw[0, 0] ^ px[0, 0]) == g["xor_word"]
    assert int(pw[0, 0] ^ px[0, 0]).bit_count() == g["popcount"]
    K = len(g["w_b"])
    assert K - 2 * g["popcount"] == g["dot"]


def check_pack_examples(o, golden):
    """Hand-computed packed words ('First Principles ...', section 1)."""
    g = json.load(open(os.path.join(golden, "pack_examples.json")))
    for case in g["cases"]:
        K = case["K"]
        b = np.ones((1, K), np.int8)
        b[0, case["negative_positions"]] = -1
        got = o.pack_pm1(b)
        assert got.shape[1] == len(case["words"]), (K, got.shape)
        assert [int(v) for v in got[0]] == case["words"], (K, got[0])


def check_sign_rule(o, golden):
    """Notation section of 'Extreme Quantization ...': +1 for x >= 0, -1 for x < 0."""
    g = json.load(open(os.path.join(golden, "sign_rule.json")))
    vals = np.array([float(v) for v, _ in g["cases"]], dtype=np.float32)
    want = np.array([e for _, e in g["cases"]], dtype=np.int8)
    assert np.array_equal(o.sign_pm1(vals), want), (o.sign_pm1(vals), want)
    # bf16 inputs are taken as stored (widened exactly)
    tb = torch.tensor(vals).to(torch.bfloat16)
    wb = np.where(np.isnan(tb.float().numpy()) | (tb.float().numpy() >= 0), 1, -1)
    assert np.array_equal(o.sign_pm1(tb), wb.astype(np.int8))


def check_pad_rule(o, Ks=(1, 31, 33, 63, 65, 1000), seed=0):
    """Pad bits encode +1 ('First Principles ...', section 1): pad bits are
    0 and the identity uses the true K whatever the padding width."""
    rng = np.random.default_rng(seed)
    for K in Ks:
        a = rng.choice(np.array([-1, 1], np.int8), size=(5, K))
        w = rng.choice(np.array([-1, 1], np.int8), size=(7, K))
        s = o.matmul_pm1(a, w).astype(np.int64)
        for extra in (0, 4, 8):
            ld = o.ld_words(K) + extra
            pa, pw = o.pack_pm1(a, ld), o.pack_pm1(w, ld)
            # pad bits of the last partial word and every pad word are zero
            nbits = ld * 32
            for r in range(pa.shape[0]):
                bits = sum(int(v) << (32 * i) for i, v in enumerate(pa[r]))
                assert bits >> K == 0, (K, extra)
            d = np.zeros((5, 7), np.int64)
            for i in range(ld):
                d += _popcount_u32(pa[:, i][:, None] ^ pw[:, i][None, :])
            assert np.array_equal(s, K - 2 * d), (K, extra)
            assert nbits >= K
        # 64-bit words see the same bytes (little-endian view of the uint32 rows)
        p64 = o.pack_pm1(a).view(np.uint64)
        d64 = np.zeros((5, 5), np.int64)
        for i in range(p64.shape[1]):
            x = p64[:, i][:, None] ^ p64[:, i][None, :]
            d64 += np.array([int(v).bit_count() for v in x.ravel()]).reshape(5, 5)
        assert np.array_equal(o.matmul_pm1(a, a).astype(np.int64), K - 2 * d64)


def check_ld_words(o):
    """ceil(K/32) words rounded up to a multiple of 4 (16-byte rows)."""
    table = {1: 4, 31: 4, 32: 4, 33: 4, 128: 4, 129: 8, 576: 20, 1000: 32, 4096: 128, 8192: 256}
    for K, want in table.items():
        assert o.ld_words(K) == want, (K, o.ld_words(K), want)


def check_memory_ratio(o):
    """32x memory ('Binary Neural Network (BNN)' glossary; 'First Principles ...',
    section 2 table: 0.125 bytes per binary weight vs 4 for FP32)."""
    for K in (128, 1024, 4096, 8192):
        packed_bytes = o.pack_pm1(np.ones((1, K), np.int8)).nbytes
        assert packed_bytes * 8 == K          # 0.125 B per weight
        assert (4 * K) // packed_bytes == 32


def check_alpha(o, seed=0):
    """alpha = (1/n) sum |w_i| (eq. (1) of 'Extreme Quantization ...'):
    closed form for constant magnitude, a hand value, and numpy's mean."""
    rng = np.random.default_rng(seed)
    for K in (1, 7, 1000):
        for c in (0.25, 3.0):
            w = (c * rng.choice([-1.0, 1.0], size=(3, K))).astype(np.float32)
            assert np.allclose(o.alpha(w), c, rtol=0, atol=0), (K, c)
    w = np.array([[1.0, -2.0, 3.0, -4.0]], np.float32)
    assert o.alpha(w)[0] == 2.5
    w = rng.standard_normal((17, 333)).astype(np.float32)
    ref = np.abs(w.astype(np.float64)).mean(axis=1)
    assert np.allclose(o.alpha(w), ref, rtol=1e-14, atol=0)


def check_matmul_library(o, seed=0):
    """Special case that reduces to a library routine: torch float64 matmul on
    the +1/-1 tensors is exact (|s| <= K < 2^53)."""
    rng = np.random.default_rng(seed)
    for (M, N, K) in [(1, 1, 1), (3, 5, 7), (64, 256, 1000), (33, 17, 65), (8, 9, 4096)]:
        a = rng.choice(np.array([-1, 1], np.int8), size=(M, K))
        w = rng.choice(np.array([-1, 1], np.int8), size=(N, K))
        ref = torch.from_numpy(a.astype(np.float64)) @ torch.from_numpy(w.astype(np.float64)).T
        assert np.array_equal(o.matmul_pm1(a, w), ref.numpy().astype(np.int32)), (M, N, K)
    # asymmetric operands so a transposed operand cannot pass
    a = rng.choice(np.array([-1, 1], np.int8), size=(4, 9))
    w = rng.choice(np.array([-1, 1], np.int8), size=(6, 9))
    s = o.matmul_pm1(a, w)
    for m in range(4):
        for n in range(6):
            assert s[m, n] == int(np.dot(a[m].astype(np.int64), w[n].astype(np.int64)))


def check_closed_forms(o, seed=0):
    """W = X gives K on the diagonal; W = -X gives -K; all +1 gives K;
    Sylvester-Hadamard rows are orthogonal (0 off the diagonal)."""
    rng = np.random.default_rng(seed)
    K = 77
    x = rng.choice(np.array([-1, 1], np.int8), size=(6, K))
    s = o.matmul_pm1(x, x)
    assert np.all(np.diag(s) == K)
    assert np.all(np.diag(o.matmul_pm1(x, (-x).astype(np.int8))) == -K)
    assert np.all(o.matmul_pm1(np.ones((2, K), np.int8), np.ones((3, K), np.int8)) == K)
    H = np.array([[1]], np.int64)
    for _ in range(6):                                   # 64 x 64
        H = np.block([[H, H], [H, -H]])
    s = o.matmul_pm1(H.astype(np.int8), H.astype(np.int8))
    assert np.array_equal(s, 64 * np.eye(64, dtype=np.int32))


def check_conv_library(o, seed=0):
    """Binary convolution against torch float64 conv2d on +1/-1 tensors, the
    input padded with +1 (zero-padded real input, then sign)."""
    rng = np.random.default_rng(seed)
    for (n, c, h, w, co, stride, pad) in [(2, 3, 5, 6, 4, 1, 1), (1, 64, 9, 7, 5, 1, 1),
                                          (2, 33, 8, 8, 3, 2, 1), (1, 2, 4, 4, 2, 1, 0)]:
        x = rng.choice(np.array([-1, 1], np.int8), size=(n, c, h, w))
        f = rng.choice(np.array([-1, 1], np.int8), size=(co, c, 3, 3))
        xt = F.pad(torch.from_numpy(x.astype(np.float64)), (pad, pad, pad, pad), value=1.0)
        ref = F.conv2d(xt, torch.from_numpy(f.astype(np.float64)), stride=stride)
        got = o.conv2d_pm1(x, f, stride, pad)
        assert np.array_equal(got, ref.numpy().astype(np.int32)), (n, c, h, w, co, stride, pad)
    # 1x1 kernels with stride (the downsampling projection), no padding
    for (n, c, h, w, co, stride) in [(2, 40, 9, 7, 5, 2), (1, 64, 8, 8, 3, 2), (2, 3, 5, 5, 4, 1), (1, 7, 6, 6, 2, 3)]:
        x = rng.choice(np.array([-1, 1], np.int8), size=(n, c, h, w))
        f = rng.choice(np.array([-1, 1], np.int8), size=(co, c, 1, 1))
        ref = F.conv2d(torch.from_numpy(x.astype(np.float64)), torch.from_numpy(f.astype(np.float64)), stride=stride)
        assert np.array_equal(o.conv2d_pm1(x, f, stride, 0), ref.numpy().astype(np.int32)), (n, c, h, w, co, stride)
    # closed form: all +1 input and filters give 9*c everywhere, padding included
    x = np.ones((1, 5, 4, 4), np.int8)
    f = np.ones((2, 5, 3, 3), np.int8)
    assert np.all(o.conv2d_pm1(x, f, 1, 1) == 45)


def check_bn(o, seed=0):
    """BatchNorm before re-binarisation ('Binary Neural Network (BNN)' glossary,
    BatchNorm paragraph): identity parameters reduce to sign(alpha*s); a
    negative gamma flips the decision; values agree with torch's inference
    batch_norm in float64."""
    rng = np.random.default_rng(seed)
    N, K = 64, 99
    s = (K - 2 * rng.integers(0, K + 1, size=(10, N))).astype(np.int32)
    a = rng.uniform(0.5, 1.5, N).astype(np.float32)
    one, zero = np.ones(N, np.float32), np.zeros(N, np.float32)
    # gamma=1, beta=0, mean=0, var+eps=1 -> alpha*s; s is odd so never 0
    got = o.bn_sign(s, a, one, zero, zero, one - np.float32(0.0), 0.0)
    assert np.array_equal(got, np.where(s >= 0, 1, -1).astype(np.int8))
    g = rng.uniform(0.5, 1.5, N).astype(np.float32)
    b = (0.1 * rng.standard_normal(N)).astype(np.float32)
    mu = rng.standard_normal(N).astype(np.float32)
    var = rng.uniform(0.5, 2.0, N).astype(np.float32)
    eps = 1e-5
    v = o.bn_value(s, a, g, b, mu, var, eps)
    x = torch.from_numpy(a.astype(np.float64) * s.astype(np.float64))
    ref = F.batch_norm(x, torch.from_numpy(mu.astype(np.float64)),
                       torch.from_numpy(var.astype(np.float64)),
                       torch.from_numpy(g.astype(np.float64)),
                       torch.from_numpy(b.astype(np.float64)), training=False, eps=eps)
    assert np.allclose(v, ref.numpy(), rtol=1e-12, atol=1e-12)
    flip = o.bn_sign(s, a, -g, -b, mu, var, eps)
    base = o.bn_sign(s, a, g, b, mu, var, eps)
    vv = o.bn_value(s, a, g, b, mu, var, eps)
    nz = vv != 0
    assert np.array_equal(flip[nz], -base[nz])


def check_mlp_library(o, seed=0):
    """A small fully binary MLP against a torch float64 composition of sign,
    matmul, inference batch_norm and the alpha scale."""
    rng = np.random.default_rng(seed)
    B, D = 16, 96
    x0 = rng.standard_normal((B, D)).astype(np.float32)
    ws = [rng.standard_normal((D, D)).astype(np.float32) for _ in range(3)]
    bns = []
    for _ in range(2):
        bns.append((rng.uniform(0.5, 1.5, D).astype(np.float32),
                    (0.1 * rng.standard_normal(D)).astype(np.float32),
                    rng.standard_normal(D).astype(np.float32),
                    rng.uniform(0.5, 2.0, D).astype(np.float32), 1e-5))
    acts, logits = o.mlp_forward(x0, ws, bns)

    def tsign(t):
        return torch.where(t >= 0, 1.0, -1.0).to(torch.float64)

    h = tsign(torch.from_numpy(x0))
    for l, w in enumerate(ws):
        wt = torch.from_numpy(w)
        al = wt.double().abs().mean(dim=1)
        s = h @ tsign(wt).T
        if l < len(ws) - 1:
            g, b, mu, var, eps = bns[l]
            y = F.batch_norm(al.float().double() * s, torch.from_numpy(mu).double(),
                             torch.from_numpy(var).double(), torch.from_numpy(g).double(),
                             torch.from_numpy(b).double(), training=False, eps=eps)
            h = tsign(y)
            assert np.array_equal(acts[l + 1], h.numpy().astype(np.int8)), l
        else:
            assert np.allclose(logits, (al * s).numpy(), rtol=1e-13, atol=0)


def check_binary_weight_product(o):
    """eq. (1)-(2) of 'Extreme Quantization ...' (binary weights, real x):
    brute force by the case split of eq. (2) for K <= 6, the closed form for a
    constant x, torch float64 matmul, and the reduction to the binary product
    when x itself is +1/-1."""
    rng = np.random.default_rng(11)
    for K in range(1, 7):
        V = all_pm1_vectors(K)
        x = rng.standard_normal(K)
        y = o.binary_weight_product(V, x)
        for r, w in enumerate(V):
            ref = 0.0
            for i in range(K):
                ref = ref + (x[i] if w[i] == 1 else -x[i])      # eq. (2), term by term
            assert abs(y[r] - ref) <= 1e-12 * np.abs(x).sum(), (K, r)
    w = np.where(rng.random((9, 300)) < 0.4, -1, 1).astype(np.int8)
    c = 0.75
    y = o.binary_weight_product(w, np.full(300, c))
    assert np.array_equal(y, c * (300 - 2 * (w == -1).sum(axis=1)))
    x = rng.standard_normal(300)
    ref = (torch.from_numpy(w).double() @ torch.from_numpy(x)).numpy()
    assert np.allclose(o.binary_weight_product(w, x), ref, rtol=0, atol=1e-12 * np.abs(x).sum())
    xb = np.where(rng.random(300) < 0.5, -1, 1).astype(np.int8)
    assert np.array_equal(o.binary_weight_product(w, xb).astype(np.int64), o.gemv_pm1(w, xb).astype(np.int64))



def check_ternary_examples(o, golden):
    """Hand-computed ternary quantisation, packing and add/skip/sub sums
    ('Extreme Quantization ...', eq. (7) and eq. (9); 'First Principles ...',
    the op-per-element and memory tables)."""
    g = json.load(open(os.path.join(golden, "ternary_examples.json")))
    for c in g["quantize_eq9"]:
        t, _ = o.ternary_quantize(np.array(c["w"], np.float32))
        assert t.tolist() == c["t"], (c["w"], t)
    for c in g["quantize_eq7"]:
        t, _ = o.ternary_quantize(np.array(c["w"], np.float32), c["delta"])
        assert t.tolist() == c["t"], (c["w"], t)
    for c in g["pack"]:
        K = c["K"]
        t = np.zeros(K, np.int8)
        if "t" in c:
            t[:] = c["t"]
        else:
            for k, v in c["t_nonzero"].items():
                t[int(k)] = v
        got = o.pack_ternary(t)
        assert [int(v) for v in got[0]] == c["words"], (K, [hex(int(v)) for v in got[0]])
    for c in g["product"]:
        got = o.ternary_product(np.array([c["t"]], np.int8), np.array(c["x"]))
        assert int(got[0]) == c["sum"], (c, got)


def check_ternary_quantizer(o):
    """eq. (9) against closed forms, a library mean and eq. (7):
    * gamma is the entrywise mean |w| of the whole matrix (torch float64 mean);
    * weights of equal magnitude quantise to their signs (w / gamma = +-1);
    * eq. (9) equals eq. (7) with Delta = gamma / 2 on random matrices (the
      threshold form and the round-and-clip form agree away from exact ties);
    * scaling W by a power of two changes nothing (gamma scales with it);
    * RoundClip closed forms: halves to even, clipping at +-1;
    * packed row length: the fewest multiples of 4 words holding 2 K bits."""
    rng = np.random.default_rng(21)
    w = (rng.standard_normal((7, 333)) * np.array([1, 0.01, 3, 1, 1, 0.5, 2])[:, None]).astype(np.float32)
    gl = torch.from_numpy(w).double().abs().mean().item()
    assert abs(o.ternary_gamma(w) - gl) <= 1e-15 * gl
    t9, g9 = o.ternary_quantize(w)
    assert abs(g9 - gl) <= 1e-15 * gl
    t7, _ = o.ternary_quantize(w, delta=g9 / 2)
    assert np.array_equal(t9, t7)
    assert set(np.unique(t9).tolist()) == {-1, 0, 1}
    assert np.all(t9[np.abs(w) > 1.5 * g9] == np.sign(w[np.abs(w) > 1.5 * g9]))     # clipped
    for e in (-3, 5):
        assert np.array_equal(o.ternary_quantize(w * np.float32(2.0 ** e))[0], t9)
    c = np.float32(0.3)
    ws = np.where(rng.random((5, 50)) < 0.5, -c, c).astype(np.float32)
    ts, gs = o.ternary_quantize(ws)
    assert abs(gs - float(c)) <= 1e-15 and np.array_equal(ts, np.sign(ws).astype(np.int8))
    v = np.array([0.5, -0.5, 1.5, -1.5, 2.5, -2.5, 0.49, -0.51, 0.0, 7.0])
    assert o.round_clip(v, -1, 1).tolist() == [0, 0, 1, -1, 1, -1, 0, -1, 0, 1]
    for K in range(1, 300):
        words = 4
        while words * 32 < 2 * K:
            words += 4
        assert o.ternary_ld_words(K) == words, K
    assert o.ternary_ld_words(4096) * 4 / 4096 == 0.25    # 2 bits per weight (pages: ~0.2 B at 1.58 bits)


def check_ternary_product(o):
    """The add/skip/sub sum against brute force over every ternary vector for
    K <= 4 (as a sum of products), torch int64 matmul, the binary product
    when no weight is 0, and the dequantised output's scale."""
    rng = np.random.default_rng(23)
    for K in range(1, 5):
        T = np.array(list(itertools.product([-1, 0, 1], repeat=K)), dtype=np.int8)
        x = rng.integers(-128, 128, K)
        got = o.ternary_product(T, x)
        for r in range(len(T)):
            ref = 0
            for k in range(K):
                ref += int(T[r, k]) * int(x[k])
            assert int(got[r]) == ref, (K, T[r], x)
    t = rng.integers(-1, 2, (40, 1000)).astype(np.int8)
    x = rng.integers(-128, 128, 1000)
    ref = (torch.from_numpy(t).long() @ torch.from_numpy(x).long()).numpy()
    assert np.array_equal(o.ternary_product(t, x), ref)
    tb = np.where(rng.random((9, 300)) < 0.5, -1, 1).astype(np.int8)
    xb = np.where(rng.random(300) < 0.5, -1, 1).astype(np.int8)
    assert np.array_equal(o.ternary_product(tb, xb), o.gemv_pm1(tb, xb).astype(np.int64))
    acc, y = o.ternary_gemv_i8(t, x, 0.25, 8.0)
    assert np.array_equal(acc, ref) and np.array_equal(y, 2.0 * ref.astype(np.float64))



def check_rsign(o, golden):
    """RSign (the survey's ReActNet row) as sign(x - beta_c): hand-computed
    cases, the comparison form x < beta on random and special values, beta = 0
    reducing to the Notation sign, invariance under a common exact shift, and
    the channel axis against explicit loops."""
    g = json.load(open(os.path.join(golden, "rsign_rule.json")))
    x = np.array([float(a) for a, _, _ in g["cases"]], np.float32)
    b = np.array([float(c) for _, c, _ in g["cases"]], np.float32)
    want = [e for *_, e in g["cases"]]
    got = [int(o.rsign_pm1(np.array([xi]), np.array([bi]))[0]) for xi, bi in zip(x, b)]
    assert got == want, (got, want)
    rng = np.random.default_rng(31)
    xs = rng.standard_normal((6, 40)).astype(np.float32)
    xs[0, :8] = [0.0, -0.0, np.inf, -np.inf, np.nan, 1e-45, -1e-45, 0.25]
    bs = rng.standard_normal(40).astype(np.float32)
    bs[:4] = [0.0, 0.0, np.inf, -np.inf]
    with np.errstate(invalid="ignore"):
        cmp = np.where(xs < bs[None, :], -1, 1).astype(np.int8)
    assert np.array_equal(o.rsign_pm1(xs, bs, axis=1), cmp)
    assert np.array_equal(o.rsign_pm1(xs, np.zeros(40, np.float32), axis=1), o.sign_pm1(xs))
    xi = rng.integers(-50, 50, (5, 30)).astype(np.float32)
    bi = rng.integers(-50, 50, 30).astype(np.float32)
    assert np.array_equal(o.rsign_pm1(xi + 7, bi + 7, axis=1), o.rsign_pm1(xi, bi, axis=1))
    x4 = rng.standard_normal((2, 3, 4, 5)).astype(np.float32)
    b4 = rng.standard_normal(3).astype(np.float32)
    r4 = o.rsign_pm1(x4, b4, axis=1)
    for n in range(2):
        for c in range(3):
            for h in range(4):
                for w in range(5):
                    assert r4[n, c, h, w] == (-1 if x4[n, c, h, w] < b4[c] else 1)



def check_multibit(o):
    """Bit planes and the two multi-bit products of the survey's DoReFa-Net and
    ABC-Net rows: plane reconstruction and a hand example; the integer product
    against brute force and against the bit-serial identity
    sum 2^(b+b') popcount(a_b AND w_b') evaluated on Python integers; the
    all-ones closed form; the binary-bases product against brute force, its
    single-basis case (the +1/-1 product) and bilinearity in the scales."""
    assert o.bit_planes(np.array([5, 0, 7]), 3).tolist() == [[1, 0, 1], [0, 0, 1], [1, 0, 1]]
    rng = np.random.default_rng(41)
    x = rng.integers(0, 16, (3, 7))
    pl = o.bit_planes(x, 4)
    assert np.array_equal(sum((1 << bb) * pl[bb].astype(np.int64) for bb in range(4)), x)
    for ka, kw, M, N, K in [(1, 1, 3, 4, 9), (2, 3, 4, 3, 33), (4, 2, 2, 5, 70), (8, 8, 2, 2, 40)]:
        a = rng.integers(0, 1 << ka, (M, K))
        w = rng.integers(0, 1 << kw, (N, K))
        got = o.bitserial_product(a, w)
        for m in range(M):
            for n in range(N):
                ref = 0
                for k in range(K):
                    ref += int(a[m, k]) * int(w[n, k])
                assert int(got[m, n]) == ref
                bits = 0
                for b1 in range(ka):
                    for b2 in range(kw):
                        am = sum(((int(a[m, k]) >> b1) & 1) << k for k in range(K))
                        wm = sum(((int(w[n, k]) >> b2) & 1) << k for k in range(K))
                        bits += (1 << (b1 + b2)) * (am & wm).bit_count()
                assert bits == ref
    assert np.all(o.bitserial_product(np.full((2, 10), 7), np.full((3, 10), 3)) == 7 * 3 * 10)
    J, I, M, N, K = 2, 3, 3, 4, 21
    h = np.where(rng.random((J, M, K)) < 0.5, -1, 1).astype(np.int8)
    b = np.where(rng.random((I, N, K)) < 0.5, -1, 1).astype(np.int8)
    al = rng.uniform(0.1, 1.0, (I, N))
    be = rng.uniform(0.1, 1.0, J)
    got = o.binary_bases_product(h, b, al, be)
    for m in range(M):
        for n in range(N):
            ref = 0.0
            for j in range(J):
                for i in range(I):
                    ref += be[j] * al[i, n] * sum(int(h[j, m, k]) * int(b[i, n, k]) for k in range(K))
            assert abs(got[m, n] - ref) <= 1e-12 * (1 + abs(ref))
    one = o.binary_bases_product(h[:1], b[:1], np.ones((1, N)), np.ones(1))
    assert np.array_equal(one, o.matmul_pm1(h[0], b[0]).astype(np.float64))
    assert np.allclose(o.binary_bases_product(h, b, 2 * al, 3 * be), 6 * got, rtol=1e-14, atol=0)



def check_compositions(o):
    """The layer-level compositions the GPU tests compare against: alpha*s and
    gamma*(alpha*s) + beta by hand values (alpha on the channel axis), the
    XNOR-Net linear layer, the convolution with its affine epilogue (3x3 and
    1x1 strided) and the binary-weight GEMV against torch float64, and alpha
    rounded once to fp32."""
    assert o.scaled(np.array([[3, -5, 0]]), np.array([0.5, 2.0, 7.0])).tolist() == [[1.5, -10.0, 0.0]]
    assert o.scaled(np.array([[1, 1, 1], [2, 2, 2]]), np.array([1.0, 2.0, 3.0])).tolist() == [[1, 2, 3], [2, 4, 6]]
    assert o.affine(np.array([[4, -2]]), np.array([0.25, 0.5]), np.array([2.0, -1.0]),
                    np.array([-1.0, 0.5])).tolist() == [[1.0, 1.5]]
    # sign then pack: negatives at 0 and 4 (-0.0 is +1) -> bits 0 and 4
    assert o.pack_real(np.array([[-1.0, 0.0, 2.0, -0.0, -3.0]], np.float32)).tolist() == [[17, 0, 0, 0]]
    rng = np.random.default_rng(51)

    def tsign(t):
        return torch.where(t >= 0, 1.0, -1.0).to(torch.float64)

    x = rng.standard_normal((6, 70)).astype(np.float32)
    w = rng.standard_normal((9, 70)).astype(np.float32)
    s, a = o.binary_linear(x, w)
    xt, wt = torch.from_numpy(x), torch.from_numpy(w)
    assert np.array_equal(s, (tsign(xt) @ tsign(wt).T).numpy().astype(np.int32))
    assert np.allclose(a, wt.double().abs().mean(dim=1).numpy(), rtol=1e-15, atol=0)
    af = o.alpha_f32(w)
    assert af.dtype == np.float32
    assert np.all(np.abs(af.astype(np.float64) - a) <= np.spacing(af).astype(np.float64) / 2)
    for (n, c, h, wd, co, k, stride, pad) in [(2, 5, 7, 6, 4, 3, 1, 1), (1, 40, 9, 8, 3, 1, 2, 0), (2, 3, 6, 6, 2, 3, 2, 1)]:
        X = rng.standard_normal((n, c, h, wd)).astype(np.float32)
        Wc = rng.standard_normal((co, c, k, k)).astype(np.float32)
        g = rng.uniform(0.5, 1.5, co)
        b = rng.standard_normal(co) * 0.1
        s_c, y_c = o.conv_affine(X, Wc, g, b, stride, pad)
        xp = F.pad(tsign(torch.from_numpy(X)), (pad, pad, pad, pad), value=1.0)
        s_ref = F.conv2d(xp, tsign(torch.from_numpy(Wc)), stride=stride)
        a_ref = torch.from_numpy(Wc).double().abs().mean(dim=(1, 2, 3))
        y_ref = torch.from_numpy(g)[None, :, None, None] * (a_ref[None, :, None, None] * s_ref) \
            + torch.from_numpy(b)[None, :, None, None]
        assert np.array_equal(s_c, s_ref.numpy().astype(np.int32))
        assert np.allclose(y_c, y_ref.numpy(), rtol=1e-13, atol=1e-13)
        if k == 3:
            assert np.array_equal(o.conv3x3_affine(X, Wc, g, b, stride, pad)[1], y_c)
    xv = rng.standard_normal(70).astype(np.float32)
    a_bw, y_bw = o.binary_weight_gemv(w, xv)
    y_t = wt.double().abs().mean(dim=1) * (tsign(wt) @ torch.from_numpy(xv).double())
    assert np.allclose(a_bw, a, rtol=0, atol=0)
    assert np.allclose(y_bw, y_t.numpy(), rtol=1e-13, atol=1e-13 * np.abs(xv).sum())


ALL_CHECKS = [
    ("identity_bruteforce", lambda o, g: check_identity_bruteforce(o)),
    ("elementwise_xnor_form", lambda o, g: check_elementwise_xnor_form(o)),
    ("exercise1", check_exercise1),
    ("pack_examples", check_pack_examples),
    ("sign_rule", check_sign_rule),
    ("pad_rule", lambda o, g: check_pad_rule(o)),
    ("ld_words", lambda o, g: check_ld_words(o)),
    ("memory_ratio", lambda o, g: check_memory_ratio(o)),
    ("alpha", lambda o, g: check_alpha(o)),
    ("matmul_library", lambda o, g: check_matmul_library(o)),
    ("closed_forms", lambda o, g: check_closed_forms(o)),
    ("conv_library", lambda o, g: check_conv_library(o)),
    ("bn", lambda o, g: check_bn(o)),
    ("mlp_library", lambda o, g: check_mlp_library(o)),
    ("binary_weight_product", lambda o, g: check_binary_weight_product(o)),
    ("ternary_examples", check_ternary_examples),
    ("ternary_quantizer", lambda o, g: check_ternary_quantizer(o)),
    ("ternary_product", lambda o, g: check_ternary_product(o)),
    ("rsign", check_rsign),
    ("multibit", lambda o, g: check_multibit(o)),
    ("compositions", lambda o, g: check_compositions(o)),
]


@pytest.mark.parametrize("name,check", ALL_CHECKS, ids=[c[0] for c in ALL_CHECKS])
def test_oracle_pin(name, check, golden_dir):
    check(oracle, golden_dir)


def test_oracle_on_workload_shapes():
    """The tiny workload end to end through the oracle: shapes, ranges, parity of s."""
    t = workloads.tiny()
    s, al = oracle.binary_linear(t.X, t.W)
    assert s.shape == (64, 256) and al.shape == (256,)
    assert np.all(np.abs(s) <= t.K) and np.all((s - t.K) % 2 == 0)
    y = oracle.scaled(s, al)
    assert np.all(np.sign(y) == np.sign(s))
