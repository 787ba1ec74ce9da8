"""Plant plausible mistakes in the oracle (on the CPU) and show that the pins
of ``test_oracle_pins.py`` catch every one of them.

Each mutant is the oracle with one function replaced by a numpy version that
carries a single slip: a wrong tie rule, a reversed bit order, a dropped term,
a transposed operand, a wrong pad value, a wrong divisor...
"""
import types

import numpy as np
import pytest

import oracle
from test_oracle_pins import ALL_CHECKS


def _mutant(**overrides):
    ns = types.SimpleNamespace(**{k: getattr(oracle, k) for k in dir(oracle) if not k.startswith("_")})
    for k, v in overrides.items():
        setattr(ns, k, v)
    # composite helpers must see the mutated primitives
    ns.mlp_forward = lambda x0, ws, bns: _mlp_with(ns, x0, ws, bns)
    return ns


def _mlp_with(o, x0, ws, bns):
    a = o.sign_pm1(x0)
    acts = [a]
    logits = None
    for l, w in enumerate(ws):
        s = o.matmul_pm1(a, o.sign_pm1(w))
        al = o.alpha(w)
        if l < len(ws) - 1:
            g, b, mu, var, eps = bns[l]
            a = o.bn_sign(s, al.astype(np.float32), g, b, mu, var, eps)
            acts.append(a)
        else:
            logits = o.scaled(s, al)
    return acts, logits


def _sign_gt(x):                       # 0 -> -1 (the glossary's reading)
    x = oracle._f32(x)
    return np.where(x > 0, 1, -1).astype(np.int8)


def _sign_bit(x):                      # sign-bit test: -0.0 -> -1
    x = oracle._f32(x)
    return np.where(np.signbit(x), -1, 1).astype(np.int8)


def _pack_msb(b, ld=None):             # bit order reversed inside a word
    b = np.atleast_2d(np.asarray(b, np.int8))
    rows, K = b.shape
    ld = oracle.ld_words(K) if ld is None else ld
    out = np.zeros((rows, ld), np.uint32)
    for r in range(rows):
        for k in range(K):
            if b[r, k] == -1:
                out[r, k // 32] |= np.uint32(1 << (31 - k % 32))
    return out


def _pack_inverted(b, ld=None):        # bit 1 for +1
    b = np.atleast_2d(np.asarray(b, np.int8))
    return oracle.pack_pm1((-b).astype(np.int8), ld)


def _ld_no_round(K):                   # rows not padded to 4 words
    return (int(K) + 31) // 32


def _alpha_padded(w):                  # divides by the padded length
    w = np.atleast_2d(oracle._f32(w)).astype(np.float64)
    K = w.shape[1]
    return np.abs(w).sum(axis=1) / (32 * oracle.ld_words(K))


def _alpha_noabs(w):                   # mean of w, not of |w|
    w = np.atleast_2d(oracle._f32(w)).astype(np.float64)
    return np.abs(w.sum(axis=1)) / w.shape[1]


def _matmul_transposed(a, w):          # reads w as [K, N] storage
    a = np.atleast_2d(np.asarray(a, np.int64))
    w = np.asarray(w, np.int64)
    N, K = w.shape
    wt = w.reshape(-1)[: N * K].reshape(K, N).T
    return (a @ wt.T).astype(np.int32)


def _matmul_drop_first(a, w):          # loop starts at k = 1
    a = np.atleast_2d(np.asarray(a, np.int64))
    w = np.asarray(w, np.int64)
    return (a[:, 1:] @ w[:, 1:].T).astype(np.int32)


def _conv_pad_minus(x, f, stride=1, pad=1):   # padded taps read -1
    import torch
    import torch.nn.functional as F
    xt = F.pad(torch.from_numpy(np.asarray(x, np.float64)), (pad,) * 4, value=-1.0)
    return F.conv2d(xt, torch.from_numpy(np.asarray(f, np.float64)), stride=stride).numpy().astype(np.int32)


def _conv_flipped(x, f, stride=1, pad=1):     # true convolution (flipped kernel)
    return oracle.conv2d_pm1(x, np.ascontiguousarray(np.asarray(f)[:, :, ::-1, ::-1]), stride, pad)


def _bn_value_no_gamma(s, a, g, b, mu, var, eps):
    return oracle.bn_value(s, a, np.ones_like(np.asarray(g)), b, mu, var, eps)


def _bn_value_mean_sign(s, a, g, b, mu, var, eps):
    return oracle.bn_value(s, a, g, b, -np.asarray(mu), var, eps)


def _bn_sign_strict(s, a, g, b, mu, var, eps):   # tie (value 0) goes to -1
    y = oracle.bn_value(s, a, g, b, mu, var, eps)
    return np.where(y > 0, 1, -1).astype(np.int8)


def _bw_sign_swapped(w, x):            # +x where the weight is -1 (encoding read backwards)
    w = np.asarray(w, np.int8)
    xd = np.asarray(x, np.float64)
    return np.where(w > 0, -xd[None, :], xd[None, :]).sum(axis=1)


def _bw_drop_last(w, x):               # the last term is lost
    w = np.asarray(w, np.int8)
    xd = np.asarray(x, np.float64)
    return np.where(w > 0, xd[None, :], -xd[None, :])[:, :-1].sum(axis=1)


def _bw_abs_x(w, x):                   # adds |x| instead of x
    w = np.asarray(w, np.int8)
    xd = np.abs(np.asarray(x, np.float64))
    return np.where(w > 0, xd[None, :], -xd[None, :]).sum(axis=1)



def _tern_gamma_noabs(w, delta=None):  # gamma from the mean of w, not of |w|
    wd = oracle._f32(w).astype(np.float64)
    g = abs(float(wd.mean())) or 1.0
    return oracle.round_clip(wd / g, -1, 1).astype(np.int8), g


def _tern_round_half_away(w, delta=None):   # halves round away from zero
    wd = oracle._f32(w).astype(np.float64)
    g = oracle.ternary_gamma(w)
    if g == 0.0:
        return np.zeros(wd.shape, np.int8), g
    q = wd / g
    return np.clip(np.sign(q) * np.floor(np.abs(q) + 0.5), -1, 1).astype(np.int8), g


def _tern_no_clip(w, delta=None):      # RoundClip without the clip
    wd = oracle._f32(w).astype(np.float64)
    g = oracle.ternary_gamma(w)
    if g == 0.0:
        return np.zeros(wd.shape, np.int8), g
    return np.rint(wd / g).astype(np.int8), g


def _tern_per_row_gamma(w, delta=None):     # one gamma per row instead of per matrix
    wd = np.atleast_2d(oracle._f32(w).astype(np.float64))
    g = np.abs(wd).mean(axis=1, keepdims=True)
    g[g == 0] = 1.0
    return oracle.round_clip(wd / g, -1, 1).astype(np.int8).reshape(np.shape(w)), float(g.mean())


def _tern_pack_codes_t(t, ld=None):    # stores t itself (two's complement bits), not t + 1
    t = np.atleast_2d(np.asarray(t, np.int8))
    rows, K = t.shape
    ld = oracle.ternary_ld_words(K) if ld is None else ld
    out = np.zeros((rows, ld), np.uint32)
    for r in range(rows):
        for k in range(K):
            out[r, k // 16] |= np.uint32((int(t[r, k]) & 3) << (2 * (k % 16)))
    return out


def _tern_pack_msb(t, ld=None):        # codes placed from the top of the word down
    t = np.atleast_2d(np.asarray(t, np.int8))
    rows, K = t.shape
    ld = oracle.ternary_ld_words(K) if ld is None else ld
    out = np.full((rows, ld), 0x55555555, np.uint32)
    for r in range(rows):
        for k in range(K):
            sh = 30 - 2 * (k % 16)
            w = int(out[r, k // 16]) & ~(3 << sh)
            out[r, k // 16] = np.uint32(w | ((int(t[r, k]) + 1) << sh))
    return out


def _tern_minus_as_skip(t, x):         # -1 weights skipped instead of subtracted
    t = np.atleast_2d(np.asarray(t, np.int8))
    xi = np.asarray(x, np.int64)
    return np.where(t > 0, xi[None, :], 0).sum(axis=1)


def _tern_sign_swapped(t, x):          # add where -1, subtract where +1
    return -oracle.ternary_product(t, x)



def _rsign_tie_negative(x, beta, axis=-1):      # x = beta mapped to -1
    xf = oracle._f32(x).astype(np.float64)
    b = oracle._f32(beta).astype(np.float64).reshape(-1)
    shape = [1] * xf.ndim
    shape[axis % xf.ndim] = b.size
    with np.errstate(invalid="ignore"):
        return np.where(xf - b.reshape(shape) <= 0.0, -1, 1).astype(np.int8)


def _rsign_reversed(x, beta, axis=-1):          # sign(beta - x)
    xf = oracle._f32(x).astype(np.float64)
    b = oracle._f32(beta).astype(np.float64).reshape(-1)
    shape = [1] * xf.ndim
    shape[axis % xf.ndim] = b.size
    with np.errstate(invalid="ignore"):
        return np.where(b.reshape(shape) - xf < 0.0, -1, 1).astype(np.int8)


def _rsign_last_axis(x, beta, axis=-1):         # threshold applied along the last axis
    xf = oracle._f32(x).astype(np.float64)
    b = oracle._f32(beta).astype(np.float64).reshape(-1)
    if b.size != xf.shape[-1]:
        b = np.resize(b, xf.shape[-1])
    with np.errstate(invalid="ignore"):
        return np.where(xf - b < 0.0, -1, 1).astype(np.int8)



def _planes_msb(x_u, k):                        # plane 0 holds the top bit
    x = np.asarray(x_u, np.int64)
    return np.stack([(x >> (k - 1 - b)) & 1 for b in range(k)]).astype(np.uint8)


def _bitserial_unweighted(a_u, w_u):            # plane pairs added without 2^(b+b')
    a = np.asarray(a_u, np.int64)
    w = np.asarray(w_u, np.int64)
    ka = max(1, int(a.max()).bit_length())
    kw = max(1, int(w.max()).bit_length())
    out = np.zeros((a.shape[0], w.shape[0]), np.int64)
    for b1 in range(ka):
        for b2 in range(kw):
            out += (((a >> b1) & 1)[:, None, :] * ((w >> b2) & 1)[None, :, :]).sum(axis=2)
    return out


def _bases_diagonal_only(h_pm1, b_pm1, alpha, beta):    # only the i == j cross terms
    h = np.asarray(h_pm1, np.int8)
    b = np.asarray(b_pm1, np.int8)
    al = np.asarray(alpha, np.float64)
    be = np.asarray(beta, np.float64).reshape(-1)
    y = np.zeros((h.shape[1], b.shape[1]))
    for j in range(min(h.shape[0], b.shape[0])):
        y += be[j] * al[j][None, :] * oracle.matmul_pm1(h[j], b[j]).astype(np.float64)
    return y



def _affine_no_beta(s, alpha_n, gamma, beta):     # beta dropped
    return np.asarray(gamma, np.float64) * (np.asarray(alpha_n, np.float64) * np.asarray(s, np.float64))


def _scaled_row_axis(s, alpha_n):                 # alpha applied along rows
    s = np.asarray(s, np.float64)
    a = np.asarray(alpha_n, np.float64)
    return a.reshape(-1, 1)[: s.shape[0]] * s if a.size >= s.shape[0] else s * 0


def _conv_affine_center_alpha(x_real, w_real, gamma, beta, stride=1, pad=1):   # alpha from the centre tap only
    xb = oracle.sign_pm1(x_real)
    fb = oracle.sign_pm1(w_real)
    wf = oracle._f32(w_real).astype(np.float64)
    k = wf.shape[2]
    a = np.abs(wf[:, :, k // 2, k // 2]).mean(axis=1)
    s = oracle.conv2d_pm1(xb, fb, stride, pad)
    y = oracle.affine(np.moveaxis(s, 1, -1), a, gamma, beta)
    return s, np.moveaxis(y, -1, 1)


def _binary_linear_alpha_from_x(x_real, w_real):  # alpha taken from the activations
    s, _ = oracle.binary_linear(x_real, w_real)
    return s, np.abs(np.atleast_2d(oracle._f32(x_real)).astype(np.float64)).mean()


def _bw_gemv_no_alpha(w_real, x_real):            # alpha left out of y
    a = oracle.alpha(w_real)
    return a, oracle.binary_weight_product(oracle.sign_pm1(w_real), oracle._f32(x_real))


MUTANTS = {
    "affine_without_beta": dict(affine=_affine_no_beta),
    "scaled_on_row_axis": dict(scaled=_scaled_row_axis),
    "conv_alpha_centre_tap": dict(conv_affine=_conv_affine_center_alpha),
    "linear_alpha_from_activations": dict(binary_linear=_binary_linear_alpha_from_x),
    "bw_gemv_without_alpha": dict(binary_weight_gemv=_bw_gemv_no_alpha),
    "planes_msb_first": dict(bit_planes=_planes_msb),
    "bitserial_unweighted_planes": dict(bitserial_product=_bitserial_unweighted),
    "bases_diagonal_only": dict(binary_bases_product=_bases_diagonal_only),
    "rsign_tie_negative": dict(rsign_pm1=_rsign_tie_negative),
    "rsign_reversed": dict(rsign_pm1=_rsign_reversed),
    "rsign_wrong_axis": dict(rsign_pm1=_rsign_last_axis),
    "ternary_gamma_without_abs": dict(ternary_quantize=_tern_gamma_noabs),
    "ternary_round_half_away": dict(ternary_quantize=_tern_round_half_away),
    "ternary_no_clip": dict(ternary_quantize=_tern_no_clip),
    "ternary_per_row_gamma": dict(ternary_quantize=_tern_per_row_gamma),
    "ternary_pack_codes_t": dict(pack_ternary=_tern_pack_codes_t),
    "ternary_pack_msb_first": dict(pack_ternary=_tern_pack_msb),
    "ternary_minus_as_skip": dict(ternary_product=_tern_minus_as_skip),
    "ternary_sign_swapped": dict(ternary_product=_tern_sign_swapped),
    "bw_sign_swapped": dict(binary_weight_product=_bw_sign_swapped),
    "bw_dropped_term": dict(binary_weight_product=_bw_drop_last),
    "bw_abs_activation": dict(binary_weight_product=_bw_abs_x),
    "sign_zero_negative": dict(sign_pm1=_sign_gt),
    "sign_bit_test": dict(sign_pm1=_sign_bit),
    "pack_msb_first": dict(pack_pm1=_pack_msb),
    "pack_inverted_encoding": dict(pack_pm1=_pack_inverted),
    "ld_not_rounded": dict(ld_words=_ld_no_round),
    "alpha_padded_divisor": dict(alpha=_alpha_padded),
    "alpha_without_abs": dict(alpha=_alpha_noabs),
    "matmul_transposed_operand": dict(matmul_pm1=_matmul_transposed),
    "matmul_dropped_term": dict(matmul_pm1=_matmul_drop_first),
    "conv_pad_minus_one": dict(conv2d_pm1=_conv_pad_minus),
    "conv_flipped_kernel": dict(conv2d_pm1=_conv_flipped),
    "bn_missing_gamma": dict(bn_value=_bn_value_no_gamma),
    "bn_mean_sign": dict(bn_value=_bn_value_mean_sign),
}


def _bn_sign_from_value(o):
    def f(s, a, g, b, mu, var, eps):
        y = o.bn_value(s, a, g, b, mu, var, eps)
        return np.where(y >= 0.0, 1, -1).astype(np.int8)
    return f


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, golden_dir):
    o = _mutant(**MUTANTS[name])
    if "bn_value" in MUTANTS[name]:
        o.bn_sign = _bn_sign_from_value(o)
    failed = []
    for check_name, check in ALL_CHECKS:
        try:
            check(o, golden_dir)
        except AssertionError:
            failed.append(check_name)
        except (ValueError, IndexError):
            failed.append(check_name)
    assert failed, f"planted mistake {name!r} passed every pin"


def test_tie_rule_mistake_is_caught():
    """A BN decision that sends an exact 0 to -1 contradicts the sign tie rule
    (sign(0) = +1): an exact zero is reachable when mean = alpha*s and beta = 0."""
    s = np.array([[4]], np.int32)
    a = np.array([0.5], np.float32)
    one = np.ones(1, np.float32)
    zero = np.zeros(1, np.float32)
    mu = np.array([2.0], np.float32)
    assert oracle.bn_sign(s, a, one, zero, mu, one, 0.0)[0, 0] == 1
    assert _bn_sign_strict(s, a, one, zero, mu, one, 0.0)[0, 0] == -1
