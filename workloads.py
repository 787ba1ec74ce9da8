"""Seeded synthetic inputs for the binary (±1) matrix-product workloads.

This module only draws random numbers and builds tensors of the right shape,
dtype and distribution.  It holds none of the method's arithmetic (no sign,
no packing, no popcount, no scaling), so both the CUDA path and the CPU oracle
can take their inputs from here without sharing any of the computation.

All draws use a CPU ``torch.Generator`` with a fixed seed, so the oracle and
the GPU see identical bytes: tensors are generated on the host and copied to
the device by the caller.  ``N(0, s)`` means mean 0, standard deviation ``s``.
bf16 tensors are the fp32 draws cast to bf16 (round to nearest even).

Workloads (shapes from the binary-network pages: an XNOR-Net style layer, a
batch-1 LLM decode projection, a ResNet-18-class hidden 3x3 convolution and a
fully binary MLP):

* ``tiny``   X fp32 [64, 1000], W fp32 [256, 1000], both N(0, 1), seed 1.
* ``gemv``   W fp32 [11008, 4096] N(0, 0.02) seed 2; x bf16 [4096] N(0, 1) seed 3.
* ``square`` A, W fp32 [8192, 8192] N(0, 1), seeds 4 and 5.
* ``conv``   X bf16 [64, 64, 56, 56] N(0, 1) seed 6; W fp32 [64, 64, 3, 3]
             N(0, 0.1) seed 7; gamma U(0.5, 1.5), beta N(0, 0.1) [64] seed 8.
* ``downsample`` X bf16 [64, 64, 56, 56] N(0, 1) seed 6 (the conv input); W fp32
             [128, 64, 1, 1] N(0, 0.1) seed 18; gamma U(0.5, 1.5), beta N(0, 0.1)
             [128] seed 19 (1x1 stride-2 projection to 128 channels).
* ``ternary`` W fp32 [11008, 4096] N(0, 0.02) seed 2 (the decode weights, to be
             ternarised); x int8 [4096] uniform over [-128, 127] seed 17.
* ``mlp``    X0 fp32 [4096, 4096] N(0, 1) seed 9; W_l fp32 [4096, 4096] N(0, 1)
             seeds 10..13; BatchNorm after layers 1..3 with gamma U(0.5, 1.5),
             beta N(0, 0.1), running mean N(0, 1), running var U(0.5, 2),
             seeds 14..16; eps 1e-5.
* ``bitserial`` unsigned codes a uint8 [4096, 4096] (2 bits) seed 20 and w uint8
             [4096, 4096] (2 bits) seed 21, uniform over [0, 2^bits): DoReFa-style
             low-bit activations and weights at the MLP's layer shape.
* ``bases``  J = 3 activation bases and I = 3 weight bases at the same shape: real
             draws N(0, 1) [J, 4096, 4096] seed 22 and [I, 4096, 4096] seed 23 (their
             signs are the bases), alpha_i[n] |N(0, 0.3)| + 0.01 seed 24, beta_j
             |N(0, 0.5)| + 0.05 seed 25 (ABC-Net-style weighted binary bases).
* ``chain``  a batch-1 decode step through a fully binary MLP: x bf16 [4096] N(0, 1)
             seed 30; 8 layers alternating up [11008, 4096] and down [4096, 11008]
             (the decode projection's shape and weight law, N(0, 0.02), seeds 31..);
             BatchNorm after every hidden layer drawn as for ``mlp`` (seeds 50..).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

BN_EPS = 1e-5


def _gen(seed: int) -> torch.Generator:
    return torch.Generator().manual_seed(int(seed))


def normal(shape, std: float, seed: int, dtype=torch.float32) -> torch.Tensor:
    """N(0, std) draws in fp32 from ``seed``, optionally cast to ``dtype``."""
    t = torch.randn(*shape, generator=_gen(seed), dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype) if dtype != torch.float32 else t


def uniform(shape, lo: float, hi: float, seed: int) -> torch.Tensor:
    t = torch.rand(*shape, generator=_gen(seed), dtype=torch.float32)
    return t.mul_(hi - lo).add_(lo)


@dataclass
class BatchNormParams:
    gamma: torch.Tensor
    beta: torch.Tensor
    mean: torch.Tensor
    var: torch.Tensor
    eps: float = BN_EPS


def batchnorm_params(n: int, seed: int) -> BatchNormParams:
    g = _gen(seed)
    gamma = torch.rand(n, generator=g).mul_(1.0).add_(0.5)           # U(0.5, 1.5)
    beta = torch.randn(n, generator=g).mul_(0.1)                       # N(0, 0.1)
    mean = torch.randn(n, generator=g)                                 # N(0, 1)
    var = torch.rand(n, generator=g).mul_(1.5).add_(0.5)               # U(0.5, 2)
    return BatchNormParams(gamma, beta, mean, var, BN_EPS)


# --------------------------------------------------------------------------
# the five workloads
# --------------------------------------------------------------------------

@dataclass
class Tiny:
    M: int = 64
    N: int = 256
    K: int = 1000
    X: torch.Tensor = None
    W: torch.Tensor = None


def tiny(M=64, N=256, K=1000, seed=1) -> Tiny:
    g = _gen(seed)
    X = torch.randn(M, K, generator=g)
    W = torch.randn(N, K, generator=g)
    return Tiny(M, N, K, X, W)


@dataclass
class Gemv:
    N: int
    K: int
    W: torch.Tensor      # fp32 [N, K]
    x: torch.Tensor      # bf16 [K]


def gemv(N=11008, K=4096, w_seed=2, x_seed=3, x_dtype=torch.bfloat16) -> Gemv:
    W = normal((N, K), 0.02, w_seed)
    x = normal((K,), 1.0, x_seed, dtype=x_dtype)
    return Gemv(N, K, W, x)


def downsample(n=64, c=64, h=56, w=56, cout=128, x_seed=6, w_seed=18, bn_seed=19, stride=2,
               x_dtype=torch.bfloat16) -> Conv:
    X = normal((n, c, h, w), 1.0, x_seed, dtype=x_dtype)
    W = normal((cout, c, 1, 1), 0.1, w_seed)
    g = _gen(bn_seed)
    gamma = torch.rand(cout, generator=g).add_(0.5)
    beta = torch.randn(cout, generator=g).mul_(0.1)
    return Conv(X, W, gamma, beta, stride, 0)


@dataclass
class Ternary:
    N: int
    K: int
    W: torch.Tensor      # fp32 [N, K]
    x: torch.Tensor      # int8 [K]


def int8_uniform(shape, seed: int) -> torch.Tensor:
    """int8 draws, uniform over [-128, 127]."""
    return torch.randint(-128, 128, tuple(shape), generator=_gen(seed), dtype=torch.int8)


def ternary(N=11008, K=4096, w_seed=2, x_seed=17) -> Ternary:
    return Ternary(N, K, normal((N, K), 0.02, w_seed), int8_uniform((K,), x_seed))


@dataclass
class Square:
    M: int
    N: int
    K: int
    A: torch.Tensor
    W: torch.Tensor


def square(M=8192, N=8192, K=8192, a_seed=4, w_seed=5) -> Square:
    A = normal((M, K), 1.0, a_seed)
    W = normal((N, K), 1.0, w_seed)
    return Square(M, N, K, A, W)


@dataclass
class Conv:
    X: torch.Tensor      # bf16 [n, c, h, w]
    W: torch.Tensor      # fp32 [cout, cin, 3, 3]
    gamma: torch.Tensor  # fp32 [cout]
    beta: torch.Tensor   # fp32 [cout]
    stride: int = 1
    pad: int = 1


def conv(n=64, c=64, h=56, w=56, cout=64, x_seed=6, w_seed=7, bn_seed=8,
         stride=1, pad=1, x_dtype=torch.bfloat16) -> Conv:
    X = normal((n, c, h, w), 1.0, x_seed, dtype=x_dtype)
    W = normal((cout, c, 3, 3), 0.1, w_seed)
    g = _gen(bn_seed)
    gamma = torch.rand(cout, generator=g).add_(0.5)
    beta = torch.randn(cout, generator=g).mul_(0.1)
    return Conv(X, W, gamma, beta, stride, pad)


@dataclass
class Mlp:
    X0: torch.Tensor                    # fp32 [batch, width]
    Ws: list = field(default_factory=list)   # 4 x fp32 [width, width]
    bns: list = field(default_factory=list)  # 3 x BatchNormParams


def mlp(batch=4096, width=4096, layers=4, x_seed=9, w_seed0=10, bn_seed0=14) -> Mlp:
    X0 = normal((batch, width), 1.0, x_seed)
    Ws = [normal((width, width), 1.0, w_seed0 + l) for l in range(layers)]
    bns = [batchnorm_params(width, bn_seed0 + l) for l in range(layers - 1)]
    return Mlp(X0, Ws, bns)


def codes(shape, bits: int, seed: int) -> torch.Tensor:
    """Unsigned integer codes, uniform over [0, 2^bits), as uint8."""
    return torch.randint(0, 1 << bits, tuple(shape), generator=_gen(seed), dtype=torch.int64).to(torch.uint8)


@dataclass
class Bitserial:
    a: torch.Tensor      # uint8 [M, K], a_bits-bit codes
    w: torch.Tensor      # uint8 [N, K], w_bits-bit codes
    a_bits: int
    w_bits: int


def bitserial(M=4096, N=4096, K=4096, a_bits=2, w_bits=2, a_seed=20, w_seed=21) -> Bitserial:
    return Bitserial(codes((M, K), a_bits, a_seed), codes((N, K), w_bits, w_seed), a_bits, w_bits)


@dataclass
class Bases:
    h_real: torch.Tensor  # fp32 [J, M, K]: the activation bases are their signs
    b_real: torch.Tensor  # fp32 [I, N, K]: the weight bases are their signs
    alpha: torch.Tensor   # fp32 [I, N]
    beta: torch.Tensor    # fp32 [J]


def bases(M=4096, N=4096, K=4096, J=3, I=3, seed=22) -> Bases:
    h_real = normal((J, M, K), 1.0, seed)
    b_real = normal((I, N, K), 1.0, seed + 1)
    alpha = normal((I, N), 0.3, seed + 2).abs_().add_(0.01)
    beta = normal((J,), 0.5, seed + 3).abs_().add_(0.05)
    return Bases(h_real, b_real, alpha, beta)


# --------------------------------------------------------------------------
# edge-case values for the sign rule
# --------------------------------------------------------------------------

def sign_edge_values(dtype=torch.float32) -> torch.Tensor:
    """Values at which a sign rule is easy to get wrong: signed zeros,
    denormals, infinities, NaN, and the smallest normals of both signs."""
    vals = [0.0, -0.0, 1e-45, -1e-45, 1e-40, -1e-40, 1.17549435e-38,
            -1.17549435e-38, float("inf"), float("-inf"), float("nan"),
            1.0, -1.0, 3.0e38, -3.0e38]
    t = torch.tensor(vals, dtype=torch.float32)
    if dtype == torch.bfloat16:
        t = t.to(torch.bfloat16)
    return t


def random_with_edges(rows: int, K: int, seed: int, dtype=torch.float32,
                      edge_fraction: float = 0.05, finite: bool = True) -> torch.Tensor:
    """N(0, 1) matrix with a seeded fraction of entries replaced by edge values.

    With ``finite`` (the default) infinities and NaN are left out, so a
    per-row mean magnitude stays finite; the non-finite values are drawn in
    only when ``finite=False``."""
    g = _gen(seed)
    t = torch.randn(rows, K, generator=g)
    edges = sign_edge_values(torch.float32)
    if finite:
        edges = edges[torch.isfinite(edges)]
    mask = torch.rand(rows, K, generator=g) < edge_fraction
    idx = torch.randint(0, edges.numel(), (rows, K), generator=g)
    t = torch.where(mask, edges[idx], t)
    if dtype == torch.bfloat16:
        t = t.to(torch.bfloat16)
    return t


@dataclass
class Chain:
    x0: torch.Tensor                    # [K0] real input (bf16 or fp32)
    Ws: list = field(default_factory=list)   # fp32 [N_l, K_l], K_l = N_{l-1}
    bns: list = field(default_factory=list)  # BatchNormParams after each hidden layer


def chain(widths=(11008, 4096) * 4, K0=4096, x_seed=30, w_seed0=31, bn_seed0=50, w_std=0.02,
          x_dtype=torch.bfloat16) -> Chain:
    x0 = normal((K0,), 1.0, x_seed, dtype=x_dtype)
    Ws, k = [], K0
    for l, n in enumerate(widths):
        Ws.append(normal((n, k), w_std, w_seed0 + l))
        k = n
    bns = [batchnorm_params(n, bn_seed0 + l) for l, n in enumerate(widths[:-1])]
    return Chain(x0, Ws, bns)
