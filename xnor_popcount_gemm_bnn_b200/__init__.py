"""Python binding of libbnn.so: the binary (+1/-1) matrix product on packed bits.

Thin ``ctypes`` marshalling over the C ABI in ``include/bnn.h``; the functions
keep the C names.  Tensors are torch tensors (device memory on the current
CUDA device, host memory for ``bnn_fold_bn_threshold``); every device call is
launched on ``torch.cuda.current_stream()`` unless a stream is given.  All
computation happens in the library's CUDA kernels; nothing here computes.
There is no CPU fallback: importing the package fails if ``libbnn.so`` has
not been built (``python xnor_popcount_gemm_bnn_b200/build.py``).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbnn.so")

BNN_OK = 0
BNN_ERR_INVALID_ARG = 1
BNN_ERR_ALIGNMENT = 2
BNN_ERR_UNSUPPORTED = 3
BNN_ERR_CUDA = 4
BNN_ERR_DEVICE_TIMEOUT = 5

BNN_F32 = 0
BNN_BF16 = 1

BNN_OUT_INT32 = 1
BNN_OUT_SCALED_F32 = 2
BNN_OUT_AFFINE_F32 = 4
BNN_OUT_THRESHOLD_PACK = 8

BNN_GEMV_WEIGHTS_STATIC = 1
BNN_GEMV_INPUTS_STATIC = 2
BNN_GEMV_OUTPUT_FREE = 4

BNN_GEMM_ENGINE_AUTO = 0
BNN_GEMM_ENGINE_POPCOUNT = 1
BNN_GEMM_ENGINE_TENSOR = 2
BNN_GEMM_ENGINE_TENSOR_I8 = 3

# Every symbol declared in include/bnn.h.
EXPORTS = (
    "bnn_packed_ld_words", "bnn_conv3x3_ld_words", "bnn_status_string", "bnn_device_error",
    "bnn_pack_sign", "bnn_pack_sign_nchw", "bnn_pack_conv3x3_weights", "bnn_xnor_gemm",
    "bnn_xnor_gemv", "bnn_xnor_gemv_ex", "bnn_xnor_gemv_host", "bnn_binary_linear_fused", "bnn_binary_conv3x3_fused",
    "bnn_fold_bn_threshold", "bnn_set_gemm_engine", "bnn_get_gemm_engine", "bnn_selftest_wait_timeout",
    "bnn_binary_weight_gemv", "bnn_ternary_ld_words", "bnn_ternary_workspace_bytes", "bnn_ternary_pack",
    "bnn_ternary_gemv_i8", "bnn_ternary_pack_noalloc", "bnn_pack_sign_rsign", "bnn_pack_sign_nchw_rsign",
    "bnn_binary_conv1x1_fused", "bnn_probe_int_pipes", "bnn_pack_bit_planes", "bnn_bitserial_gemm",
    "bnn_binary_bases_gemm", "bnn_binary_weight_gemv_i8", "bnn_gemv_chain_workspace_words",
    "bnn_xnor_gemv_chain",
)


class BnnError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} failed: status {status} ({msg})")
        self.status = status


class bnn_epilogue(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("alpha", ctypes.c_void_p), ("gamma", ctypes.c_void_p),
                ("beta", ctypes.c_void_p), ("popc_thresh", ctypes.c_void_p),
                ("thresh_mode", ctypes.c_void_p)]


class bnn_chain_layer(ctypes.Structure):
    _fields_ = [("W", ctypes.c_void_p), ("ldw", ctypes.c_int64), ("N", ctypes.c_int64),
                ("popc_thresh", ctypes.c_void_p), ("thresh_mode", ctypes.c_void_p), ("alpha", ctypes.c_void_p)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python xnor_popcount_gemm_bnn_b200/build.py` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    i64, p, i32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int32
    sig = {
        "bnn_packed_ld_words": (i64, [i64]),
        "bnn_conv3x3_ld_words": (i64, [i64]),
        "bnn_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "bnn_device_error": (i32, [p]),
        "bnn_pack_sign": (i32, [p, i32, i64, i64, i64, p, i64, p, p]),
        "bnn_pack_sign_nchw": (i32, [p, i32, i64, i64, i64, i64, p, p]),
        "bnn_pack_conv3x3_weights": (i32, [p, i32, i64, i64, p, i64, p, p]),
        "bnn_xnor_gemm": (i32, [p, i64, p, i64, i64, i64, i64, p, p, i64, p, i64, p]),
        "bnn_xnor_gemv": (i32, [p, i64, p, i32, i64, i64, p, p, p, p]),
        "bnn_xnor_gemv_ex": (i32, [p, i64, p, i32, i64, i64, p, p, p, ctypes.c_uint32, p]),
        "bnn_xnor_gemv_host": (i32, [p, i64, p, i32, i64, i64, p, p, p, p, ctypes.c_uint32, p]),
        "bnn_binary_weight_gemv": (i32, [p, i64, p, i32, i64, i64, p, p, ctypes.c_uint32, p]),
        "bnn_binary_linear_fused": (i32, [p, i64, p, i64, i64, i64, i64,
                                          ctypes.POINTER(bnn_epilogue), p, i64, p]),
        "bnn_binary_conv3x3_fused": (i32, [p, i64, i64, i64, i64, p, i64, i64, i64, i64,
                                           ctypes.POINTER(bnn_epilogue), p, p]),
        "bnn_fold_bn_threshold": (i32, [p, p, p, p, p, ctypes.c_double, i64, i64, p, p]),
        "bnn_set_gemm_engine": (i32, [ctypes.c_int]),
        "bnn_get_gemm_engine": (ctypes.c_int, []),
        "bnn_selftest_wait_timeout": (i32, [i64, p]),
        "bnn_ternary_ld_words": (i64, [i64]),
        "bnn_ternary_workspace_bytes": (i64, [i64]),
        "bnn_ternary_pack": (i32, [p, i32, i64, i64, i64, ctypes.c_double, p, i64, p, p, i64, p]),
        "bnn_ternary_gemv_i8": (i32, [p, i64, p, i64, i64, p, p, p, p, ctypes.c_uint32, p]),
        "bnn_ternary_pack_noalloc": (i32, [p, i32, i64, i64, i64, ctypes.c_double, p, i64, p, p]),
        "bnn_pack_sign_rsign": (i32, [p, i32, i64, i64, i64, p, p, i64, p]),
        "bnn_pack_sign_nchw_rsign": (i32, [p, i32, i64, i64, i64, i64, p, p, p]),
        "bnn_binary_conv1x1_fused": (i32, [p, i64, i64, i64, i64, p, i64, i64, i64,
                                           ctypes.POINTER(bnn_epilogue), p, p]),
        "bnn_probe_int_pipes": (i32, [i64, p, p, p]),
        "bnn_pack_bit_planes": (i32, [p, i64, i64, i64, i32, p, i64, p]),
        "bnn_bitserial_gemm": (i32, [p, i64, i32, p, i64, i32, i64, i64, i64, p, p, i64, p, i64, p]),
        "bnn_binary_bases_gemm": (i32, [p, i64, i32, p, i64, i32, i64, i64, i64, p, p, i64, p, i64, p]),
        "bnn_binary_weight_gemv_i8": (i32, [p, i64, p, i64, i64, p, i32, p, p, p, ctypes.c_uint32, p]),
        "bnn_gemv_chain_workspace_words": (i64, []),
        "bnn_xnor_gemv_chain": (i32, [ctypes.POINTER(bnn_chain_layer), i32, p, i32, i64, p, p, p, i64, p, p]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()
lib = _lib


def _check(fn: str, status: int) -> None:
    if status != BNN_OK:
        raise BnnError(fn, status, _lib.bnn_status_string(status).decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return BNN_F32
    if t.dtype == torch.bfloat16:
        return BNN_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; expected float32 or bfloat16")


def _ld(t: torch.Tensor) -> int:
    return t.stride(0) if t.dim() >= 2 else t.shape[-1]


# --------------------------------------------------------------------------
# sizes and status
# --------------------------------------------------------------------------

def bnn_packed_ld_words(K: int) -> int:
    return int(_lib.bnn_packed_ld_words(int(K)))


def bnn_conv3x3_ld_words(cin: int) -> int:
    return int(_lib.bnn_conv3x3_ld_words(int(cin)))


def bnn_ternary_ld_words(K: int) -> int:
    return int(_lib.bnn_ternary_ld_words(int(K)))


def bnn_ternary_workspace_bytes(rows: int) -> int:
    return int(_lib.bnn_ternary_workspace_bytes(int(rows)))


def bnn_status_string(status: int) -> str:
    return _lib.bnn_status_string(int(status)).decode()


def bnn_set_gemm_engine(engine: int) -> None:
    _check("bnn_set_gemm_engine", _lib.bnn_set_gemm_engine(int(engine)))


def bnn_get_gemm_engine() -> int:
    return int(_lib.bnn_get_gemm_engine())


class gemm_engine:
    """Context manager: run the enclosed calls with one GEMM engine."""

    def __init__(self, engine: int):
        self.engine = int(engine)

    def __enter__(self):
        self.prev = bnn_get_gemm_engine()
        bnn_set_gemm_engine(self.engine)
        return self

    def __exit__(self, *exc):
        bnn_set_gemm_engine(self.prev)


def bnn_probe_int_pipes(iters: int = 4096) -> dict:
    """Integer-pipe rates of the current device, per SM clock:
    {"popc": POPC, "lop3": LOP3, "csa_words": XOR words through the carry-save step}."""
    a, b, c = ctypes.c_double(), ctypes.c_double(), ctypes.c_double()
    _check("bnn_probe_int_pipes", _lib.bnn_probe_int_pipes(int(iters), ctypes.byref(a), ctypes.byref(b),
                                                           ctypes.byref(c)))
    return {"popc": a.value, "lop3": b.value, "csa_words": c.value}


def bnn_selftest_wait_timeout(timeout_ns: int) -> bool:
    """Run the bounded-wait diagnostic; True when the wait ran out (expected)."""
    out = ctypes.c_int32(-1)
    _check("bnn_selftest_wait_timeout", _lib.bnn_selftest_wait_timeout(int(timeout_ns), ctypes.byref(out)))
    return bool(out.value)


def bnn_device_error() -> int:
    code = ctypes.c_int32(0)
    _check("bnn_device_error", _lib.bnn_device_error(ctypes.byref(code)))
    return int(code.value)


# --------------------------------------------------------------------------
# packing
# --------------------------------------------------------------------------

def bnn_pack_sign(x: torch.Tensor, packed: torch.Tensor, alpha_out: Optional[torch.Tensor] = None,
                  K: Optional[int] = None, stream=None) -> None:
    """x [rows, K] (fp32/bf16, unit inner stride) -> packed uint32 [rows, ld] (int32 storage)."""
    if x.dim() == 1:
        x = x.view(1, -1)
    assert x.stride(-1) == 1 and packed.stride(-1) == 1
    rows, Kx = x.shape
    K = Kx if K is None else int(K)
    _check("bnn_pack_sign", _lib.bnn_pack_sign(
        _ptr(x), _dtype(x), rows, K, _ld(x), _ptr(packed), _ld(packed) if packed.dim() >= 2 else packed.shape[-1],
        _ptr(alpha_out), _stream(stream)))


def bnn_pack_sign_nchw(x: torch.Tensor, packed_nhwc: torch.Tensor, stream=None) -> None:
    assert x.is_contiguous() and packed_nhwc.is_contiguous()
    n, c, h, w = x.shape
    _check("bnn_pack_sign_nchw", _lib.bnn_pack_sign_nchw(
        _ptr(x), _dtype(x), n, c, h, w, _ptr(packed_nhwc), _stream(stream)))



def bnn_pack_sign_rsign(x: torch.Tensor, beta: torch.Tensor, packed: torch.Tensor, K: Optional[int] = None,
                        stream=None) -> None:
    """x [rows, K] -> packed bits of sign(x - beta_k), beta fp32 [K] per column."""
    if x.dim() == 1:
        x = x[None, :]
    assert x.stride(-1) == 1 and packed.stride(-1) == 1 and beta.dtype == torch.float32
    rows, Kx = x.shape
    K = Kx if K is None else int(K)
    _check("bnn_pack_sign_rsign", _lib.bnn_pack_sign_rsign(
        _ptr(x), _dtype(x), rows, K, _ld(x), _ptr(beta), _ptr(packed),
        _ld(packed) if packed.dim() >= 2 else packed.shape[-1], _stream(stream)))


def bnn_pack_sign_nchw_rsign(x: torch.Tensor, beta: torch.Tensor, packed_nhwc: torch.Tensor, stream=None) -> None:
    """NCHW x -> per-pixel channel words of sign(x - beta_c), beta fp32 [c]."""
    assert x.is_contiguous() and packed_nhwc.is_contiguous() and beta.dtype == torch.float32
    n, c, h, w = x.shape
    _check("bnn_pack_sign_nchw_rsign", _lib.bnn_pack_sign_nchw_rsign(
        _ptr(x), _dtype(x), n, c, h, w, _ptr(beta), _ptr(packed_nhwc), _stream(stream)))

def bnn_pack_conv3x3_weights(w_oihw: torch.Tensor, packed: torch.Tensor,
                             alpha_out: Optional[torch.Tensor] = None, stream=None) -> None:
    assert w_oihw.is_contiguous() and tuple(w_oihw.shape[2:]) == (3, 3)
    cout, cin = w_oihw.shape[:2]
    _check("bnn_pack_conv3x3_weights", _lib.bnn_pack_conv3x3_weights(
        _ptr(w_oihw), _dtype(w_oihw), cout, cin, _ptr(packed), _ld(packed), _ptr(alpha_out),
        _stream(stream)))


# --------------------------------------------------------------------------
# products
# --------------------------------------------------------------------------

def bnn_xnor_gemm(A: torch.Tensor, W: torch.Tensor, K: int, alpha: Optional[torch.Tensor] = None,
                  C_i32: Optional[torch.Tensor] = None, C_f32: Optional[torch.Tensor] = None,
                  M: Optional[int] = None, N: Optional[int] = None, stream=None) -> None:
    M = A.shape[0] if M is None else M
    N = W.shape[0] if N is None else N
    _check("bnn_xnor_gemm", _lib.bnn_xnor_gemm(
        _ptr(A), _ld(A), _ptr(W), _ld(W), M, N, int(K), _ptr(alpha),
        _ptr(C_i32), _ld(C_i32) if C_i32 is not None else 0,
        _ptr(C_f32), _ld(C_f32) if C_f32 is not None else 0, _stream(stream)))


def bnn_xnor_gemv(W: torch.Tensor, x: torch.Tensor, K: Optional[int] = None,
                  alpha: Optional[torch.Tensor] = None, y_i32: Optional[torch.Tensor] = None,
                  y_f32: Optional[torch.Tensor] = None, N: Optional[int] = None, stream=None) -> None:
    N = W.shape[0] if N is None else N
    K = x.shape[-1] if K is None else int(K)
    _check("bnn_xnor_gemv", _lib.bnn_xnor_gemv(
        _ptr(W), _ld(W), _ptr(x), _dtype(x), N, K, _ptr(alpha), _ptr(y_i32), _ptr(y_f32),
        _stream(stream)))


def bnn_xnor_gemv_ex(W: torch.Tensor, x: torch.Tensor, K: Optional[int] = None,
                     alpha: Optional[torch.Tensor] = None, y_i32: Optional[torch.Tensor] = None,
                     y_f32: Optional[torch.Tensor] = None, flags: int = 0, N: Optional[int] = None,
                     stream=None) -> None:
    N = W.shape[0] if N is None else N
    K = x.shape[-1] if K is None else int(K)
    _check("bnn_xnor_gemv_ex", _lib.bnn_xnor_gemv_ex(
        _ptr(W), _ld(W), _ptr(x), _dtype(x), N, K, _ptr(alpha), _ptr(y_i32), _ptr(y_f32),
        int(flags), _stream(stream)))


def bnn_xnor_gemv_host(W: torch.Tensor, x_host: torch.Tensor, K: Optional[int], alpha: torch.Tensor,
                       x_dev: torch.Tensor, y_dev: torch.Tensor, y_host: torch.Tensor, flags: int = 0,
                       N: Optional[int] = None, stream=None) -> None:
    """The GEMV with x and y in host memory: copies x in, runs the GEMV, copies y (fp32) out, all on
    `stream`; x_dev and y_dev are the caller's device scratch."""
    assert not x_host.is_cuda and not y_host.is_cuda and x_dev.is_cuda and y_dev.is_cuda
    N = W.shape[0] if N is None else N
    K = x_host.shape[-1] if K is None else int(K)
    assert x_dev.dtype == x_host.dtype and x_dev.numel() >= K and y_dev.numel() >= N and y_host.numel() >= N
    _check("bnn_xnor_gemv_host", _lib.bnn_xnor_gemv_host(
        _ptr(W), _ld(W), _ptr(x_host), _dtype(x_host), N, K, _ptr(alpha), _ptr(x_dev), _ptr(y_dev), _ptr(y_host),
        int(flags), _stream(stream)))


def bnn_binary_weight_gemv(W: torch.Tensor, x: torch.Tensor, K: Optional[int], alpha: torch.Tensor,
                           y: torch.Tensor, flags: int = 0, N: Optional[int] = None, stream=None) -> None:
    """y = alpha * (sign(W) x) with a real x (fp32 or bf16), W packed."""
    N = W.shape[0] if N is None else N
    K = x.shape[-1] if K is None else int(K)
    _check("bnn_binary_weight_gemv", _lib.bnn_binary_weight_gemv(
        _ptr(W), _ld(W), _ptr(x), _dtype(x), N, K, _ptr(alpha), _ptr(y), int(flags), _stream(stream)))



def bnn_binary_weight_gemv_i8(W: torch.Tensor, x: torch.Tensor, K: Optional[int] = None,
                              alpha: Optional[torch.Tensor] = None, x_scale: Optional[torch.Tensor] = None,
                              y_i32: Optional[torch.Tensor] = None, y_f32: Optional[torch.Tensor] = None,
                              flags: int = 0, stream=None) -> None:
    """Packed binary W [N, ld] x int8 x [K]; alpha [N] (per row) or [1] (one scale for the matrix)."""
    assert x.dtype == torch.int8
    K = x.shape[-1] if K is None else int(K)
    per_row = 1 if (alpha is None or alpha.numel() == W.shape[0]) else 0
    if alpha is not None and not per_row:
        assert alpha.numel() == 1
    _check("bnn_binary_weight_gemv_i8", _lib.bnn_binary_weight_gemv_i8(
        _ptr(W), _ld(W), _ptr(x), W.shape[0], K, _ptr(alpha), per_row, _ptr(x_scale), _ptr(y_i32), _ptr(y_f32),
        int(flags), _stream(stream)))


def bnn_ternary_pack(w: torch.Tensor, codes: torch.Tensor, gamma_out: Optional[torch.Tensor] = None,
                     delta: Optional[float] = None, workspace: Optional[torch.Tensor] = None,
                     K: Optional[int] = None, stream=None) -> None:
    """w [rows, K] (fp32/bf16) -> ternary codes [rows, ldq] (int32 storage).
    delta None: eq. (9) (absmean gamma); else eq. (7) with that threshold.
    The workspace (needed for gamma) is allocated here with torch when not
    given."""
    if w.dim() == 1:
        w = w[None, :]
    assert w.stride(-1) == 1 and codes.stride(-1) == 1
    rows, Kw = w.shape
    K = Kw if K is None else int(K)
    d = -1.0 if delta is None else float(delta)
    if workspace is None and (delta is None or gamma_out is not None):
        workspace = torch.empty(max(1, bnn_ternary_workspace_bytes(rows) // 8), dtype=torch.float64,
                                device=w.device)
    wsb = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("bnn_ternary_pack", _lib.bnn_ternary_pack(
        _ptr(w), _dtype(w), rows, K, _ld(w), d, _ptr(codes), _ld(codes) if codes.dim() >= 2 else codes.shape[-1],
        _ptr(gamma_out), _ptr(workspace), wsb, _stream(stream)))



BNN_TERNARY_PACK_NOALLOC_MAX_ROWS = 262144


def bnn_ternary_pack_noalloc(w: torch.Tensor, codes: torch.Tensor, gamma_out: Optional[torch.Tensor] = None,
                             delta: Optional[float] = None, K: Optional[int] = None, stream=None) -> None:
    """bnn_ternary_pack for callers that cannot allocate device memory: the
    scratch space lives in the library (rows <= 262144); this wrapper
    allocates nothing either."""
    if w.dim() == 1:
        w = w[None, :]
    assert w.stride(-1) == 1 and codes.stride(-1) == 1
    rows, Kw = w.shape
    K = Kw if K is None else int(K)
    d = -1.0 if delta is None else float(delta)
    _check("bnn_ternary_pack_noalloc", _lib.bnn_ternary_pack_noalloc(
        _ptr(w), _dtype(w), rows, K, _ld(w), d, _ptr(codes), _ld(codes) if codes.dim() >= 2 else codes.shape[-1],
        _ptr(gamma_out), _stream(stream)))

def bnn_ternary_gemv_i8(codes: torch.Tensor, x: torch.Tensor, K: Optional[int] = None,
                        y_i32: Optional[torch.Tensor] = None, y_f32: Optional[torch.Tensor] = None,
                        w_scale: Optional[torch.Tensor] = None, x_scale: Optional[torch.Tensor] = None,
                        flags: int = 0, N: Optional[int] = None, stream=None) -> None:
    """acc = t x (int8 x, exact int32) and/or y = w_scale * x_scale * acc."""
    assert x.dtype == torch.int8
    N = codes.shape[0] if N is None else N
    K = x.shape[-1] if K is None else int(K)
    _check("bnn_ternary_gemv_i8", _lib.bnn_ternary_gemv_i8(
        _ptr(codes), _ld(codes), _ptr(x), N, K, _ptr(w_scale), _ptr(x_scale), _ptr(y_i32), _ptr(y_f32),
        int(flags), _stream(stream)))

def bnn_gemv_chain_workspace_words() -> int:
    return int(_lib.bnn_gemv_chain_workspace_words())


def gemv_chain_workspace(device) -> torch.Tensor:
    """A zeroed workspace for bnn_xnor_gemv_chain (each call leaves it zero)."""
    return torch.zeros(bnn_gemv_chain_workspace_words(), dtype=torch.int32, device=device)


def chain_layers(layers) -> ctypes.Array:
    """bnn_chain_layer array from dicts with keys W (packed [N, ld]), and
    popc_thresh / thresh_mode (hidden layers) or alpha (last layer); N defaults
    to W.shape[0].  The array keeps references to the tensors."""
    arr = (bnn_chain_layer * len(layers))()
    keep = []
    for i, ly in enumerate(layers):
        W = ly["W"]
        arr[i] = bnn_chain_layer(W.data_ptr(), _ld(W), int(ly.get("N", W.shape[0])), _ptr(ly.get("popc_thresh")),
                                 _ptr(ly.get("thresh_mode")), _ptr(ly.get("alpha")))
        keep.append(ly)
    arr._keep = keep
    return arr


def bnn_xnor_gemv_chain(layers, x: torch.Tensor, workspace: torch.Tensor, K: Optional[int] = None,
                        y_i32: Optional[torch.Tensor] = None, y_f32: Optional[torch.Tensor] = None,
                        acts: Optional[torch.Tensor] = None, stream=None) -> None:
    """A batch-1 fully binary layer chain in one launch; ``layers`` is a list
    of dicts (see chain_layers) or an array it returned."""
    arr = layers if isinstance(layers, ctypes.Array) else chain_layers(layers)
    K = x.shape[-1] if K is None else int(K)
    _check("bnn_xnor_gemv_chain", _lib.bnn_xnor_gemv_chain(
        arr, len(arr), _ptr(x), _dtype(x), K, _ptr(y_i32), _ptr(y_f32), _ptr(acts),
        _ld(acts) if acts is not None else 0, _ptr(workspace), _stream(stream)))


def make_epilogue(mode: int, alpha=None, gamma=None, beta=None, popc_thresh=None,
                  thresh_mode=None) -> bnn_epilogue:
    """The epilogue struct with raw device pointers.  It keeps references to
    the tensors it points into, so that temporaries (``t.to(device)``) stay
    alive for as long as the struct does."""
    ep = bnn_epilogue(int(mode), _ptr(alpha), _ptr(gamma), _ptr(beta), _ptr(popc_thresh),
                      _ptr(thresh_mode))
    ep._keep = (alpha, gamma, beta, popc_thresh, thresh_mode)
    return ep


def bnn_binary_linear_fused(A: torch.Tensor, W: torch.Tensor, K: int, ep: bnn_epilogue,
                            out: torch.Tensor, M: Optional[int] = None, N: Optional[int] = None,
                            stream=None) -> None:
    M = A.shape[0] if M is None else M
    N = W.shape[0] if N is None else N
    _check("bnn_binary_linear_fused", _lib.bnn_binary_linear_fused(
        _ptr(A), _ld(A), _ptr(W), _ld(W), M, N, int(K), ctypes.byref(ep), _ptr(out), _ld(out),
        _stream(stream)))


def bnn_binary_conv3x3_fused(X_bits: torch.Tensor, c: int, W_packed: torch.Tensor,
                             ep: bnn_epilogue, out_nchw: torch.Tensor, stride: int = 1, pad: int = 1,
                             stream=None) -> None:
    n, h, w = X_bits.shape[:3]
    cout = W_packed.shape[0]
    _check("bnn_binary_conv3x3_fused", _lib.bnn_binary_conv3x3_fused(
        _ptr(X_bits), n, int(c), h, w, _ptr(W_packed), _ld(W_packed), cout, int(stride), int(pad),
        ctypes.byref(ep), _ptr(out_nchw), _stream(stream)))



def bnn_binary_conv1x1_fused(X_bits: torch.Tensor, c: int, W_packed: torch.Tensor, ep: bnn_epilogue,
                             out_nchw: torch.Tensor, stride: int = 2, stream=None) -> None:
    """Binary 1x1 convolution (stride, no padding) of packed NHWC words."""
    n, h, w = X_bits.shape[:3]
    cout = W_packed.shape[0]
    _check("bnn_binary_conv1x1_fused", _lib.bnn_binary_conv1x1_fused(
        _ptr(X_bits), n, int(c), h, w, _ptr(W_packed), _ld(W_packed), cout, int(stride), ctypes.byref(ep),
        _ptr(out_nchw), _stream(stream)))

def bnn_fold_bn_threshold(alpha: torch.Tensor, gamma: torch.Tensor, beta: torch.Tensor,
                          mean: torch.Tensor, var: torch.Tensor, eps: float, K: int):
    """Host call: returns (popc_thresh int32 [N], thresh_mode int8 [N]) as CPU tensors."""
    ts = [t.detach().to("cpu", torch.float32).contiguous() for t in (alpha, gamma, beta, mean, var)]
    N = ts[0].numel()
    thr = torch.empty(N, dtype=torch.int32)
    mode = torch.empty(N, dtype=torch.int8)
    _check("bnn_fold_bn_threshold", _lib.bnn_fold_bn_threshold(
        *[_ptr(t) for t in ts], float(eps), N, int(K), _ptr(thr), _ptr(mode)))
    return thr, mode


# --------------------------------------------------------------------------
# allocation helpers (torch device memory; the library itself allocates nothing)
# --------------------------------------------------------------------------

def bnn_pack_bit_planes(codes: torch.Tensor, bits: int, planes: torch.Tensor, K: Optional[int] = None,
                        stream=None) -> None:
    """uint8 codes [rows, K] -> plane-interleaved packed planes [rows * bits, ld]."""
    assert codes.dtype == torch.uint8 and codes.dim() == 2 and planes.dtype == torch.int32
    rows = codes.shape[0]
    K = codes.shape[1] if K is None else int(K)
    assert planes.shape[0] == rows * bits
    _check("bnn_pack_bit_planes", _lib.bnn_pack_bit_planes(_ptr(codes), rows, K, _ld(codes), int(bits),
                                                           _ptr(planes), _ld(planes), _stream(stream)))


def bnn_bitserial_gemm(A: torch.Tensor, a_bits: int, W: torch.Tensor, w_bits: int, K: int,
                       alpha: Optional[torch.Tensor] = None, C_i32: Optional[torch.Tensor] = None,
                       C_f32: Optional[torch.Tensor] = None, stream=None) -> None:
    """A, W: plane-interleaved packed planes [M * a_bits, ld], [N * w_bits, ld]."""
    M, N = A.shape[0] // a_bits, W.shape[0] // w_bits
    assert A.shape[0] == M * a_bits and W.shape[0] == N * w_bits
    _check("bnn_bitserial_gemm", _lib.bnn_bitserial_gemm(
        _ptr(A), _ld(A), int(a_bits), _ptr(W), _ld(W), int(w_bits), M, N, int(K), _ptr(alpha),
        _ptr(C_i32), _ld(C_i32) if C_i32 is not None else 0, _ptr(C_f32), _ld(C_f32) if C_f32 is not None else 0,
        _stream(stream)))


def bnn_binary_bases_gemm(H: torch.Tensor, J: int, B: torch.Tensor, I: int, K: int, beta: torch.Tensor,
                          alpha: torch.Tensor, Y: torch.Tensor, stream=None) -> None:
    """H, B: plane-interleaved packed +1/-1 bases [M * J, ld], [N * I, ld]; beta [J]; alpha [I, N]; Y [M, N]."""
    M, N = H.shape[0] // J, B.shape[0] // I
    assert H.shape[0] == M * J and B.shape[0] == N * I and tuple(Y.shape) == (M, N)
    _check("bnn_binary_bases_gemm", _lib.bnn_binary_bases_gemm(
        _ptr(H), _ld(H), int(J), _ptr(B), _ld(B), int(I), M, N, int(K), _ptr(beta), _ptr(alpha), _ld(alpha),
        _ptr(Y), _ld(Y), _stream(stream)))


def empty_packed(rows: int, K: int, device="cuda") -> torch.Tensor:
    """int32-typed storage for a packed [rows, bnn_packed_ld_words(K)] matrix."""
    return torch.empty(rows, bnn_packed_ld_words(K), dtype=torch.int32, device=device)


def empty_ternary(rows: int, K: int, device="cuda") -> torch.Tensor:
    """int32-typed storage for ternary codes [rows, bnn_ternary_ld_words(K)]."""
    return torch.empty(rows, bnn_ternary_ld_words(K), dtype=torch.int32, device=device)


def empty_packed_nhwc(n: int, c: int, h: int, w: int, device="cuda") -> torch.Tensor:
    return torch.empty(n, h, w, (c + 31) // 32, dtype=torch.int32, device=device)


def empty_conv3x3_weights(cout: int, cin: int, device="cuda") -> torch.Tensor:
    return torch.empty(cout, bnn_conv3x3_ld_words(cin), dtype=torch.int32, device=device)
