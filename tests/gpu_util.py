"""Helpers for the GPU parity tests (comparison rules, device transfer)."""
import numpy as np
import torch

# fp32 outputs: |y - y_ref| <= REL * |y_ref| for alpha*s (alpha*0 must be exactly 0);
# |y - y_ref| <= REL * (|gamma*alpha*s| + |beta|) for the affine epilogue, whose
# two terms may cancel.  Integers and packed bits: bit-exact.
REL = 1e-6


def dev():
    return torch.device("cuda", torch.cuda.current_device())


def u32(t: torch.Tensor) -> np.ndarray:
    """uint32 view of an int32-stored packed tensor, on the host."""
    return t.detach().cpu().contiguous().numpy().view(np.uint32)


def assert_scaled_close(y: torch.Tensor, y_ref: np.ndarray):
    y = y.detach().cpu().numpy().astype(np.float64)
    assert y.shape == y_ref.shape, (y.shape, y_ref.shape)
    err = np.abs(y - y_ref)
    bad = err > REL * np.abs(y_ref)
    assert not bad.any(), (f"{bad.sum()} fp32 outputs beyond {REL} relative; worst at "
                           f"{np.unravel_index(np.argmax(err / np.maximum(np.abs(y_ref), 1e-300)), y.shape)}")
    assert np.all(y[y_ref == 0] == 0)


def assert_affine_close(y: torch.Tensor, y_ref: np.ndarray, scale: np.ndarray):
    y = y.detach().cpu().numpy().astype(np.float64)
    assert y.shape == y_ref.shape
    err = np.abs(y - y_ref)
    bad = err > REL * scale
    assert not bad.any(), f"{bad.sum()} affine outputs beyond tolerance; max err {err.max()}"


def assert_no_device_error():
    import xnor_popcount_gemm_bnn_b200 as bnn
    assert bnn.bnn_device_error() == 0
