"""The C ABI without a GPU: the library loads, exports every symbol that
include/bnn.h declares, and rejects bad arguments on the host before any CUDA
call (so these checks run on a machine without a GPU)."""
import ctypes
import os
import re

import pytest

import oracle
import xnor_popcount_gemm_bnn_b200 as bnn

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "bnn.h")
FAKE = ctypes.c_void_p(0x10000)        # aligned, never dereferenced: validation fails first
FAKE_ODD = ctypes.c_void_p(0x10004)    # 4-byte but not 16-byte aligned
NULL = None


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bnn_[a-z0-9_]+)\s*\(", text)))


def test_header_declarations_match_binding():
    assert declared_functions() == sorted(bnn.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(bnn.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_packed_ld_words_matches_layout_reading():
    for K in (1, 31, 32, 33, 127, 128, 129, 576, 1000, 4095, 4096, 4097, 8192, 123457):
        assert bnn.bnn_packed_ld_words(K) == oracle.ld_words(K)
    assert bnn.bnn_packed_ld_words(0) == -1
    assert bnn.bnn_conv3x3_ld_words(64) == 20      # 9 taps x 2 words, rounded to 4
    assert bnn.bnn_conv3x3_ld_words(1) == 12
    assert bnn.bnn_conv3x3_ld_words(128) == 36
    assert bnn.bnn_conv3x3_ld_words(0) == -1


def test_status_strings():
    for s in range(6):
        assert isinstance(bnn.bnn_status_string(s), str) and bnn.bnn_status_string(s)
    assert bnn.bnn_status_string(99) == "unknown status"


L = bnn.lib


def test_pack_sign_rejects_bad_arguments():
    st = L.bnn_pack_sign
    assert st(NULL, 0, 4, 32, 32, FAKE, 4, NULL, NULL) == bnn.BNN_ERR_INVALID_ARG
    assert st(FAKE, 0, 4, 0, 32, FAKE, 4, NULL, NULL) == bnn.BNN_ERR_INVALID_ARG      # K < 1
    assert st(FAKE, 0, 4, 64, 32, FAKE, 4, NULL, NULL) == bnn.BNN_ERR_INVALID_ARG     # ld_x < K
    assert st(FAKE, 0, 4, 200, 200, FAKE, 4, NULL, NULL) == bnn.BNN_ERR_INVALID_ARG   # ld too small
    assert st(FAKE, 0, 4, 32, 32, FAKE, 6, NULL, NULL) == bnn.BNN_ERR_ALIGNMENT       # ld % 4
    assert st(FAKE, 0, 4, 32, 32, FAKE_ODD, 4, NULL, NULL) == bnn.BNN_ERR_ALIGNMENT
    assert st(FAKE, 7, 4, 32, 32, FAKE, 4, NULL, NULL) == bnn.BNN_ERR_INVALID_ARG     # dtype
    assert st(FAKE, 0, -1, 32, 32, FAKE, 4, NULL, NULL) == bnn.BNN_ERR_INVALID_ARG
    assert st(FAKE, 0, 0, 32, 32, FAKE, 4, NULL, NULL) == bnn.BNN_OK                  # empty: no launch


def test_gemm_rejects_bad_arguments():
    g = L.bnn_xnor_gemm
    ok = dict()
    assert g(NULL, 4, FAKE, 4, 8, 8, 32, NULL, FAKE, 8, NULL, 0, NULL) == bnn.BNN_ERR_INVALID_ARG
    assert g(FAKE, 4, FAKE, 4, 8, 8, 0, NULL, FAKE, 8, NULL, 0, NULL) == bnn.BNN_ERR_INVALID_ARG
    assert g(FAKE, 4, FAKE, 4, 8, 8, 32, NULL, NULL, 0, NULL, 0, NULL) == bnn.BNN_ERR_INVALID_ARG  # no output
    assert g(FAKE, 4, FAKE, 4, 8, 8, 32, NULL, NULL, 0, FAKE, 8, NULL) == bnn.BNN_ERR_INVALID_ARG  # f32 w/o alpha
    assert g(FAKE, 4, FAKE, 4, 8, 8, 32, NULL, FAKE, 7, NULL, 0, NULL) == bnn.BNN_ERR_INVALID_ARG  # ldc < N
    assert g(FAKE, 2, FAKE, 4, 8, 8, 32, NULL, FAKE, 8, NULL, 0, NULL) == bnn.BNN_ERR_INVALID_ARG  # lda < kw
    assert g(FAKE, 6, FAKE, 4, 8, 8, 32, NULL, FAKE, 8, NULL, 0, NULL) == bnn.BNN_ERR_ALIGNMENT    # lda % 4
    assert g(FAKE_ODD, 4, FAKE, 4, 8, 8, 32, NULL, FAKE, 8, NULL, 0, NULL) == bnn.BNN_ERR_ALIGNMENT
    assert g(FAKE, 4, FAKE, 4, -1, 8, 32, NULL, FAKE, 8, NULL, 0, NULL) == bnn.BNN_ERR_INVALID_ARG
    assert g(FAKE, 4, FAKE, 4, 0, 8, 32, NULL, FAKE, 8, NULL, 0, NULL) == bnn.BNN_OK               # M = 0
    assert g(FAKE, 4, FAKE, 4, 8, 0, 32, NULL, FAKE, 8, NULL, 0, NULL) == bnn.BNN_OK               # N = 0
    del ok


def test_linear_fused_rejects_bad_epilogues():
    f = L.bnn_binary_linear_fused
    def ep(mode, **kw):
        e = bnn.bnn_epilogue(mode, None, None, None, None, None)
        for k, v in kw.items():
            setattr(e, k, v)
        return ctypes.byref(e)
    args = (FAKE, 4, FAKE, 4, 8, 8, 32)
    assert f(*args, NULL, FAKE, 8, NULL) == bnn.BNN_ERR_INVALID_ARG
    assert f(*args, ep(99), FAKE, 8, NULL) == bnn.BNN_ERR_INVALID_ARG
    assert f(*args, ep(bnn.BNN_OUT_SCALED_F32), FAKE, 8, NULL) == bnn.BNN_ERR_INVALID_ARG
    assert f(*args, ep(bnn.BNN_OUT_AFFINE_F32, alpha=0x10000), FAKE, 8, NULL) == bnn.BNN_ERR_INVALID_ARG
    assert f(*args, ep(bnn.BNN_OUT_THRESHOLD_PACK), FAKE, 4, NULL) == bnn.BNN_ERR_INVALID_ARG
    assert f(*args, ep(bnn.BNN_OUT_THRESHOLD_PACK, popc_thresh=0x10000, thresh_mode=0x10000),
             FAKE, 2, NULL) == bnn.BNN_ERR_INVALID_ARG     # ld_out < ld_words(N)
    assert f(*args, ep(bnn.BNN_OUT_THRESHOLD_PACK, popc_thresh=0x10000, thresh_mode=0x10000),
             FAKE, 6, NULL) == bnn.BNN_ERR_ALIGNMENT
    assert f(*args, ep(bnn.BNN_OUT_INT32), FAKE, 7, NULL) == bnn.BNN_ERR_INVALID_ARG


def test_gemv_rejects_bad_arguments():
    g = L.bnn_xnor_gemv
    assert g(FAKE, 4, NULL, 0, 8, 32, NULL, FAKE, NULL, NULL) == bnn.BNN_ERR_INVALID_ARG
    assert g(FAKE, 4, FAKE, 0, 8, 32, NULL, NULL, NULL, NULL) == bnn.BNN_ERR_INVALID_ARG
    assert g(FAKE, 4, FAKE, 0, 8, 32, NULL, NULL, FAKE, NULL) == bnn.BNN_ERR_INVALID_ARG   # f32 w/o alpha
    assert g(FAKE, 4, FAKE, 0, 8, 129, NULL, FAKE, NULL, NULL) == bnn.BNN_ERR_INVALID_ARG  # ldw < kw
    assert g(FAKE_ODD, 4, FAKE, 0, 8, 32, NULL, FAKE, NULL, NULL) == bnn.BNN_ERR_ALIGNMENT
    assert g(FAKE, 4, FAKE, 5, 8, 32, NULL, FAKE, NULL, NULL) == bnn.BNN_ERR_INVALID_ARG
    assert g(FAKE, 4, FAKE, 0, 0, 32, NULL, FAKE, NULL, NULL) == bnn.BNN_OK


def test_gemv_ex_rejects_bad_flags():
    g = L.bnn_xnor_gemv_ex
    assert g(FAKE, 4, FAKE, 0, 8, 32, NULL, FAKE, NULL, 8, NULL) == bnn.BNN_ERR_INVALID_ARG
    assert g(FAKE, 4, FAKE, 0, 8, 32, NULL, FAKE, NULL, 15, NULL) == bnn.BNN_ERR_INVALID_ARG
    for flags in range(8):
        assert g(FAKE, 4, FAKE, 0, 0, 32, NULL, FAKE, NULL, flags, NULL) == bnn.BNN_OK


def test_conv_rejects_bad_arguments():
    c = L.bnn_binary_conv3x3_fused
    e = bnn.bnn_epilogue(bnn.BNN_OUT_INT32, None, None, None, None, None)
    E = ctypes.byref(e)
    assert c(NULL, 1, 64, 8, 8, FAKE, 20, 4, 1, 1, E, FAKE, NULL) == bnn.BNN_ERR_INVALID_ARG
    assert c(FAKE, 1, 64, 8, 8, FAKE, 17, 4, 1, 1, E, FAKE, NULL) == bnn.BNN_ERR_INVALID_ARG   # ldw < 18
    assert c(FAKE, 1, 64, 8, 8, FAKE, 20, 4, 0, 1, E, FAKE, NULL) == bnn.BNN_ERR_INVALID_ARG   # stride
    assert c(FAKE, 1, 64, 1, 1, FAKE, 20, 4, 1, 0, E, FAKE, NULL) == bnn.BNN_ERR_INVALID_ARG   # no output
    assert c(FAKE, 1, 160, 8, 8, FAKE, 48, 4, 1, 1, E, FAKE, NULL) == bnn.BNN_ERR_UNSUPPORTED  # c > 128
    e2 = bnn.bnn_epilogue(bnn.BNN_OUT_THRESHOLD_PACK, None, None, None, None, None)
    assert c(FAKE, 1, 64, 8, 8, FAKE, 20, 4, 1, 1, ctypes.byref(e2), FAKE, NULL) == bnn.BNN_ERR_UNSUPPORTED
    assert c(FAKE, 0, 64, 8, 8, FAKE, 20, 4, 1, 1, E, FAKE, NULL) == bnn.BNN_OK


def test_fold_rejects_bad_arguments():
    import torch
    a = torch.ones(4)
    with pytest.raises(bnn.BnnError):
        bnn.bnn_fold_bn_threshold(a, a, a, a, a * 0 - 1.0, 0.0, 16)         # var + eps <= 0
    with pytest.raises(bnn.BnnError):
        bnn.bnn_fold_bn_threshold(a * float("nan"), a, a, a, a, 1e-5, 16)   # non-finite
    with pytest.raises(bnn.BnnError):
        bnn.bnn_fold_bn_threshold(-a, a, a, a, a, 1e-5, 16)                 # alpha < 0
    with pytest.raises(bnn.BnnError):
        bnn.bnn_fold_bn_threshold(a, a, a, a, a, 1e-5, 0)                   # K < 1


def test_gemm_engine_setting_on_host():
    prev = bnn.bnn_get_gemm_engine()
    assert L.bnn_set_gemm_engine(4) == bnn.BNN_ERR_INVALID_ARG
    assert L.bnn_set_gemm_engine(-1) == bnn.BNN_ERR_INVALID_ARG
    assert L.bnn_set_gemm_engine(bnn.BNN_GEMM_ENGINE_TENSOR) == bnn.BNN_OK
    assert bnn.bnn_get_gemm_engine() == bnn.BNN_GEMM_ENGINE_TENSOR
    assert L.bnn_set_gemm_engine(bnn.BNN_GEMM_ENGINE_TENSOR_I8) == bnn.BNN_OK
    assert bnn.bnn_get_gemm_engine() == bnn.BNN_GEMM_ENGINE_TENSOR_I8
    bnn.bnn_set_gemm_engine(prev)


def test_gemv_host_entry_rejects_bad_arguments():
    f = L.bnn_xnor_gemv_host
    # W, ldw, x_host, dt, N, K, alpha, x_dev, y_dev, y_host, flags, stream
    assert f(FAKE, 128, FAKE, 1, 8, 4096, FAKE, FAKE, FAKE, FAKE, 8, NULL) == bnn.BNN_ERR_INVALID_ARG    # unknown bit
    assert f(FAKE, 128, FAKE, 1, 8, 4096, FAKE, FAKE, FAKE, FAKE, 7, NULL) == bnn.BNN_ERR_INVALID_ARG    # all three
    assert f(FAKE, 128, FAKE, 1, 8, 4096, FAKE, FAKE, FAKE, FAKE, 4, NULL) == bnn.BNN_ERR_INVALID_ARG    # output free
    assert f(FAKE, 128, NULL, 1, 8, 4096, FAKE, FAKE, FAKE, FAKE, 0, NULL) == bnn.BNN_ERR_INVALID_ARG    # no x_host
    assert f(FAKE, 128, FAKE, 1, 8, 4096, FAKE, NULL, FAKE, FAKE, 0, NULL) == bnn.BNN_ERR_INVALID_ARG    # no x_dev
    assert f(FAKE, 128, FAKE, 1, 8, 4096, FAKE, FAKE, FAKE, NULL, 0, NULL) == bnn.BNN_ERR_INVALID_ARG    # no y_host
    assert f(FAKE, 128, FAKE, 1, 8, 4096, NULL, FAKE, FAKE, FAKE, 0, NULL) == bnn.BNN_ERR_INVALID_ARG    # no alpha
    assert f(FAKE, 128, FAKE, 7, 8, 4096, FAKE, FAKE, FAKE, FAKE, 0, NULL) == bnn.BNN_ERR_INVALID_ARG    # dtype
    assert f(FAKE, 128, FAKE, 1, 8, 0, FAKE, FAKE, FAKE, FAKE, 0, NULL) == bnn.BNN_ERR_INVALID_ARG       # K < 1
    assert f(FAKE, 128, FAKE, 1, 8, 4096, FAKE, FAKE_ODD, FAKE, FAKE, 0, NULL) == bnn.BNN_ERR_ALIGNMENT  # x_dev


def test_binary_weight_gemv_rejects_bad_arguments():
    f = L.bnn_binary_weight_gemv
    assert f(FAKE, 4, FAKE, 0, 8, 32, FAKE, FAKE, 8, NULL) == bnn.BNN_ERR_INVALID_ARG       # unknown flag
    assert f(FAKE, 4, NULL, 0, 8, 32, FAKE, FAKE, 0, NULL) == bnn.BNN_ERR_INVALID_ARG       # no x
    assert f(FAKE, 4, FAKE, 0, 8, 32, NULL, FAKE, 0, NULL) == bnn.BNN_ERR_INVALID_ARG       # alpha required
    assert f(FAKE, 4, FAKE, 0, 8, 32, FAKE, NULL, 0, NULL) == bnn.BNN_ERR_INVALID_ARG       # no y
    assert f(FAKE, 4, FAKE, 7, 8, 32, FAKE, FAKE, 0, NULL) == bnn.BNN_ERR_INVALID_ARG       # dtype
    assert f(FAKE, 6, FAKE, 0, 8, 32, FAKE, FAKE, 0, NULL) == bnn.BNN_ERR_ALIGNMENT         # ld % 4
    assert f(FAKE_ODD, 4, FAKE, 0, 8, 32, FAKE, FAKE, 0, NULL) == bnn.BNN_ERR_ALIGNMENT
    assert f(FAKE, 388, FAKE, 0, 8, 12289, FAKE, FAKE, 0, NULL) == bnn.BNN_ERR_UNSUPPORTED  # table too large
    assert f(FAKE, 4, FAKE, 0, 0, 32, FAKE, FAKE, 7, NULL) == bnn.BNN_OK                    # N = 0: nothing to do


def test_make_epilogue_keeps_its_tensors_alive():
    """The struct holds raw pointers; it must keep the tensors it points into
    alive (e.g. temporaries from ``t.to(device)``)."""
    import gc
    import weakref
    import torch
    ep = bnn.make_epilogue(bnn.BNN_OUT_AFFINE_F32, alpha=torch.ones(3), gamma=torch.ones(3), beta=torch.zeros(3))
    refs = [weakref.ref(t) for t in ep._keep if t is not None]
    gc.collect()
    assert len(refs) == 3 and all(r() is not None for r in refs)


def test_ternary_layout_sizes():
    """Ternary row length and workspace size match the layout reading (2 bits
    per weight, rows of whole 16-byte units) as the oracle states it."""
    for K in (1, 15, 16, 17, 64, 65, 1000, 4096, 11008):
        assert bnn.bnn_ternary_ld_words(K) == oracle.ternary_ld_words(K)
    assert bnn.bnn_ternary_ld_words(0) == -1
    assert bnn.bnn_ternary_workspace_bytes(11008) == 8 * 11009
    assert bnn.bnn_ternary_workspace_bytes(-1) == -1


def test_ternary_pack_rejects_bad_arguments():
    f = L.bnn_ternary_pack
    ws = 8 * 9
    assert f(NULL, 0, 8, 32, 32, -1.0, FAKE, 4, NULL, FAKE, ws, NULL) == bnn.BNN_ERR_INVALID_ARG    # no w
    assert f(FAKE, 0, 8, 32, 32, -1.0, NULL, 4, NULL, FAKE, ws, NULL) == bnn.BNN_ERR_INVALID_ARG    # no codes
    assert f(FAKE, 0, 8, 32, 31, -1.0, FAKE, 4, NULL, FAKE, ws, NULL) == bnn.BNN_ERR_INVALID_ARG    # ld_w < K
    assert f(FAKE, 5, 8, 32, 32, -1.0, FAKE, 4, NULL, FAKE, ws, NULL) == bnn.BNN_ERR_INVALID_ARG    # dtype
    assert f(FAKE, 0, 8, 32, 32, float("nan"), FAKE, 4, NULL, NULL, 0, NULL) == bnn.BNN_ERR_INVALID_ARG
    assert f(FAKE, 0, 8, 100, 100, -1.0, FAKE, 4, NULL, FAKE, ws, NULL) == bnn.BNN_ERR_INVALID_ARG  # ldq < 8
    assert f(FAKE, 0, 8, 32, 32, -1.0, FAKE, 4, NULL, NULL, 0, NULL) == bnn.BNN_ERR_INVALID_ARG     # eq. (9) needs ws
    assert f(FAKE, 0, 8, 32, 32, -1.0, FAKE, 4, NULL, FAKE, ws - 8, NULL) == bnn.BNN_ERR_INVALID_ARG  # ws too small
    assert f(FAKE, 0, 8, 32, 32, 0.5, FAKE, 4, FAKE, NULL, 0, NULL) == bnn.BNN_ERR_INVALID_ARG      # gamma_out needs ws
    assert f(FAKE, 0, 8, 32, 32, -1.0, FAKE, 6, NULL, FAKE, ws, NULL) == bnn.BNN_ERR_ALIGNMENT      # ldq % 4
    assert f(FAKE, 0, 8, 32, 32, -1.0, FAKE_ODD, 4, NULL, FAKE, ws, NULL) == bnn.BNN_ERR_ALIGNMENT
    assert f(FAKE, 0, 8, 32, 32, -1.0, FAKE, 4, NULL, ctypes.c_void_p(0x10004), ws, NULL) == bnn.BNN_ERR_ALIGNMENT
    assert f(FAKE, 0, 0, 32, 32, 0.5, FAKE, 4, NULL, NULL, 0, NULL) == bnn.BNN_OK                  # rows = 0


def test_ternary_gemv_rejects_bad_arguments():
    f = L.bnn_ternary_gemv_i8
    assert f(FAKE, 4, FAKE, 8, 32, NULL, NULL, FAKE, NULL, 8, NULL) == bnn.BNN_ERR_INVALID_ARG   # unknown flag
    assert f(NULL, 4, FAKE, 8, 32, NULL, NULL, FAKE, NULL, 0, NULL) == bnn.BNN_ERR_INVALID_ARG   # no codes
    assert f(FAKE, 4, NULL, 8, 32, NULL, NULL, FAKE, NULL, 0, NULL) == bnn.BNN_ERR_INVALID_ARG   # no x
    assert f(FAKE, 4, FAKE, 8, 32, NULL, NULL, NULL, NULL, 0, NULL) == bnn.BNN_ERR_INVALID_ARG   # no output
    assert f(FAKE, 4, FAKE, 8, 100, NULL, NULL, FAKE, NULL, 0, NULL) == bnn.BNN_ERR_INVALID_ARG  # ldq too small
    assert f(FAKE, 6, FAKE, 8, 32, NULL, NULL, FAKE, NULL, 0, NULL) == bnn.BNN_ERR_ALIGNMENT     # ldq % 4
    assert f(FAKE_ODD, 4, FAKE, 8, 32, NULL, NULL, FAKE, NULL, 0, NULL) == bnn.BNN_ERR_ALIGNMENT
    assert f(FAKE, 4, FAKE, 8, 32, NULL, NULL, ctypes.c_void_p(0x10002), NULL, 0, NULL) == bnn.BNN_ERR_ALIGNMENT
    assert f(FAKE, 6148, FAKE, 8, 98305, NULL, NULL, FAKE, NULL, 0, NULL) == bnn.BNN_ERR_UNSUPPORTED
    assert f(FAKE, 4, FAKE, 0, 32, NULL, NULL, FAKE, NULL, 7, NULL) == bnn.BNN_OK                # N = 0


def test_rsign_packs_reject_bad_arguments():
    f, g = L.bnn_pack_sign_rsign, L.bnn_pack_sign_nchw_rsign
    assert f(FAKE, 0, 8, 32, 32, NULL, FAKE, 4, NULL) == bnn.BNN_ERR_INVALID_ARG               # beta required
    assert f(FAKE, 0, 8, 32, 32, ctypes.c_void_p(0x10002), FAKE, 4, NULL) == bnn.BNN_ERR_ALIGNMENT
    assert f(FAKE, 0, 8, 32, 31, FAKE, FAKE, 4, NULL) == bnn.BNN_ERR_INVALID_ARG               # ld_x < K
    assert f(FAKE, 0, 0, 32, 32, FAKE, FAKE, 4, NULL) == bnn.BNN_OK                            # rows = 0
    assert g(FAKE, 0, 2, 64, 5, 5, NULL, FAKE, NULL) == bnn.BNN_ERR_INVALID_ARG                # beta required
    assert g(FAKE, 0, 2, 64, 5, 5, ctypes.c_void_p(0x10002), FAKE, NULL) == bnn.BNN_ERR_ALIGNMENT
    assert g(FAKE, 0, 0, 64, 5, 5, FAKE, FAKE, NULL) == bnn.BNN_OK                             # n = 0


def test_conv1x1_rejects_bad_arguments():
    f = L.bnn_binary_conv1x1_fused
    ep = bnn.make_epilogue(bnn.BNN_OUT_INT32)
    epb = ctypes.byref(ep)
    assert f(NULL, 2, 64, 8, 8, FAKE, 4, 16, 2, epb, FAKE, NULL) == bnn.BNN_ERR_INVALID_ARG     # no input
    assert f(FAKE, 2, 64, 8, 8, FAKE, 4, 16, 0, epb, FAKE, NULL) == bnn.BNN_ERR_INVALID_ARG     # stride 0
    assert f(FAKE, 2, 64, 8, 8, FAKE, 1, 16, 2, epb, FAKE, NULL) == bnn.BNN_ERR_INVALID_ARG     # ldw < cw
    assert f(FAKE, 2, 600, 8, 8, FAKE, 20, 16, 2, epb, FAKE, NULL) == bnn.BNN_ERR_UNSUPPORTED   # c > 512
    thr = bnn.make_epilogue(bnn.BNN_OUT_THRESHOLD_PACK)
    assert f(FAKE, 2, 64, 8, 8, FAKE, 4, 16, 2, ctypes.byref(thr), FAKE, NULL) == bnn.BNN_ERR_UNSUPPORTED
    sc = bnn.make_epilogue(bnn.BNN_OUT_SCALED_F32)
    assert f(FAKE, 2, 64, 8, 8, FAKE, 4, 16, 2, ctypes.byref(sc), FAKE, NULL) == bnn.BNN_ERR_INVALID_ARG  # no alpha
    assert f(FAKE, 0, 64, 8, 8, FAKE, 4, 16, 2, epb, FAKE, NULL) == bnn.BNN_OK                   # n = 0


def test_conv1x1_rejects_indices_past_32_bits():
    """n*oh*ow at or past 2^31 - 4096 is refused before any launch."""
    ep = bnn.make_epilogue(bnn.BNN_OUT_INT32)
    st = L.bnn_binary_conv1x1_fused(FAKE, 1 << 22, 64, 64, 64, FAKE, 4, 16, 2, ctypes.byref(ep), FAKE, NULL)
    assert st == bnn.BNN_ERR_UNSUPPORTED


def test_header_constants_match_binding():
    """Numeric constants of include/bnn.h (enums, #defines) equal the binding's."""
    text = open(HEADER).read()
    m = re.search(r"#define\s+BNN_TERNARY_PACK_NOALLOC_MAX_ROWS\s+(\d+)", text)
    assert m and int(m.group(1)) == bnn.BNN_TERNARY_PACK_NOALLOC_MAX_ROWS
    for name in ("BNN_GEMV_WEIGHTS_STATIC", "BNN_GEMV_INPUTS_STATIC", "BNN_GEMV_OUTPUT_FREE", "BNN_OUT_INT32",
                 "BNN_OUT_SCALED_F32", "BNN_OUT_AFFINE_F32", "BNN_OUT_THRESHOLD_PACK", "BNN_GEMM_ENGINE_AUTO",
                 "BNN_GEMM_ENGINE_POPCOUNT", "BNN_GEMM_ENGINE_TENSOR", "BNN_GEMM_ENGINE_TENSOR_I8", "BNN_F32", "BNN_BF16",
                 "BNN_ERR_DEVICE_TIMEOUT"):
        m = re.search(rf"\b{name}\s*=\s*(\d+)", text)
        assert m, name
        assert int(m.group(1)) == getattr(bnn, name), name


def test_gemv_chain_rejects_bad_arguments():
    f = L.bnn_xnor_gemv_chain
    assert bnn.bnn_gemv_chain_workspace_words() == 16 + 4 * 512 * 2

    def layers(*specs):       # (W, ldw, N, popc_thresh, thresh_mode, alpha)
        arr = (bnn.bnn_chain_layer * len(specs))()
        for i, s in enumerate(specs):
            arr[i] = bnn.bnn_chain_layer(*s)
        return arr

    W, T, M, A = 0x10000, 0x20000, 0x30000, 0x40000
    good = layers((W, 32, 64, T, M, None), (W, 4, 10, None, None, A))   # K = 1000 -> 64 -> 10
    INV, ALN, UNS = bnn.BNN_ERR_INVALID_ARG, bnn.BNN_ERR_ALIGNMENT, bnn.BNN_ERR_UNSUPPORTED

    def call(arr=good, n=2, x=FAKE, dt=0, K=1000, yi=FAKE, yf=FAKE, acts=NULL, ld_acts=0, ws=FAKE):
        return f(arr, n, x, dt, K, yi, yf, acts, ld_acts, ws, NULL)

    assert call(arr=NULL) == INV
    assert call(n=0) == INV
    assert call(n=17) == INV
    assert call(x=NULL) == INV
    assert call(dt=7) == INV
    assert call(K=0) == INV
    assert call(yi=NULL, yf=NULL) == INV
    assert call(ws=NULL) == INV
    assert call(ws=FAKE_ODD) == ALN
    assert call(acts=FAKE, ld_acts=2) == INV                                  # hidden N = 64 needs 4 words
    assert call(arr=layers((W, 32, 0, T, M, None), (W, 4, 10, None, None, A))) == INV       # N = 0
    assert call(arr=layers((W, 32, 64, NULL, M, None), (W, 4, 10, None, None, A))) == INV   # no thresholds
    assert call(arr=layers((W, 32, 64, T, NULL, None), (W, 4, 10, None, None, A))) == INV
    assert call(arr=layers((W, 32, 64, T, M, None), (W, 4, 10, None, None, None))) == INV   # y_f32 needs alpha
    assert call(arr=layers((W, 28, 64, T, M, None), (W, 4, 10, None, None, A))) == INV      # ldw < words of K
    assert call(arr=layers((W, 34, 64, T, M, None), (W, 4, 10, None, None, A))) == ALN      # ldw % 4
    assert call(arr=layers((0x10008, 32, 64, T, M, None), (W, 4, 10, None, None, A))) == ALN
    assert call(arr=layers((W, 516, 64, T, M, None), (W, 4, 10, None, None, A)), K=16385) == UNS
    assert call(arr=layers((W, 32, 16385, T, M, None), (W, 516, 10, None, None, A))) == UNS  # hidden N > 16384
