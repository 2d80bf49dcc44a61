"""Host-side checks of the C ABI (no GPU needed).

The library must build, load, and export every function include/sq.h
declares; layout queries are pure; argument errors come back as status codes
before anything touches a device.
"""
from __future__ import annotations

import ctypes

import pytest

import mixed_precision_gemm_b200 as sq
from mixed_precision_gemm_b200 import _build


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return sq.load()


def test_exports_every_header_function(lib):
    names = sq.header_functions()
    assert {"sq_prepare_weights", "sq_quant_gather", "sq_gemm", "sq_linear"} <= set(names)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in sq.h but not exported"
        assert ctypes.cast(getattr(lib, n), ctypes.c_void_p).value


def test_layout_queries(lib):
    assert sq.sq_kn_pad(256, 8) == 256
    assert sq.sq_kn_pad(4096, 256) == 3840
    assert sq.sq_kn_pad(14336, 1792) == 12544
    assert sq.sq_kn_pad(200, 3) == 256
    assert sq.sq_kn_pad(64, 64) == 0
    assert sq.sq_no_pad(0) == 0 and sq.sq_no_pad(1) == 64 and sq.sq_no_pad(1792) == 1792
    assert sq.sq_chan_table_words(8192) == 1024
    M, K, nO = 2048, 4096, 256
    ws = sq.sq_linear_workspace_bytes(M, K, nO)
    assert ws >= M * 3840 // 2 + 4 * M + 2 * M * 256
    assert ws % 256 == 0
    assert sq.sq_linear_workspace_bytes(0, K, nO) == 0
    for s in range(6):
        assert sq.sq_status_string(s).startswith("SQ_")


P = ctypes.c_void_p


def test_invalid_K_rejected_before_device(lib):
    assert lib.sq_quant_gather(None, 4, 12, 16, None, 0, None, None, None, None) == sq.SQ_ERR_INVALID_ARG
    assert b"multiple of 8" in lib.sq_last_error_detail()
    assert lib.sq_quant_gather(None, 4, 8 * 10000, 80000, None, 0, None, None, None, None) == sq.SQ_ERR_INVALID_ARG


def test_invalid_nO_and_strides(lib):
    assert lib.sq_quant_gather(None, 4, 64, 64, None, 65, None, None, None, None) == sq.SQ_ERR_INVALID_ARG
    assert lib.sq_quant_gather(None, 4, 64, 60, None, 0, None, None, None, None) == sq.SQ_ERR_INVALID_ARG
    assert lib.sq_gemm(None, None, None, None, None, None, 4, 12, 64, 0, None, 16, None, None, None) == sq.SQ_ERR_INVALID_ARG
    assert lib.sq_gemm(None, None, None, None, None, None, 4, 16, 64, 0, None, 12, None, None, None) == sq.SQ_ERR_INVALID_ARG


def test_misaligned_pointer_rejected(lib):
    st = lib.sq_quant_gather(P(0x1008), 4, 64, 64, P(0x2000), 0, P(0x3000), P(0x4000), None, None)
    assert st == sq.SQ_ERR_MISALIGNED
    st = lib.sq_gemm(P(0x1000), P(0x2000), None, P(0x3004), P(0x4000), None, 4, 16, 64, 0, P(0x5000), 16,
                     None, None, None)
    assert st == sq.SQ_ERR_MISALIGNED


def test_null_operand_rejected(lib):
    st = lib.sq_gemm(P(0x1000), P(0x2000), None, P(0x3000), P(0x4000), None, 4, 16, 64, 8, P(0x5000), 16,
                     None, None, None)
    assert st == sq.SQ_ERR_INVALID_ARG  # nO > 0 needs X_O and W_O
    assert b"X_O" in lib.sq_last_error_detail()


@pytest.mark.parametrize("O", [[3, 1], [2, 2], [-1], [64]])
def test_bad_outlier_set_rejected(lib, O):
    arr = (ctypes.c_int32 * len(O))(*O)
    st = lib.sq_prepare_weights(P(0x1000), 16, 64, 64, arr, len(O), P(0x2000), P(0x3000), P(0x4000), P(0x5000), None)
    assert st == sq.SQ_ERR_INVALID_ARG


def test_workspace_too_small_rejected(lib):
    need = lib.sq_linear_workspace_bytes(8, 64, 8)
    st = lib.sq_linear(P(0x1000), 8, 64, 64, P(0x2000), P(0x3000), P(0x4000), P(0x5000), 16, 8, P(0x6000), 16,
                       P(0x7000), need - 1, None)
    assert st == sq.SQ_ERR_INVALID_ARG


def test_watchdog_timeout_range_checked(lib):
    assert lib.sq_selftest_watchdog(0, None) == sq.SQ_ERR_INVALID_ARG
    assert lib.sq_selftest_watchdog(20000, None) == sq.SQ_ERR_INVALID_ARG


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(sq, "_lib", None)
    monkeypatch.setattr(_build, "LIB_PATH", str(tmp_path / "nope.so"))
    with pytest.raises(RuntimeError, match="missing"):
        sq.load()


def test_mx_layout_queries(lib):
    assert sq.sq_kn_pad_mx(4096, 256) == 3840
    assert sq.sq_kn_pad_mx(1040, 24) == 1024
    assert sq.sq_kn_pad_mx(200, 3) == 256
    assert sq.sq_kn_pad_mx(64, 64) == 0
    # 128-row bands of one byte per 32 codes
    assert sq.sq_mx_scale_bytes(300, 4096, 256) == 384 * 3840 // 32
    assert sq.sq_mx_scale_bytes(128, 4096, 0) == 128 * 4096 // 32
    assert sq.sq_mx_scale_bytes(0, 4096, 0) == 0
    assert sq.sq_mx_scale_bytes(5, 64, 64) == 0
    M, K, nO = 2048, 4096, 256
    ws = sq.sq_linear_workspace_bytes_mx(M, K, nO)
    assert ws >= M * 3840 // 2 + sq.sq_mx_scale_bytes(M, K, nO) + 2 * M * 256 and ws % 256 == 0
    assert sq.sq_linear_workspace_bytes_mx(0, K, nO) == 0


def test_mx_argument_errors_before_device(lib):
    assert lib.sq_quant_gather_mx(None, 4, 12, 16, None, 0, None, None, None, None) == sq.SQ_ERR_INVALID_ARG
    assert lib.sq_quant_gather_mx(None, 4, 64, 60, None, 0, None, None, None, None) == sq.SQ_ERR_INVALID_ARG
    assert lib.sq_gemm_mx(None, None, None, None, None, None, 4, 12, 64, 0, None, 16, None, None) == \
        sq.SQ_ERR_INVALID_ARG
    assert lib.sq_gemm_mx(None, None, None, None, None, None, 4, 16, 64, 0, None, 16, None, None) == \
        sq.SQ_ERR_INVALID_ARG   # NULL operands
    buf = ctypes.create_string_buffer(64)
    mis = ctypes.c_void_p(ctypes.addressof(buf) + 1)
    assert lib.sq_gemm_mx(mis, mis, None, mis, mis, None, 4, 16, 64, 0, mis, 16, None, None) == sq.SQ_ERR_MISALIGNED
    assert lib.sq_linear_mx(None, 4, 64, 64, None, None, None, None, 16, 0, None, 16, None, 0, None) == \
        sq.SQ_ERR_INVALID_ARG   # workspace too small
    O = (ctypes.c_int32 * 2)(5, 3)
    assert lib.sq_prepare_weights_mx(None, 4, 64, 64, O, 2, None, None, None, None, None) == sq.SQ_ERR_INVALID_ARG
