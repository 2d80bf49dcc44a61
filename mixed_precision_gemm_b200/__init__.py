"""Dual-path sparse-quantized linear layer on B200 (sm_100a).

    Y = s_x[m] * s_w[n] * sum_{k not in O} q4(X)[m,k] * q4(W)[n,k]  +  sum_{k in O} X[m,k] * W[n,k]

A thin Python binding of the C ABI in ``include/sq.h`` (library
``libsq_b200.so``, built from ``csrc/``).  Every step of the layer runs in the
library's CUDA kernels; this module only checks tensor metadata, marshals
pointers and sizes, and allocates buffers with torch.  There is no CPU
fallback: if the library is missing the calls raise.

The ABI calls keep their C names (``sq_prepare_weights``, ``sq_quant_gather``,
``sq_gemm``, ``sq_linear``, ...).  ``prepare_weights`` / ``SQLinear`` are
small conveniences that allocate the buffers and call them.

Method: OSC (arXiv:2604.12782, abstract and technical framework) -- static
outlier channels coalesced into a compact bf16 tensor for a 16-bit branch
GEMM, all other channels through a 4-bit GEMM, results fused; SQ-format
write-up of arXiv:2512.05409, sections 5 and 9 -- static mask chosen offline,
symmetric quantization, weight columns reordered by the mask.  Two more low
paths keep the same split: FP8 E4M3 (OSC's fallback for the inputs of W2)
and MXFP4 (OSC abstract: the split fits 4-bit micro-scaling hardware).
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import re
from typing import Optional, Sequence

import torch

from . import _build

__all__ = [
    "SQError", "load", "library_path", "header_functions",
    "sq_status_string", "sq_kn_pad", "sq_no_pad", "sq_chan_table_words", "sq_linear_workspace_bytes",
    "sq_prepare_weights", "sq_quant_gather", "sq_gemm", "sq_linear", "sq_linear_noalloc", "sq_check",
    "sq_selftest_watchdog", "sq_linear_workspace_bytes_fp8", "sq_prepare_weights_fp8", "sq_quant_gather_fp8",
    "sq_gemm_fp8", "sq_linear_fp8", "sq_kn_pad_mx", "sq_mx_scale_bytes", "sq_linear_workspace_bytes_mx",
    "sq_prepare_weights_mx", "sq_quant_gather_mx", "sq_gemm_mx", "sq_linear_mx",
    "sq_linear_workspace_bytes_sqf", "sq_prepare_weights_sqf", "sq_quant_gather_sqf", "sq_gemm_sqf", "sq_linear_sqf",
    "PreparedSQF", "prepare_weights_sqf", "quant_gather_sqf", "gemm_sqf",
    "sq_select_outliers_workspace_bytes", "sq_select_outliers", "select_outliers",
    "PreparedWeights", "prepare_weights", "quant_gather", "gemm", "SQLinear",
]

SQ_OK = 0
SQ_ERR_INVALID_ARG = 1
SQ_ERR_UNSUPPORTED = 2
SQ_ERR_MISALIGNED = 3
SQ_ERR_CUDA = 4
SQ_ERR_TIMEOUT = 5

HEADER = os.path.join(_build.ROOT, "include", "sq.h")


class SQError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        super().__init__(f"{where}: {_STATUS_NAMES.get(status, status)}: {detail}")


_STATUS_NAMES = {0: "SQ_OK", 1: "SQ_ERR_INVALID_ARG", 2: "SQ_ERR_UNSUPPORTED",
                 3: "SQ_ERR_MISALIGNED", 4: "SQ_ERR_CUDA", 5: "SQ_ERR_TIMEOUT"}

_lib = None


def library_path() -> str:
    return _build.LIB_PATH


def load():
    """Load libsq_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    path = _build.LIB_PATH
    if not os.path.exists(path):
        raise RuntimeError(
            f"CUDA library {path} is missing; build it with "
            "`python -m mixed_precision_gemm_b200._build` (or __graft_entry__.build())")
    lib = ctypes.CDLL(path)
    P, I, Z, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int
    lib.sq_status_string.argtypes = [F]
    lib.sq_status_string.restype = ctypes.c_char_p
    lib.sq_last_error_detail.argtypes = []
    lib.sq_last_error_detail.restype = ctypes.c_char_p
    lib.sq_kn_pad.argtypes = [I, I]
    lib.sq_kn_pad.restype = I
    lib.sq_no_pad.argtypes = [I]
    lib.sq_no_pad.restype = I
    lib.sq_chan_table_words.argtypes = [I]
    lib.sq_chan_table_words.restype = I
    lib.sq_linear_workspace_bytes.argtypes = [I, I, I]
    lib.sq_linear_workspace_bytes.restype = Z
    lib.sq_prepare_weights.argtypes = [P, I, I, I, P, I, P, P, P, P, P]
    lib.sq_quant_gather.argtypes = [P, I, I, I, P, I, P, P, P, P]
    lib.sq_gemm.argtypes = [P, P, P, P, P, P, I, I, I, I, P, I, P, P, P]
    lib.sq_linear.argtypes = [P, I, I, I, P, P, P, P, I, I, P, I, P, Z, P]
    lib.sq_linear_noalloc.argtypes = [P, I, I, I, P, P, P, P, I, I, P, I, P]
    lib.sq_check.argtypes = [P]
    lib.sq_selftest_watchdog.argtypes = [F, P]
    lib.sq_linear_workspace_bytes_fp8.argtypes = [I, I, I]
    lib.sq_linear_workspace_bytes_fp8.restype = Z
    lib.sq_prepare_weights_fp8.argtypes = [P, I, I, I, P, I, P, P, P, P, P]
    lib.sq_quant_gather_fp8.argtypes = [P, I, I, I, P, I, P, P, P, P]
    lib.sq_gemm_fp8.argtypes = [P, P, P, P, P, P, I, I, I, I, P, I, P, P, P]
    lib.sq_linear_fp8.argtypes = [P, I, I, I, P, P, P, P, I, I, P, I, P, Z, P]
    lib.sq_kn_pad_mx.argtypes = [I, I]
    lib.sq_kn_pad_mx.restype = I
    lib.sq_mx_scale_bytes.argtypes = [I, I, I]
    lib.sq_mx_scale_bytes.restype = Z
    lib.sq_linear_workspace_bytes_mx.argtypes = [I, I, I]
    lib.sq_linear_workspace_bytes_mx.restype = Z
    lib.sq_prepare_weights_mx.argtypes = [P, I, I, I, P, I, P, P, P, P, P]
    lib.sq_quant_gather_mx.argtypes = [P, I, I, I, P, I, P, P, P, P]
    lib.sq_gemm_mx.argtypes = [P, P, P, P, P, P, I, I, I, I, P, I, P, P]
    lib.sq_linear_mx.argtypes = [P, I, I, I, P, P, P, P, I, I, P, I, P, Z, P]
    C = ctypes.c_int
    lib.sq_linear_workspace_bytes_sqf.argtypes = [I, I, I]
    lib.sq_linear_workspace_bytes_sqf.restype = Z
    lib.sq_prepare_weights_sqf.argtypes = [P, I, I, I, C, C, P, P, P, P, P, P, P]
    lib.sq_quant_gather_sqf.argtypes = [P, I, I, I, P, P, P, P, P, P]
    lib.sq_gemm_sqf.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, P, I, P, P, P]
    lib.sq_linear_sqf.argtypes = [P, I, I, I, P, P, P, P, P, P, I, P, I, P, Z, P]
    lib.sq_select_outliers_workspace_bytes.argtypes = [I, I, I, I]
    lib.sq_select_outliers_workspace_bytes.restype = Z
    lib.sq_select_outliers.argtypes = [P, I, I, I, P, I, I, I, I, P, P, P, Z, P]
    for f in (lib.sq_prepare_weights, lib.sq_quant_gather, lib.sq_gemm, lib.sq_linear, lib.sq_check,
              lib.sq_selftest_watchdog, lib.sq_linear_noalloc, lib.sq_prepare_weights_fp8, lib.sq_quant_gather_fp8,
              lib.sq_gemm_fp8, lib.sq_linear_fp8, lib.sq_select_outliers, lib.sq_prepare_weights_mx,
              lib.sq_quant_gather_mx, lib.sq_gemm_mx, lib.sq_linear_mx, lib.sq_prepare_weights_sqf,
              lib.sq_quant_gather_sqf, lib.sq_gemm_sqf, lib.sq_linear_sqf):
        f.restype = F
    _lib = lib
    return lib


def header_functions() -> list[str]:
    """Names of the functions include/sq.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sq_[a-z0-9_]+)\s*\(", text)))


def _raise(st: int, where: str):
    if st != SQ_OK:
        detail = load().sq_last_error_detail().decode(errors="replace")
        raise SQError(st, where, detail)


def _ptr(t: Optional[torch.Tensor]):
    if t is None or t.numel() == 0:
        return None
    if not t.is_cuda:
        raise ValueError("device tensor expected")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _rowmajor(t: torch.Tensor, name: str, dtype=None):
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name}: expected a 2-D row-major tensor (unit inner stride)")
    return t


# ----------------------------------------------------------------- pure queries
def sq_status_string(st: int) -> str:
    return load().sq_status_string(st).decode()


def sq_kn_pad(K: int, nO: int) -> int:
    return int(load().sq_kn_pad(K, nO))


def sq_no_pad(nO: int) -> int:
    return int(load().sq_no_pad(nO))


def sq_chan_table_words(K: int) -> int:
    return int(load().sq_chan_table_words(K))


def sq_linear_workspace_bytes(M: int, K: int, nO: int) -> int:
    return int(load().sq_linear_workspace_bytes(M, K, nO))


# ----------------------------------------------------------------- ABI calls
def sq_prepare_weights(W: torch.Tensor, O, W_N: torch.Tensor, s_w: torch.Tensor, W_O: Optional[torch.Tensor],
                       chan_tab: torch.Tensor, stream=None) -> None:
    """Offline weight step: static channel table + both weight operands (waits for the stream)."""
    _rowmajor(W, "W", torch.bfloat16)
    N, K = W.shape
    O_host = torch.as_tensor(O, dtype=torch.int32).reshape(-1).contiguous().cpu()
    nO = O_host.numel()
    st = load().sq_prepare_weights(_ptr(W), N, K, W.stride(0),
                                   ctypes.c_void_p(O_host.data_ptr()) if nO else None, nO,
                                   _ptr(W_N), _ptr(s_w), _ptr(W_O), _ptr(chan_tab), _stream(stream))
    _raise(st, "sq_prepare_weights")


def sq_quant_gather(X: torch.Tensor, chan_tab: torch.Tensor, nO: int, X_N: Optional[torch.Tensor],
                    s_x: torch.Tensor, X_O: Optional[torch.Tensor], stream=None) -> None:
    _rowmajor(X, "X", torch.bfloat16)
    M, K = X.shape
    st = load().sq_quant_gather(_ptr(X), M, K, X.stride(0), _ptr(chan_tab), nO, _ptr(X_N), _ptr(s_x), _ptr(X_O),
                                _stream(stream))
    _raise(st, "sq_quant_gather")


def sq_gemm(X_N, s_x, X_O, W_N, s_w, W_O, M: int, N: int, K: int, nO: int, Y: torch.Tensor,
            dbg_acc_i32: Optional[torch.Tensor] = None, dbg_acc_f32: Optional[torch.Tensor] = None,
            stream=None) -> None:
    _rowmajor(Y, "Y", torch.bfloat16)
    st = load().sq_gemm(_ptr(X_N), _ptr(s_x), _ptr(X_O), _ptr(W_N), _ptr(s_w), _ptr(W_O), M, N, K, nO,
                        _ptr(Y), Y.stride(0), _ptr(dbg_acc_i32), _ptr(dbg_acc_f32), _stream(stream))
    _raise(st, "sq_gemm")


def sq_linear(X: torch.Tensor, chan_tab: torch.Tensor, W_N, s_w, W_O, N: int, nO: int, Y: torch.Tensor,
              workspace: torch.Tensor, stream=None) -> None:
    _rowmajor(X, "X", torch.bfloat16)
    _rowmajor(Y, "Y", torch.bfloat16)
    M, K = X.shape
    st = load().sq_linear(_ptr(X), M, K, X.stride(0), _ptr(chan_tab), _ptr(W_N), _ptr(s_w), _ptr(W_O), N, nO,
                          _ptr(Y), Y.stride(0), _ptr(workspace), workspace.numel() * workspace.element_size(),
                          _stream(stream))
    _raise(st, "sq_linear")


def sq_linear_noalloc(X: torch.Tensor, chan_tab: torch.Tensor, W_N, s_w, W_O, N: int, nO: int, Y: torch.Tensor,
                      stream=None) -> None:
    """sq_linear for callers that cannot allocate device memory for a workspace.

    The scratch lives in a fixed 16 MiB array inside the library (see
    SQ_NOALLOC_WS_BYTES in include/sq.h): calls that need more raise
    SQError(SQ_ERR_UNSUPPORTED), and calls that overlap on the GPU race on the
    shared array, so serialize them.
    """
    _rowmajor(X, "X", torch.bfloat16)
    _rowmajor(Y, "Y", torch.bfloat16)
    M, K = X.shape
    st = load().sq_linear_noalloc(_ptr(X), M, K, X.stride(0), _ptr(chan_tab), _ptr(W_N), _ptr(s_w), _ptr(W_O), N, nO,
                                  _ptr(Y), Y.stride(0), _stream(stream))
    _raise(st, "sq_linear_noalloc")


# FP8 low path (OSC: FP8 fallback for the inputs of W2): the same calls with
# one E4M3 byte per normal channel (u8 [rows, kn_pad]) instead of packed INT4.
def sq_linear_workspace_bytes_fp8(M: int, K: int, nO: int) -> int:
    return int(load().sq_linear_workspace_bytes_fp8(M, K, nO))


def sq_prepare_weights_fp8(W: torch.Tensor, O, W_N8: torch.Tensor, s_w: torch.Tensor, W_O: Optional[torch.Tensor],
                           chan_tab: torch.Tensor, stream=None) -> None:
    _rowmajor(W, "W", torch.bfloat16)
    N, K = W.shape
    O_host = torch.as_tensor(O, dtype=torch.int32).reshape(-1).contiguous().cpu()
    nO = O_host.numel()
    st = load().sq_prepare_weights_fp8(_ptr(W), N, K, W.stride(0),
                                       ctypes.c_void_p(O_host.data_ptr()) if nO else None, nO,
                                       _ptr(W_N8), _ptr(s_w), _ptr(W_O), _ptr(chan_tab), _stream(stream))
    _raise(st, "sq_prepare_weights_fp8")


def sq_quant_gather_fp8(X: torch.Tensor, chan_tab: torch.Tensor, nO: int, X_N8: Optional[torch.Tensor],
                        s_x: torch.Tensor, X_O: Optional[torch.Tensor], stream=None) -> None:
    _rowmajor(X, "X", torch.bfloat16)
    M, K = X.shape
    st = load().sq_quant_gather_fp8(_ptr(X), M, K, X.stride(0), _ptr(chan_tab), nO, _ptr(X_N8), _ptr(s_x),
                                    _ptr(X_O), _stream(stream))
    _raise(st, "sq_quant_gather_fp8")


def sq_gemm_fp8(X_N8, s_x, X_O, W_N8, s_w, W_O, M: int, N: int, K: int, nO: int, Y: torch.Tensor,
                dbg_acc_8: Optional[torch.Tensor] = None, dbg_acc_f32: Optional[torch.Tensor] = None,
                stream=None) -> None:
    _rowmajor(Y, "Y", torch.bfloat16)
    st = load().sq_gemm_fp8(_ptr(X_N8), _ptr(s_x), _ptr(X_O), _ptr(W_N8), _ptr(s_w), _ptr(W_O), M, N, K, nO,
                            _ptr(Y), Y.stride(0), _ptr(dbg_acc_8), _ptr(dbg_acc_f32), _stream(stream))
    _raise(st, "sq_gemm_fp8")


def sq_linear_fp8(X: torch.Tensor, chan_tab: torch.Tensor, W_N8, s_w, W_O, N: int, nO: int, Y: torch.Tensor,
                  workspace: torch.Tensor, stream=None) -> None:
    _rowmajor(X, "X", torch.bfloat16)
    _rowmajor(Y, "Y", torch.bfloat16)
    M, K = X.shape
    st = load().sq_linear_fp8(_ptr(X), M, K, X.stride(0), _ptr(chan_tab), _ptr(W_N8), _ptr(s_w), _ptr(W_O), N, nO,
                              _ptr(Y), Y.stride(0), _ptr(workspace), workspace.numel() * workspace.element_size(),
                              _stream(stream))
    _raise(st, "sq_linear_fp8")


# MXFP4 low path (OSC abstract: 4-bit micro-scaling hardware): packed E2M1
# codes (u8 [rows, kn_pad_mx / 2]) with tiled E8M0 block scales (u8
# [sq_mx_scale_bytes(rows, K, nO)]) in place of the fp32 row scales.
def sq_kn_pad_mx(K: int, nO: int) -> int:
    return int(load().sq_kn_pad_mx(K, nO))


def sq_mx_scale_bytes(rows: int, K: int, nO: int) -> int:
    return int(load().sq_mx_scale_bytes(rows, K, nO))


def sq_linear_workspace_bytes_mx(M: int, K: int, nO: int) -> int:
    return int(load().sq_linear_workspace_bytes_mx(M, K, nO))


def sq_prepare_weights_mx(W: torch.Tensor, O, W_N4: torch.Tensor, S_W: torch.Tensor, W_O: Optional[torch.Tensor],
                          chan_tab: torch.Tensor, stream=None) -> None:
    _rowmajor(W, "W", torch.bfloat16)
    N, K = W.shape
    O_host = torch.as_tensor(O, dtype=torch.int32).reshape(-1).contiguous().cpu()
    nO = O_host.numel()
    st = load().sq_prepare_weights_mx(_ptr(W), N, K, W.stride(0),
                                      ctypes.c_void_p(O_host.data_ptr()) if nO else None, nO,
                                      _ptr(W_N4), _ptr(S_W), _ptr(W_O), _ptr(chan_tab), _stream(stream))
    _raise(st, "sq_prepare_weights_mx")


def sq_quant_gather_mx(X: torch.Tensor, chan_tab: torch.Tensor, nO: int, X_N4: Optional[torch.Tensor],
                       S_X: Optional[torch.Tensor], X_O: Optional[torch.Tensor], stream=None) -> None:
    _rowmajor(X, "X", torch.bfloat16)
    M, K = X.shape
    st = load().sq_quant_gather_mx(_ptr(X), M, K, X.stride(0), _ptr(chan_tab), nO, _ptr(X_N4), _ptr(S_X),
                                   _ptr(X_O), _stream(stream))
    _raise(st, "sq_quant_gather_mx")


def sq_gemm_mx(X_N4, S_X, X_O, W_N4, S_W, W_O, M: int, N: int, K: int, nO: int, Y: torch.Tensor,
               dbg_acc: Optional[torch.Tensor] = None, stream=None) -> None:
    _rowmajor(Y, "Y", torch.bfloat16)
    st = load().sq_gemm_mx(_ptr(X_N4), _ptr(S_X), _ptr(X_O), _ptr(W_N4), _ptr(S_W), _ptr(W_O), M, N, K, nO,
                           _ptr(Y), Y.stride(0), _ptr(dbg_acc), _stream(stream))
    _raise(st, "sq_gemm_mx")


def sq_linear_mx(X: torch.Tensor, chan_tab: torch.Tensor, W_N4, S_W, W_O, N: int, nO: int, Y: torch.Tensor,
                 workspace: torch.Tensor, stream=None) -> None:
    _rowmajor(X, "X", torch.bfloat16)
    _rowmajor(Y, "Y", torch.bfloat16)
    M, K = X.shape
    st = load().sq_linear_mx(_ptr(X), M, K, X.stride(0), _ptr(chan_tab), _ptr(W_N4), _ptr(S_W), _ptr(W_O), N, nO,
                             _ptr(Y), Y.stride(0), _ptr(workspace), workspace.numel() * workspace.element_size(),
                             _stream(stream))
    _raise(st, "sq_linear_mx")


# Element-level SQ-format weights (SQ-format write-up sections 3, 7, 8, 9): banks
# of 4/8/16 channels with 1 or 2 E4M3 high entries (2:4 sparse tensor cores) and
# an INT4 low part carrying the mask code -8.
def sq_linear_workspace_bytes_sqf(M: int, N: int, K: int) -> int:
    return int(load().sq_linear_workspace_bytes_sqf(M, N, K))


def sq_prepare_weights_sqf(W: torch.Tensor, bank: int, h: int, W_N, s_lo, W_H, W_E, s_hi, chan_tab,
                           stream=None) -> None:
    _rowmajor(W, "W", torch.bfloat16)
    N, K = W.shape
    st = load().sq_prepare_weights_sqf(_ptr(W), N, K, W.stride(0), bank, h, _ptr(W_N), _ptr(s_lo), _ptr(W_H),
                                       _ptr(W_E), _ptr(s_hi), _ptr(chan_tab), _stream(stream))
    _raise(st, "sq_prepare_weights_sqf")


def sq_quant_gather_sqf(X: torch.Tensor, chan_tab, X_N, s_x4, X_8, s_x8, stream=None) -> None:
    _rowmajor(X, "X", torch.bfloat16)
    M, K = X.shape
    st = load().sq_quant_gather_sqf(_ptr(X), M, K, X.stride(0), _ptr(chan_tab), _ptr(X_N), _ptr(s_x4), _ptr(X_8),
                                    _ptr(s_x8), _stream(stream))
    _raise(st, "sq_quant_gather_sqf")


def sq_gemm_sqf(X_N, s_x4, X_8, s_x8, W_N, s_lo, W_H, W_E, s_hi, M: int, N: int, K: int, Y: torch.Tensor,
                P: torch.Tensor, dbg_acc_lo: Optional[torch.Tensor] = None, stream=None) -> None:
    _rowmajor(Y, "Y", torch.bfloat16)
    st = load().sq_gemm_sqf(_ptr(X_N), _ptr(s_x4), _ptr(X_8), _ptr(s_x8), _ptr(W_N), _ptr(s_lo), _ptr(W_H),
                            _ptr(W_E), _ptr(s_hi), M, N, K, _ptr(Y), Y.stride(0), _ptr(P), _ptr(dbg_acc_lo),
                            _stream(stream))
    _raise(st, "sq_gemm_sqf")


def sq_linear_sqf(X: torch.Tensor, chan_tab, W_N, s_lo, W_H, W_E, s_hi, N: int, Y: torch.Tensor,
                  workspace: torch.Tensor, stream=None) -> None:
    _rowmajor(X, "X", torch.bfloat16)
    _rowmajor(Y, "Y", torch.bfloat16)
    M, K = X.shape
    st = load().sq_linear_sqf(_ptr(X), M, K, X.stride(0), _ptr(chan_tab), _ptr(W_N), _ptr(s_lo), _ptr(W_H),
                              _ptr(W_E), _ptr(s_hi), N, _ptr(Y), Y.stride(0), _ptr(workspace),
                              workspace.numel() * workspace.element_size(), _stream(stream))
    _raise(st, "sq_linear_sqf")


# Static outlier-channel selection (the offline step that chooses O).
def sq_select_outliers_workspace_bytes(Mc: int, N: int, K: int, group: int = 1) -> int:
    return int(load().sq_select_outliers_workspace_bytes(Mc, N, K, group))


def sq_select_outliers(Xc: torch.Tensor, W: torch.Tensor, nO: int, group: int, O: Optional[torch.Tensor],
                       scores: Optional[torch.Tensor], workspace: torch.Tensor, stream=None) -> None:
    _rowmajor(Xc, "Xc", torch.bfloat16)
    _rowmajor(W, "W", torch.bfloat16)
    Mc, K = Xc.shape
    N = W.shape[0]
    if W.shape[1] != K:
        raise ValueError("Xc and W disagree on K")
    st = load().sq_select_outliers(_ptr(Xc), Mc, K, Xc.stride(0), _ptr(W), N, W.stride(0), nO, group, _ptr(O),
                                   _ptr(scores), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                   _stream(stream))
    _raise(st, "sq_select_outliers")


def sq_check(stream=None) -> None:
    _raise(load().sq_check(_stream(stream)), "sq_check")


def sq_selftest_watchdog(timeout_ms: int, stream=None) -> None:
    _raise(load().sq_selftest_watchdog(timeout_ms, _stream(stream)), "sq_selftest_watchdog")


# ----------------------------------------------------------------- conveniences
@dataclasses.dataclass
class PreparedWeights:
    """Offline artefacts of one layer: the static channel table and both weight operands."""
    N: int
    K: int
    nO: int
    W_N: torch.Tensor        # uint8 [N, kn_pad/2] packed INT4, [N, kn_pad] E4M3 (fp8), [N, kn_pad_mx/2] E2M1 (mx)
    s_w: torch.Tensor        # float32 [N]; mx: uint8 [sq_mx_scale_bytes(N, K, nO)] tiled E8M0 block scales
    W_O: torch.Tensor        # bf16 [N, no_pad]
    chan_tab: torch.Tensor   # int32 view of uint32 [K/8]
    fp8: bool = False        # low path in FP8 E4M3 (the W2 fallback) instead of INT4
    mx: bool = False         # low path in MXFP4 (E2M1 + E8M0 block scales) instead of INT4

    def state_dict(self) -> dict:
        return {"N": self.N, "K": self.K, "nO": self.nO, "W_N": self.W_N, "s_w": self.s_w,
                "W_O": self.W_O, "chan_tab": self.chan_tab, "fp8": self.fp8, "mx": self.mx}

    @classmethod
    def from_state_dict(cls, d: dict, device=None) -> "PreparedWeights":
        mv = (lambda t: t.to(device)) if device is not None else (lambda t: t)
        return cls(int(d["N"]), int(d["K"]), int(d["nO"]), mv(d["W_N"]), mv(d["s_w"]), mv(d["W_O"]),
                   mv(d["chan_tab"]), bool(d.get("fp8", False)), bool(d.get("mx", False)))

    def code_bytes(self, K: int) -> int:
        if self.mx:
            return sq_kn_pad_mx(K, self.nO) // 2
        kn = sq_kn_pad(K, self.nO)
        return kn if self.fp8 else kn // 2


def prepare_weights(W: torch.Tensor, O: Sequence[int], stream=None, fp8: bool = False,
                    mx: bool = False) -> PreparedWeights:
    """Offline weight step; fp8=True prepares the FP8 (E4M3) low path, mx=True
    the MXFP4 one, instead of INT4."""
    if fp8 and mx:
        raise ValueError("choose one low path")
    N, K = W.shape
    nO = len(torch.as_tensor(O).reshape(-1))
    dev = W.device
    W_O = torch.zeros(N, sq_no_pad(nO), dtype=torch.bfloat16, device=dev)
    tab = torch.zeros(sq_chan_table_words(K), dtype=torch.int32, device=dev)
    if mx:
        W_N = torch.zeros(N, sq_kn_pad_mx(K, nO) // 2, dtype=torch.uint8, device=dev)
        S_W = torch.zeros(max(sq_mx_scale_bytes(N, K, nO), 16), dtype=torch.uint8, device=dev)
        sq_prepare_weights_mx(W, O, W_N, S_W, W_O, tab, stream)
        return PreparedWeights(N, K, nO, W_N, S_W, W_O, tab, False, True)
    kn = sq_kn_pad(K, nO)
    W_N = torch.zeros(N, kn if fp8 else kn // 2, dtype=torch.uint8, device=dev)
    s_w = torch.zeros(N, dtype=torch.float32, device=dev)
    (sq_prepare_weights_fp8 if fp8 else sq_prepare_weights)(W, O, W_N, s_w, W_O, tab, stream)
    return PreparedWeights(N, K, nO, W_N, s_w, W_O, tab, fp8)


def quant_gather(X: torch.Tensor, pw: PreparedWeights, stream=None):
    """Online step: (X_N, s_x, X_O).  For the MX path s_x is the tiled E8M0
    block-scale buffer (uint8)."""
    M, K = X.shape
    dev = X.device
    X_N = torch.empty(M, pw.code_bytes(K), dtype=torch.uint8, device=dev)
    X_O = torch.empty(M, sq_no_pad(pw.nO), dtype=torch.bfloat16, device=dev)
    if pw.mx:
        S_X = torch.empty(max(sq_mx_scale_bytes(M, K, pw.nO), 16), dtype=torch.uint8, device=dev)
        sq_quant_gather_mx(X, pw.chan_tab, pw.nO, X_N, S_X, X_O, stream)
        return X_N, S_X, X_O
    s_x = torch.empty(M, dtype=torch.float32, device=dev)
    (sq_quant_gather_fp8 if pw.fp8 else sq_quant_gather)(X, pw.chan_tab, pw.nO, X_N, s_x, X_O, stream)
    return X_N, s_x, X_O


def gemm(X_N, s_x, X_O, pw: PreparedWeights, Y: Optional[torch.Tensor] = None, debug: bool = False, stream=None):
    """Dual GEMM.  With debug=True also returns the two accumulators: the low
    path's (int32 for INT4, fp32 for FP8) and the bf16 branch's (fp32).  For
    the MX path the two share one fp32 accumulator, returned as (Y, None, acc)."""
    M = X_N.shape[0]
    if Y is None:
        Y = torch.empty(M, pw.N, dtype=torch.bfloat16, device=X_N.device)
    if pw.mx:
        acc = torch.empty(M, pw.N, dtype=torch.float32, device=X_N.device) if debug else None
        sq_gemm_mx(X_N, s_x, X_O, pw.W_N, pw.s_w, pw.W_O, M, pw.N, pw.K, pw.nO, Y, acc, stream)
        return (Y, None, acc) if debug else Y
    dbg_i = dbg_f = None
    if debug:
        dbg_i = torch.empty(M, pw.N, dtype=torch.float32 if pw.fp8 else torch.int32, device=s_x.device)
        dbg_f = torch.empty(M, pw.N, dtype=torch.float32, device=s_x.device)
    (sq_gemm_fp8 if pw.fp8 else sq_gemm)(X_N, s_x, X_O, pw.W_N, pw.s_w, pw.W_O, M, pw.N, pw.K, pw.nO, Y, dbg_i, dbg_f,
                                         stream)
    return (Y, dbg_i, dbg_f) if debug else Y


def select_outliers(Xc: torch.Tensor, W: torch.Tensor, nO: int, group: int = 1, stream=None):
    """Static outlier channels from calibration activations Xc [Mc, K] and weights W [N, K]
    (bf16, on the GPU): returns (O int32 [nO] ascending, scores float64 [K]), both on the device."""
    dev = W.device
    K = W.shape[1]
    O = torch.zeros(nO, dtype=torch.int32, device=dev)
    scores = torch.zeros(K, dtype=torch.float64, device=dev)
    ws = torch.empty(max(256, sq_select_outliers_workspace_bytes(Xc.shape[0], W.shape[0], K, group)),
                     dtype=torch.uint8, device=dev)
    sq_select_outliers(Xc, W, nO, group, O, scores, ws, stream)
    return O, scores


class SQLinear:
    """A prepared dual-path linear layer: ``y = layer(x)`` for bf16 x [M, K] on the GPU.

    fp8=True runs the low path in FP8 E4M3 (OSC's fallback for the inputs of W2);
    mx=True runs it in MXFP4 (E2M1 codes, E8M0 scales per 32 channels)."""

    def __init__(self, W: torch.Tensor, O: Sequence[int], stream=None, fp8: bool = False, mx: bool = False):
        self.weights = prepare_weights(W, O, stream, fp8, mx)
        self._ws = None

    def workspace(self, M: int, device) -> torch.Tensor:
        pw = self.weights
        ws_fn = (sq_linear_workspace_bytes_mx if pw.mx else
                 sq_linear_workspace_bytes_fp8 if pw.fp8 else sq_linear_workspace_bytes)
        need = ws_fn(M, self.weights.K, self.weights.nO)
        if self._ws is None or self._ws.numel() < need or self._ws.device != torch.device(device):
            self._ws = torch.empty(max(need, 256), dtype=torch.uint8, device=device)
        return self._ws

    def __call__(self, X: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        pw = self.weights
        M = X.shape[0]
        if out is None:
            out = torch.empty(M, pw.N, dtype=torch.bfloat16, device=X.device)
        fn = sq_linear_mx if pw.mx else sq_linear_fp8 if pw.fp8 else sq_linear
        fn(X, pw.chan_tab, pw.W_N, pw.s_w, pw.W_O, pw.N, pw.nO, out, self.workspace(M, X.device), stream)
        return out


@dataclasses.dataclass
class PreparedSQF:
    """Element-level SQ-format weights of one layer (see sq_prepare_weights_sqf)."""
    N: int
    K: int
    bank: int
    h: int
    W_N: torch.Tensor       # uint8 [N, K/2] packed INT4, mask code -8 at high positions
    s_lo: torch.Tensor      # float32 [N]
    W_H: torch.Tensor       # uint8 [N, K/2] 2:4-compressed E4M3 high entries
    W_E: torch.Tensor       # uint8 [N, K/8] 2:4 metadata
    s_hi: torch.Tensor      # float32 [N]
    chan_tab: torch.Tensor  # int32 [K/8], all zero (no outlier channels)


def prepare_weights_sqf(W: torch.Tensor, bank: int, h: int, stream=None) -> PreparedSQF:
    N, K = W.shape
    dev = W.device
    u8 = dict(dtype=torch.uint8, device=dev)
    pw = PreparedSQF(N, K, bank, h, torch.zeros(N, K // 2, **u8), torch.zeros(N, dtype=torch.float32, device=dev),
                     torch.zeros(N, K // 2, **u8), torch.zeros(N, K // 8, **u8),
                     torch.zeros(N, dtype=torch.float32, device=dev),
                     torch.zeros(K // 8, dtype=torch.int32, device=dev))
    sq_prepare_weights_sqf(W, bank, h, pw.W_N, pw.s_lo, pw.W_H, pw.W_E, pw.s_hi, pw.chan_tab, stream)
    return pw


def quant_gather_sqf(X: torch.Tensor, pw: PreparedSQF, stream=None):
    """(X_N int4 [M, K/2], s_x4 [M], X_8 e4m3 [M, K], s_x8 [M])."""
    M, K = X.shape
    dev = X.device
    X_N = torch.empty(M, K // 2, dtype=torch.uint8, device=dev)
    X_8 = torch.empty(M, K, dtype=torch.uint8, device=dev)
    s_x4 = torch.empty(M, dtype=torch.float32, device=dev)
    s_x8 = torch.empty(M, dtype=torch.float32, device=dev)
    sq_quant_gather_sqf(X, pw.chan_tab, X_N, s_x4, X_8, s_x8, stream)
    return X_N, s_x4, X_8, s_x8


def gemm_sqf(X_N, s_x4, X_8, s_x8, pw: PreparedSQF, Y: Optional[torch.Tensor] = None, debug: bool = False,
             stream=None):
    """Y (bf16).  With debug=True returns (Y, acc_lo int32, P fp32 high part)."""
    M = X_N.shape[0]
    dev = X_N.device
    if Y is None:
        Y = torch.empty(M, pw.N, dtype=torch.bfloat16, device=dev)
    P = torch.empty(M, pw.N, dtype=torch.float32, device=dev)
    acc = torch.empty(M, pw.N, dtype=torch.int32, device=dev) if debug else None
    sq_gemm_sqf(X_N, s_x4, X_8, s_x8, pw.W_N, pw.s_lo, pw.W_H, pw.W_E, pw.s_hi, M, pw.N, pw.K, Y, P, acc, stream)
    return (Y, acc, P) if debug else Y
