"""CPU oracle for the dual-path sparse-quantized linear layer.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers.  The product library never
imports this package and this package never imports the product library.

The arithmetic lives in ``sq_oracle.c`` (plain C, fp32 quantizer decisions,
int64 integer path, fp64 16-bit branch and output).  This module compiles it
with gcc on first use and wraps it with numpy arrays.  The method it follows
is described in the C file's header: the OSC page (arXiv:2604.12782, abstract
and technical framework: static outlier channels, compact gather, 4-bit GEMM
plus 16-bit branch GEMM, fused sum) and the SQ-format write-up of
arXiv:2512.05409 (section 9: symmetric quantization, column reordering by the
static mask).  The FP8 functions follow the same page's FP8 fallback for the
inputs of W2 (E4M3 low path, scale = absolute maximum / 448; readings in the C
file).  The MX functions follow the OSC abstract's fit with 4-bit
micro-scaling hardware (and the SQ-format write-up, section 8, FP4 variant):
the normal channels in MXFP4, blocks of 32 with an E8M0 scale each (readings
in the C file).  The SQF functions follow the SQ-format write-up's element-level
format for weights (banks with a fixed number of high-precision entries chosen
by magnitude, INT4 low part with the mask code -8, E4M3 high part; readings in
the C file).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle_sq.so")
_CFLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-std=c11"]
_lock = threading.Lock()
_lib = None

QMAX = 7  # symmetric INT4 code range [-7, 7]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (if missing or older than its source)."""
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *_CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            P = ctypes.c_void_p
            I = ctypes.c_int64
            lib.orc_validate_outliers.argtypes = [P, I, I]
            lib.orc_quantize_rows.argtypes = [P, I, I, I, P, I, P, P, P]
            lib.orc_pack_int4.argtypes = [P, I, I, I, P]
            lib.orc_chan_table.argtypes = [P, I, I, P]
            lib.orc_dual_linear_rows.argtypes = [P, P, P, I, P, P, P, I, I, I, P, P, P]
            lib.orc_num_threads.argtypes = []
            lib.orc_e4m3_encode_array.argtypes = [P, I, P]
            lib.orc_e4m3_decode_array.argtypes = [P, I, P]
            lib.orc_quantize_rows_fp8.argtypes = [P, I, I, I, P, I, P, P, P]
            lib.orc_dual_linear_rows_fp8.argtypes = [P, P, P, I, P, P, P, I, I, I, P, P, P]
            lib.orc_select_outliers.argtypes = [P, I, I, I, P, I, I, I, I, P, P]
            lib.orc_e2m1_encode_array.argtypes = [P, I, P]
            lib.orc_e2m1_decode.argtypes = [ctypes.c_uint8]
            lib.orc_e2m1_decode.restype = ctypes.c_double
            lib.orc_mx_block_exponent.argtypes = [ctypes.c_double]
            lib.orc_quantize_rows_mx.argtypes = [P, I, I, I, P, I, P, P, P]
            lib.orc_dual_linear_rows_mx.argtypes = [P, P, P, I, P, P, P, I, I, I, P, P, P]
            C = ctypes.c_int
            lib.orc_sqf_weights.argtypes = [P, I, I, I, C, C, P, P, P, P, P]
            lib.orc_sqf_linear_rows.argtypes = [P, P, P, P, I, P, P, P, P, P, I, I, P, P, P]
            for f in (lib.orc_e2m1_encode_array, lib.orc_mx_block_exponent, lib.orc_quantize_rows_mx,
                      lib.orc_dual_linear_rows_mx, lib.orc_sqf_weights, lib.orc_sqf_linear_rows):
                f.restype = ctypes.c_int
            for f in (lib.orc_validate_outliers, lib.orc_quantize_rows, lib.orc_pack_int4,
                      lib.orc_chan_table, lib.orc_dual_linear_rows, lib.orc_num_threads,
                      lib.orc_e4m3_encode_array, lib.orc_e4m3_decode_array, lib.orc_quantize_rows_fp8,
                      lib.orc_dual_linear_rows_fp8, lib.orc_select_outliers):
                f.restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def _as_O(O) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(O, dtype=np.int32).reshape(-1))


def num_threads() -> int:
    """Host threads the oracle's row loops use (OMP_NUM_THREADS, else all cores)."""
    return int(_load().orc_num_threads())


def validate_outliers(O, K: int) -> bool:
    O = _as_O(O)
    return _load().orc_validate_outliers(_ptr(O), O.size, K) == 0


def quantize_rows(src_bits: np.ndarray, K: int, O):
    """Quantize-and-gather rows of a bf16 matrix given as uint16 bit patterns.

    Returns (codes int8 [rows, K-nO], scale float32 [rows], outl uint16 [rows, nO]).
    """
    src = np.ascontiguousarray(src_bits, dtype=np.uint16)
    if src.ndim != 2 or src.shape[1] < K:
        raise ValueError("src must be [rows, ld>=K]")
    O = _as_O(O)
    rows, ld = src.shape
    KN = K - O.size
    codes = np.zeros((rows, KN), np.int8)
    scale = np.zeros(rows, np.float32)
    outl = np.zeros((rows, O.size), np.uint16)
    rc = _load().orc_quantize_rows(_ptr(src), rows, K, ld, _ptr(O), O.size,
                                   _ptr(codes), _ptr(scale), _ptr(outl))
    if rc != 0:
        raise ValueError("invalid outlier channel set")
    return codes, scale, outl


def pack_int4(codes: np.ndarray, row_bytes: int) -> np.ndarray:
    """Packed storage of int4 codes: byte j = code 2j (low nibble) | code 2j+1 (high nibble)."""
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    rows, KN = codes.shape
    out = np.zeros((rows, row_bytes), np.uint8)
    if _load().orc_pack_int4(_ptr(codes), rows, KN, row_bytes, _ptr(out)) != 0:
        raise ValueError("row_bytes too small")
    return out


def chan_table(O, K: int) -> np.ndarray:
    """Static channel table: word c = (#outliers below 8c) << 8 | outlier bits of 8c..8c+7."""
    O = _as_O(O)
    tab = np.zeros(K // 8, np.uint32)
    if _load().orc_chan_table(_ptr(O), O.size, K, _ptr(tab)) != 0:
        raise ValueError("invalid outlier channel set or K % 8 != 0")
    return tab


def dual_linear_rows(qx, sx, xo, qw, sw, wo):
    """(acc_i int64, acc_o float64, y float64), each [rows of qx, rows of qw]."""
    qx = np.ascontiguousarray(qx, np.int8)
    qw = np.ascontiguousarray(qw, np.int8)
    sx = np.ascontiguousarray(sx, np.float32)
    sw = np.ascontiguousarray(sw, np.float32)
    xo = np.ascontiguousarray(xo, np.uint16)
    wo = np.ascontiguousarray(wo, np.uint16)
    Mr, KN = qx.shape
    N = qw.shape[0]
    nO = xo.shape[1]
    assert qw.shape[1] == KN and wo.shape == (N, nO) and xo.shape[0] == Mr
    acc_i = np.zeros((Mr, N), np.int64)
    acc_o = np.zeros((Mr, N), np.float64)
    y = np.zeros((Mr, N), np.float64)
    _load().orc_dual_linear_rows(_ptr(qx), _ptr(sx), _ptr(xo), Mr, _ptr(qw), _ptr(sw), _ptr(wo),
                                 N, KN, nO, _ptr(acc_i), _ptr(acc_o), _ptr(y))
    return acc_i, acc_o, y


def linear(X_bits: np.ndarray, W_bits: np.ndarray, O, rows=None):
    """Whole layer for the selected activation rows (all rows when None).

    Returns a dict with the quantizer outputs of both operands and the
    products: qx, sx, xo, qw, sw, wo, acc_i, acc_o, y.
    """
    K = W_bits.shape[1]
    Xs = X_bits if rows is None else X_bits[np.asarray(rows)]
    qx, sx, xo = quantize_rows(Xs, K, O)
    qw, sw, wo = quantize_rows(W_bits, K, O)
    acc_i, acc_o, y = dual_linear_rows(qx, sx, xo, qw, sw, wo)
    return dict(qx=qx, sx=sx, xo=xo, qw=qw, sw=sw, wo=wo, acc_i=acc_i, acc_o=acc_o, y=y)


# ---------------------------------------------------------------- FP8 low path
E4M3_MAX = 448.0  # largest finite E4M3 value


def e4m3_encode(t) -> np.ndarray:
    """E4M3 codes (uint8) nearest to float32 values, ties to even, saturating at 448."""
    t = np.ascontiguousarray(t, np.float32).reshape(-1)
    out = np.zeros(t.size, np.uint8)
    _load().orc_e4m3_encode_array(_ptr(t), t.size, _ptr(out))
    return out


def e4m3_decode(codes) -> np.ndarray:
    """float64 values of E4M3 codes."""
    c = np.ascontiguousarray(codes, np.uint8).reshape(-1)
    out = np.zeros(c.size, np.float64)
    _load().orc_e4m3_decode_array(_ptr(c), c.size, _ptr(out))
    return out


def quantize_rows_fp8(src_bits: np.ndarray, K: int, O):
    """FP8 quantize-and-gather: (codes uint8 E4M3 [rows, K-nO], scale float32 [rows], outl uint16 [rows, nO])."""
    src = np.ascontiguousarray(src_bits, dtype=np.uint16)
    if src.ndim != 2 or src.shape[1] < K:
        raise ValueError("src must be [rows, ld>=K]")
    O = _as_O(O)
    rows, ld = src.shape
    KN = K - O.size
    codes = np.zeros((rows, KN), np.uint8)
    scale = np.zeros(rows, np.float32)
    outl = np.zeros((rows, O.size), np.uint16)
    rc = _load().orc_quantize_rows_fp8(_ptr(src), rows, K, ld, _ptr(O), O.size,
                                       _ptr(codes), _ptr(scale), _ptr(outl))
    if rc != 0:
        raise ValueError("invalid outlier channel set")
    return codes, scale, outl


def dual_linear_rows_fp8(qx, sx, xo, qw, sw, wo):
    """(acc_8 float64, acc_o float64, y float64), each [rows of qx, rows of qw]."""
    qx = np.ascontiguousarray(qx, np.uint8)
    qw = np.ascontiguousarray(qw, np.uint8)
    sx = np.ascontiguousarray(sx, np.float32)
    sw = np.ascontiguousarray(sw, np.float32)
    xo = np.ascontiguousarray(xo, np.uint16)
    wo = np.ascontiguousarray(wo, np.uint16)
    Mr, KN = qx.shape
    N = qw.shape[0]
    nO = xo.shape[1]
    assert qw.shape[1] == KN and wo.shape == (N, nO) and xo.shape[0] == Mr
    acc_8 = np.zeros((Mr, N), np.float64)
    acc_o = np.zeros((Mr, N), np.float64)
    y = np.zeros((Mr, N), np.float64)
    _load().orc_dual_linear_rows_fp8(_ptr(qx), _ptr(sx), _ptr(xo), Mr, _ptr(qw), _ptr(sw), _ptr(wo),
                                     N, KN, nO, _ptr(acc_8), _ptr(acc_o), _ptr(y))
    return acc_8, acc_o, y


def linear_fp8(X_bits: np.ndarray, W_bits: np.ndarray, O, rows=None):
    """Whole layer with the FP8 low path for the selected activation rows (all when None)."""
    K = W_bits.shape[1]
    Xs = X_bits if rows is None else X_bits[np.asarray(rows)]
    qx, sx, xo = quantize_rows_fp8(Xs, K, O)
    qw, sw, wo = quantize_rows_fp8(W_bits, K, O)
    acc_8, acc_o, y = dual_linear_rows_fp8(qx, sx, xo, qw, sw, wo)
    return dict(qx=qx, sx=sx, xo=xo, qw=qw, sw=sw, wo=wo, acc_8=acc_8, acc_o=acc_o, y=y)


# ---------------------------------------------------------------- static outlier selection
def select_outliers(X_bits: np.ndarray, W_bits: np.ndarray, nO: int, group: int = 1):
    """Static outlier channels from calibration activations and the weights.

    score[k] = mean_m |X[m,k]| * ||W[:,k]||_2 (fp64, each column summed in row
    order); the nO/group groups of `group` consecutive channels with
    the largest summed score (ties to the lower index).  Returns (O int32
    ascending, score float64 [K]).
    """
    X = np.ascontiguousarray(X_bits, np.uint16)
    W = np.ascontiguousarray(W_bits, np.uint16)
    Mc, K = X.shape
    N, K2 = W.shape
    if K2 != K:
        raise ValueError("X and W disagree on K")
    O = np.zeros(nO, np.int32)
    score = np.zeros(K, np.float64)
    rc = _load().orc_select_outliers(_ptr(X), Mc, K, K, _ptr(W), N, K, nO, group, _ptr(O), _ptr(score))
    if rc != 0:
        raise ValueError("invalid sizes (group must divide K and nO)")
    return O, score


# ---------------------------------------------------------------- micro-scaling FP4 (MXFP4) low path
MX_BLOCK = 32      # entries per block scale
E2M1_MAX = 6.0     # largest E2M1 magnitude


def e2m1_encode(t) -> np.ndarray:
    """E2M1 codes (uint8, sign bit 3) nearest to float64 values, ties to even, saturating at 6."""
    t = np.ascontiguousarray(t, np.float64).reshape(-1)
    out = np.zeros(t.size, np.uint8)
    _load().orc_e2m1_encode_array(_ptr(t), t.size, _ptr(out))
    return out


def e2m1_decode(codes) -> np.ndarray:
    """float64 values of E2M1 codes (low 4 bits of each byte)."""
    c = np.asarray(codes, np.uint8).reshape(-1)
    lib = _load()
    table = np.array([lib.orc_e2m1_decode(i) for i in range(16)], np.float64)
    return table[c & 15]


def mx_block_exponent(a: float) -> int:
    """E of the block scale 2^E for a block with absolute maximum a (before the +127 bias)."""
    return int(_load().orc_mx_block_exponent(float(a)))


def quantize_rows_mx(src_bits: np.ndarray, K: int, O):
    """MXFP4 quantize-and-gather of bf16 rows (uint16 bit patterns).

    Returns (codes uint8 E2M1 [rows, K-nO] (one per byte), e8 uint8 [rows,
    ceil((K-nO)/32)] E8M0 block scales, outl uint16 [rows, nO]).
    """
    src = np.ascontiguousarray(src_bits, dtype=np.uint16)
    if src.ndim != 2 or src.shape[1] < K:
        raise ValueError("src must be [rows, ld>=K]")
    O = _as_O(O)
    rows, ld = src.shape
    KN = K - O.size
    NB = (KN + MX_BLOCK - 1) // MX_BLOCK
    codes = np.zeros((rows, KN), np.uint8)
    e8 = np.zeros((rows, NB), np.uint8)
    outl = np.zeros((rows, O.size), np.uint16)
    rc = _load().orc_quantize_rows_mx(_ptr(src), rows, K, ld, _ptr(O), O.size,
                                      _ptr(codes), _ptr(e8), _ptr(outl))
    if rc != 0:
        raise ValueError("invalid outlier channel set")
    return codes, e8, outl


def dual_linear_rows_mx(qx, ex, xo, qw, ew, wo):
    """(acc_mx float64, acc_o float64, y float64), each [rows of qx, rows of qw]."""
    qx = np.ascontiguousarray(qx, np.uint8)
    qw = np.ascontiguousarray(qw, np.uint8)
    ex = np.ascontiguousarray(ex, np.uint8)
    ew = np.ascontiguousarray(ew, np.uint8)
    xo = np.ascontiguousarray(xo, np.uint16)
    wo = np.ascontiguousarray(wo, np.uint16)
    Mr, KN = qx.shape
    N = qw.shape[0]
    nO = xo.shape[1]
    NB = (KN + MX_BLOCK - 1) // MX_BLOCK
    assert qw.shape[1] == KN and wo.shape == (N, nO) and xo.shape[0] == Mr
    assert ex.shape == (Mr, NB) and ew.shape == (N, NB)
    acc_mx = np.zeros((Mr, N), np.float64)
    acc_o = np.zeros((Mr, N), np.float64)
    y = np.zeros((Mr, N), np.float64)
    _load().orc_dual_linear_rows_mx(_ptr(qx), _ptr(ex), _ptr(xo), Mr, _ptr(qw), _ptr(ew), _ptr(wo),
                                    N, KN, nO, _ptr(acc_mx), _ptr(acc_o), _ptr(y))
    return acc_mx, acc_o, y


def linear_mx(X_bits: np.ndarray, W_bits: np.ndarray, O, rows=None):
    """Whole layer with the MXFP4 low path for the selected activation rows (all when None)."""
    K = W_bits.shape[1]
    Xs = X_bits if rows is None else X_bits[np.asarray(rows)]
    qx, ex, xo = quantize_rows_mx(Xs, K, O)
    qw, ew, wo = quantize_rows_mx(W_bits, K, O)
    acc_mx, acc_o, y = dual_linear_rows_mx(qx, ex, xo, qw, ew, wo)
    return dict(qx=qx, ex=ex, xo=xo, qw=qw, ew=ew, wo=wo, acc_mx=acc_mx, acc_o=acc_o, y=y)


def pack_fp4(codes: np.ndarray, row_bytes: int) -> np.ndarray:
    """Packed storage of 4-bit codes: byte j = code 2j (low nibble) | code 2j+1 (high nibble), zero padded."""
    codes = np.ascontiguousarray(codes, np.uint8)
    rows, KN = codes.shape
    if 2 * row_bytes < KN:
        raise ValueError("row_bytes too small")
    padded = np.zeros((rows, 2 * row_bytes), np.uint8)
    padded[:, :KN] = codes & 15
    return (padded[:, 0::2] | (padded[:, 1::2] << 4)).astype(np.uint8)


def mx_scale_tiles(e8: np.ndarray, rows_pad: int, blocks_pad: int) -> np.ndarray:
    """Block scales in the library's tiled storage order (format definition).

    Rows are grouped by 128 and blocks by 4; each (row group, block group)
    pair is a 512-byte tile in which row r and block b sit at byte
    16*(r%32) + 4*((r%128)//32) + b%4.  Tiles are ordered by row group, then
    block group.  Entries past the given rows and blocks are 0.
    """
    e8 = np.asarray(e8, np.uint8)
    rows, nb = e8.shape
    assert rows_pad % 128 == 0 and blocks_pad % 4 == 0 and rows <= rows_pad and nb <= blocks_pad
    full = np.zeros((rows_pad, blocks_pad), np.uint8)
    full[:rows, :nb] = e8
    r = np.arange(rows_pad)[:, None]
    b = np.arange(blocks_pad)[None, :]
    off = ((r // 128) * (blocks_pad // 4) + b // 4) * 512 + 16 * (r % 32) + 4 * ((r % 128) // 32) + b % 4
    out = np.zeros(rows_pad * blocks_pad, np.uint8)
    out[off.reshape(-1)] = full.reshape(-1)
    return out


# ---------------------------------------------------------------- element-level SQ-format (weights)
SQF_BANKS = [(4, 1), (4, 2), (8, 1), (8, 2), (16, 1), (16, 2)]   # (bank, high entries per bank)


def sqf_weights(W_bits: np.ndarray, bank: int, h: int):
    """Element-level SQ-format of bf16 weight rows: dict with lo (int8 [N, K], -8 at high
    positions), s_lo (fp32 [N]), hi_mask (uint8 [N, K]), hi (uint8 E4M3 [N, K], 0 at low
    positions), s_hi (fp32 [N])."""
    src = np.ascontiguousarray(W_bits, np.uint16)
    rows, K = src.shape
    lo = np.zeros((rows, K), np.int8)
    s_lo = np.zeros(rows, np.float32)
    mask = np.zeros((rows, K), np.uint8)
    hi = np.zeros((rows, K), np.uint8)
    s_hi = np.zeros(rows, np.float32)
    if _load().orc_sqf_weights(_ptr(src), rows, K, K, bank, h, _ptr(lo), _ptr(s_lo), _ptr(mask), _ptr(hi),
                               _ptr(s_hi)) != 0:
        raise ValueError("need 1 <= h < bank and K % bank == 0")
    return dict(lo=lo, s_lo=s_lo, hi_mask=mask, hi=hi, s_hi=s_hi)


def sqf_linear(X_bits: np.ndarray, W_bits: np.ndarray, bank: int, h: int, rows=None):
    """Whole layer with element-level SQ-format weights for the selected token rows (all when None):
    the weight format (sqf_weights), the tokens' INT4 and E4M3 codes over all channels, and
    acc_lo (int64), acc_hi (fp64), y (fp64), each [rows, N]."""
    Xs = X_bits if rows is None else X_bits[np.asarray(rows)]
    return sqf_products(Xs, sqf_weights(W_bits, bank, h))


def sqf_products(X_bits: np.ndarray, w: dict):
    """The layer for token rows X_bits against a weight format w from sqf_weights."""
    Xs = np.ascontiguousarray(X_bits, np.uint16)
    K = w["lo"].shape[1]
    none = np.zeros(0, np.int32)
    qx4, sx4, _ = quantize_rows(Xs, K, none)
    qx8, sx8, _ = quantize_rows_fp8(Xs, K, none)
    Mr, N = Xs.shape[0], w["lo"].shape[0]
    acc_lo = np.zeros((Mr, N), np.int64)
    acc_hi = np.zeros((Mr, N), np.float64)
    y = np.zeros((Mr, N), np.float64)
    _load().orc_sqf_linear_rows(_ptr(qx4), _ptr(sx4), _ptr(qx8), _ptr(sx8), Mr, _ptr(w["lo"]), _ptr(w["s_lo"]),
                                _ptr(w["hi_mask"]), _ptr(w["hi"]), _ptr(w["s_hi"]), N, K,
                                _ptr(acc_lo), _ptr(acc_hi), _ptr(y))
    return dict(w, qx4=qx4, sx4=sx4, qx8=qx8, sx8=sx8, acc_lo=acc_lo, acc_hi=acc_hi, y=y)


def compress_24(hi_mask: np.ndarray, hi_codes: np.ndarray):
    """2:4 storage of the high part (format definition): for every aligned group of 4
    channels, 2 value bytes (the group's high codes in channel order; a group with fewer
    than two high channels stores zeros in the free slots) and one metadata nibble (group i
    in byte i // 2, low nibble for even i) whose bits [1:0] and [3:2] give the in-group
    indices of the two stored values, first < second.  One high channel at index p uses
    indices (p, p + 1) with the zero second, or (2, 3) with the zero first when p = 3; no
    high channel uses (0, 1).  Returns (values uint8 [rows, K/2], meta uint8 [rows, K/8])."""
    mask = np.asarray(hi_mask, np.uint8).astype(bool)
    codes = np.asarray(hi_codes, np.uint8)
    rows, K = mask.shape
    m4 = mask.reshape(rows, K // 4, 4)
    c4 = codes.reshape(rows, K // 4, 4)
    cnt = m4.sum(axis=2)
    if np.any(cnt > 2):
        raise ValueError("more than two high channels in a group of four")
    first = np.argmax(m4, axis=2)                    # lowest high index (0 when none)
    last = 3 - np.argmax(m4[:, :, ::-1], axis=2)     # highest high index
    one_lo = (cnt == 1) & (first < 3)                # (p, p + 1), value first
    one_hi = (cnt == 1) & (first == 3)               # (2, 3), value second
    i0 = np.where(cnt == 2, first, np.where(one_lo, first, np.where(one_hi, 2, 0)))
    i1 = np.where(cnt == 2, last, np.where(one_lo, first + 1, np.where(one_hi, 3, 1)))
    take = lambda idx: np.take_along_axis(c4, idx[:, :, None], axis=2)[:, :, 0]
    v0 = np.where((cnt == 2) | one_lo, take(first), 0).astype(np.uint8)
    v1 = np.where(cnt == 2, take(last), np.where(one_hi, take(np.full_like(first, 3)), 0)).astype(np.uint8)
    vals = np.stack([v0, v1], axis=2).reshape(rows, K // 2)
    nib = (i0 | (i1 << 2)).astype(np.uint8)
    meta = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    return vals, meta
