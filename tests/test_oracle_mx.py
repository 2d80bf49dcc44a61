"""Pins for the oracle's micro-scaling FP4 (MXFP4) low path (no GPU).

The pages say only that the channel split fits 4-bit micro-scaling hardware
(OSC abstract) and that the SQ format also works with FP4 data (SQ-format
write-up, section 8).  The block format is the open MX definition of FP4:
blocks of 32 normal channels, one E8M0 power-of-two scale per block
(E = floor(log2 absmax) - 2, clamped to [-127, 127]), E2M1 codes (magnitudes
0, 0.5, 1, 1.5, 2, 3, 4, 6), nearest with ties to the even code, saturating.

Each test ties the oracle to something other than its own code: the printed
E2M1 value table, brute-force nearest-value search in exact rationals, the
exponent read off the bf16 bit pattern with integer arithmetic, numpy fp64
matmuls, invariants (power-of-two scaling, sign symmetry, block
independence) and loop-based restatements of the storage formats.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workloads

# The E2M1 magnitudes of codes 0..7 as the MX definition lists them.
E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
GRID = [Fraction(v) for v in E2M1_TABLE]


def nearest_code(t: Fraction, negative: bool) -> int:
    """Brute force: the E2M1 code nearest to |t| (ties to the code with mantissa bit 0), saturating."""
    v = abs(t)
    if v >= 6:
        mag = 7
    else:
        best = None
        for c, g in enumerate(GRID):
            d = abs(v - g)
            if best is None or d < best[0] or (d == best[0] and c % 2 == 0 and best[1] % 2 == 1):
                best = (d, c)
        mag = best[1]
    return mag | (8 if negative else 0)


def bf16_floor_log2(bits: int) -> int:
    """floor(log2 |x|) of a nonzero finite bf16 value, from its bit pattern."""
    e = (bits >> 7) & 0xFF
    m = bits & 0x7F
    if e == 0:
        return -133 + m.bit_length() - 1   # subnormal: m * 2^-133
    return e - 127


def exact_mx_row(bits_row: np.ndarray, normal: np.ndarray):
    """Independent statement of the MX quantizer for one row in exact rationals."""
    codes, e8 = [], []
    KN = len(normal)
    for j0 in range(0, KN, 32):
        blk = [int(bits_row[k]) for k in normal[j0:j0 + 32]]
        vals = [Fraction(float(workloads_bits_to_f32(b))) for b in blk]
        nz = [b for b in blk if b & 0x7FFF]
        if not nz:
            E = -127
        else:
            top = max(nz, key=lambda b: abs(Fraction(float(workloads_bits_to_f32(b)))))
            E = max(-127, min(127, bf16_floor_log2(top & 0x7FFF) - 2))
        e8.append(E + 127)
        for b, v in zip(blk, vals):
            codes.append(nearest_code(v / Fraction(2) ** E, bool(b & 0x8000)))
    return codes, e8


def workloads_bits_to_f32(b: int) -> np.float32:
    return np.array([b << 16], np.uint32).view(np.float32)[0]


def f32_bits(a) -> np.ndarray:
    """bf16 bit patterns (uint16) of float32 values that are exact in bf16."""
    t = torch.from_numpy(np.ascontiguousarray(a, np.float32))
    b = t.to(torch.bfloat16)
    assert torch.equal(b.float(), t)
    return workloads.bf16_bits(b)


def to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def dequant(codes: np.ndarray, e8: np.ndarray) -> np.ndarray:
    """codes [R, KN] and e8 [R, NB] -> float64 values code * 2^E."""
    R, KN = codes.shape
    vals = np.array(E2M1_TABLE, np.float64)[codes & 7] * np.where(codes & 8, -1.0, 1.0)
    E = e8.astype(np.int64) - 127
    return vals * np.exp2(np.repeat(E, 32, axis=1)[:, :KN].astype(np.float64))


def _case(M=40, K=512, nO=24, seed=3, kind="gauss"):
    O = workloads.outlier_channels(K, nO, seed=seed)
    X = workloads.activations(M, K, O, kind=kind, seed=seed + 1)
    return O.numpy(), workloads.bf16_bits(X)


# ----------------------------------------------------------------- element format
def test_e2m1_decode_matches_printed_table():
    got = oracle.e2m1_decode(np.arange(16))
    assert list(got[:8]) == E2M1_TABLE
    assert list(got[8:]) == [-v for v in E2M1_TABLE]
    assert np.signbit(got[8])   # code 8 is -0


def test_e2m1_encode_brute_force():
    """Nearest-even encoding agrees with a brute-force search in exact rationals,
    on every grid value, every midpoint (the ties), values just beside them,
    saturation and random values."""
    g = np.array(E2M1_TABLE)
    mids = (g[:-1] + g[1:]) / 2
    eps = 2.0 ** -30
    rng = np.random.default_rng(5)
    t = np.concatenate([g, mids, mids + eps, mids - eps, [6.0, 6.5, 7.0, 8.0, 1e30, 0.0],
                        rng.uniform(0, 8, 4000), rng.uniform(0, 0.5, 1000)])
    t = np.concatenate([t, -t])
    got = oracle.e2m1_encode(t)
    want = [nearest_code(Fraction(float(v)), bool(np.signbit(v))) for v in t]
    assert list(got) == want


def test_e2m1_ties_and_signed_zero():
    t = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.2, -0.0, 0.0])
    # ties go to the code with mantissa bit 0: 0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0
    assert list(oracle.e2m1_encode(t)) == [0, 2, 2, 4, 4, 6, 6, 8, 8, 0]


def test_block_exponent_from_bit_patterns():
    """E = floor(log2 a) - 2, clamped: checked against the bf16 exponent field
    (normal and subnormal patterns) with integer arithmetic."""
    pats = list(range(1, 0x7F80, 7)) + [0x0001, 0x007F, 0x0080, 0x3F80, 0x3FFF, 0x7F7F]
    for b in pats:
        a = float(workloads_bits_to_f32(b))
        want = max(-127, min(127, bf16_floor_log2(b) - 2))
        assert oracle.mx_block_exponent(a) == want, hex(b)
    assert oracle.mx_block_exponent(0.0) == -127


# ----------------------------------------------------------------- quantizer
def test_mx_quantizer_matches_exact_rational():
    O, Xb = _case(M=24, K=384, nO=40, seed=7)
    # add rows that exercise clamping, zero blocks, signed zeros and ties
    extra = np.zeros((4, 384), np.uint16)
    extra[0] = 0x0001                      # every entry the smallest subnormal: E clamps to -127
    extra[1, :] = 0x8000                   # -0 everywhere: a = 0
    extra[2] = f32_bits(np.resize(np.array([4.0, 5.0, 3.5, 1.75, 0.25, 0.75, -2.5, 7.0], np.float32),
                                             384).reshape(1, -1))[0]
    extra[3] = 0x7F7F                      # the largest finite bf16
    Xb = np.concatenate([Xb, extra])
    K = Xb.shape[1]
    codes, e8, _ = oracle.quantize_rows_mx(Xb, K, O)
    normal = np.setdiff1d(np.arange(K), O)
    for r in range(Xb.shape[0]):
        c, e = exact_mx_row(Xb[r], normal)
        assert list(codes[r]) == c, r
        assert list(e8[r]) == e, r


def test_mx_block_range_invariant():
    """Unclamped blocks: the largest |t| = a / 2^E lies in [4, 8), so the
    block's absolute maximum lands on magnitude 4 or 6 (6 above 5; 5 is a tie
    that goes to 4)."""
    O, Xb = _case(M=64, K=1024, nO=48, seed=9, kind="swiglu")
    K = Xb.shape[1]
    codes, e8, _ = oracle.quantize_rows_mx(Xb, K, O)
    normal = np.setdiff1d(np.arange(K), O)
    x = to_f64(Xb)[:, normal]
    KN = x.shape[1]
    for b in range(e8.shape[1]):
        blk = np.abs(x[:, 32 * b:32 * b + 32])
        a = blk.max(axis=1)
        t = a / np.exp2(e8[:, b].astype(np.float64) - 127)
        live = a > 0
        assert np.all((t[live] >= 4) & (t[live] < 8))
        am = blk.argmax(axis=1)
        mags = oracle.e2m1_decode(codes[np.arange(len(am)), 32 * b + am])
        assert np.all(np.abs(mags[live]) == np.where(t[live] > 5, 6.0, 4.0))
    # every element within half a grid step of its value (saturation aside)
    d = dequant(codes, e8)
    assert d.shape == (x.shape[0], KN)
    step = np.exp2(np.repeat(e8.astype(np.float64) - 127, 32, axis=1)[:, :KN])
    sat = np.abs(x) > 6 * step
    err = np.abs(d - x)
    assert np.all(err[~sat] <= np.where(np.abs(x[~sat]) < 2 * step[~sat], 0.25, 1.0) * step[~sat])


@pytest.mark.parametrize("e", [-30, -4, 3, 40])
def test_mx_power_of_two_scaling(e):
    O, Xb = _case(seed=11)
    K = Xb.shape[1]
    x = (Xb.astype(np.uint32) << 16).view(np.float32) * np.float32(2.0 ** e)
    Xe = (x.view(np.uint32) >> 16).astype(np.uint16)
    c0, e0, _ = oracle.quantize_rows_mx(Xb, K, O)
    c1, e1, _ = oracle.quantize_rows_mx(Xe, K, O)
    assert np.array_equal(c0, c1)
    assert np.array_equal(e1.astype(np.int64), e0.astype(np.int64) + e)


def test_mx_sign_symmetry():
    O, Xb = _case(seed=13)
    K = Xb.shape[1]
    c0, e0, _ = oracle.quantize_rows_mx(Xb, K, O)
    c1, e1, _ = oracle.quantize_rows_mx(Xb ^ np.uint16(0x8000), K, O)
    assert np.array_equal(e0, e1)
    assert np.array_equal(c1, c0 ^ np.uint8(8))


def test_mx_blocks_are_independent_and_outliers_excluded():
    O, Xb = _case(M=8, K=512, nO=32, seed=15)
    K = Xb.shape[1]
    c0, e0, o0 = oracle.quantize_rows_mx(Xb, K, O)
    # a huge value in an outlier channel changes nothing in the normal part
    Xh = Xb.copy()
    Xh[:, O[0]] = f32_bits(np.full((8, 1), 30720.0, np.float32))[:, 0]
    c1, e1, o1 = oracle.quantize_rows_mx(Xh, K, O)
    assert np.array_equal(c0, c1) and np.array_equal(e0, e1)
    assert np.array_equal(o1[:, 0], Xh[:, O[0]]) and np.array_equal(o1[:, 1:], o0[:, 1:])
    # a huge value in normal block 3 changes block 3 only
    normal = np.setdiff1d(np.arange(K), O)
    Xg = Xb.copy()
    Xg[:, normal[3 * 32 + 5]] = f32_bits(np.full((8, 1), 30720.0, np.float32))[:, 0]
    c2, e2, _ = oracle.quantize_rows_mx(Xg, K, O)
    keep = np.ones(c0.shape[1], bool)
    keep[96:128] = False
    assert np.array_equal(c0[:, keep], c2[:, keep])
    kb = np.ones(e0.shape[1], bool)
    kb[3] = False
    assert np.array_equal(e0[:, kb], e2[:, kb]) and np.all(e2[:, 3] > e0[:, 3])


def test_mx_partial_last_block():
    """K - nO not a multiple of 32: the last block's scale comes from its real entries only."""
    K, nO = 520, 24          # KN = 496 = 15 * 32 + 16
    O, Xb = _case(M=6, K=K, nO=nO, seed=17)
    codes, e8, _ = oracle.quantize_rows_mx(Xb, K, O)
    assert codes.shape == (6, 496) and e8.shape == (6, 16)
    normal = np.setdiff1d(np.arange(K), O)
    for r in range(6):
        c, e = exact_mx_row(Xb[r], normal)
        assert list(codes[r]) == c and list(e8[r]) == e


# ----------------------------------------------------------------- products
def test_mx_products_exact_rational():
    """acc_mx equals the exact rational sum over blocks of 2^(Ex+Ew) times the
    block's sum of decoded products (small K: exact in fp64)."""
    O, Xb = _case(M=5, K=256, nO=8, seed=19)
    Wb = workloads.bf16_bits(workloads.weights(4, 256, seed=20))
    ref = oracle.linear_mx(Xb, Wb, O)
    KN = 248
    for m in range(5):
        for n in range(4):
            tot = Fraction(0)
            for b in range(0, KN, 32):
                s = sum(Fraction(float(p)) * Fraction(float(q)) for p, q in
                        zip(oracle.e2m1_decode(ref["qx"][m, b:b + 32]), oracle.e2m1_decode(ref["qw"][n, b:b + 32])))
                tot += s * Fraction(2) ** (int(ref["ex"][m, b // 32]) - 127 + int(ref["ew"][n, b // 32]) - 127)
            assert Fraction(ref["acc_mx"][m, n]) == tot


def test_mx_reductions():
    """nO = 0: the fp64 matmul of the dequantized operands; nO = K: a plain bf16 GEMM."""
    M, K, N = 24, 384, 40
    X = workloads.activations(M, K, workloads.outlier_channels(K, 0, seed=1), seed=2)
    W = workloads.weights(N, K, seed=3)
    Xb, Wb = workloads.bf16_bits(X), workloads.bf16_bits(W)
    r0 = oracle.linear_mx(Xb, Wb, np.zeros(0, np.int32))
    y0 = dequant(r0["qx"], r0["ex"]) @ dequant(r0["qw"], r0["ew"]).T
    assert np.allclose(r0["y"], y0, rtol=1e-12, atol=1e-300)
    assert np.all(r0["acc_o"] == 0)
    rK = oracle.linear_mx(Xb, Wb, np.arange(K, dtype=np.int32))
    assert np.allclose(rK["y"], to_f64(Xb) @ to_f64(Wb).T, rtol=1e-12, atol=1e-12)
    assert rK["qx"].shape == (M, 0) and rK["ex"].shape == (M, 0) and np.all(rK["acc_mx"] == 0)


# ----------------------------------------------------------------- storage formats
def test_pack_fp4_definition():
    rng = np.random.default_rng(21)
    codes = rng.integers(0, 16, size=(3, 37)).astype(np.uint8)
    packed = oracle.pack_fp4(codes, 24)
    for r in range(3):
        for j in range(24):
            lo = int(codes[r, 2 * j]) if 2 * j < 37 else 0
            hi = int(codes[r, 2 * j + 1]) if 2 * j + 1 < 37 else 0
            assert packed[r, j] == lo | (hi << 4)


def test_mx_scale_tiles_definition():
    rng = np.random.default_rng(22)
    e8 = rng.integers(1, 255, size=(150, 10)).astype(np.uint8)
    out = oracle.mx_scale_tiles(e8, 256, 12)
    assert out.size == 256 * 12
    seen = np.zeros(out.size, int)
    for r in range(256):
        for b in range(12):
            tile = (r // 128) * 3 + b // 4
            off = tile * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (b % 4)
            seen[off] += 1
            assert out[off] == (e8[r, b] if r < 150 and b < 10 else 0)
    assert np.all(seen == 1)


# ----------------------------------------------------------------- method sanity
def test_mx_outlier_branch_helps():
    """Method sanity (information): with activations whose outlier channels are
    x30, moving those channels to the 16-bit branch lowers the MX path's error
    against the exact X W^T, as it does for INT4."""
    w = workloads.Workload("t", 64, 1024, 96, 64, x_kind="gauss", sigma=30.0)
    O, X, W = workloads.make(w)
    Xb, Wb = workloads.bf16_bits(X), workloads.bf16_bits(W)
    exact = to_f64(Xb) @ to_f64(Wb).T
    e_with = np.linalg.norm(oracle.linear_mx(Xb, Wb, O.numpy())["y"] - exact) / np.linalg.norm(exact)
    e_without = np.linalg.norm(oracle.linear_mx(Xb, Wb, np.zeros(0, np.int32))["y"] - exact) / np.linalg.norm(exact)
    assert e_with < e_without
    assert e_with < 0.05 and 5 * e_with < e_without
