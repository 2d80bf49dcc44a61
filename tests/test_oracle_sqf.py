"""Pins for the oracle's element-level SQ-format weights (no GPU).

Format (SQ-format write-up: banks with a fixed number of high-precision
entries, section 7; top (1-s) per bank by importance, the unused top code of
the symmetric low format as the mask, section 9; FP8/FP4 combination, section
8): in every bank of `bank` consecutive channels of a weight row the `h`
largest-magnitude entries (ties to the lower index) are high precision (E4M3,
scale absmax/448 over the row's high entries); the rest are symmetric INT4
(scale absmax/7 over the row's low entries) with the code -8 at every high
position.  Tokens are quantized over all channels twice (INT4 for the low
part, E4M3 for the high part).

Pins: brute-force bank selection; the low part restated with exact rational
arithmetic; the high codes against torch's float8_e4m3fn conversion; layer
outputs against numpy fp64 matmuls of the split and against exact rationals;
the 2:4 storage restated by loops and decoded back.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workloads
from test_oracle import exact_quant_row

BANKS = oracle.SQF_BANKS


def to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def brute_mask(row_bits: np.ndarray, bank: int, h: int) -> np.ndarray:
    v = np.abs(to_f32(row_bits).astype(np.float64))
    out = np.zeros(v.size, np.uint8)
    for g in range(v.size // bank):
        order = sorted(range(bank), key=lambda i: (-v[g * bank + i], i))
        for i in order[:h]:
            out[g * bank + i] = 1
    return out


def tie_rows(rng, rows, K):
    """Rows with many equal magnitudes (ties inside banks) and some zeros."""
    vals = np.array([0.0, 0.5, -0.5, 1.0, -1.0, 0.25, 2.0], np.float32)
    x = rng.choice(vals, size=(rows, K)).astype(np.float32)
    return workloads.bf16_bits(torch.from_numpy(x).to(torch.bfloat16))


@pytest.mark.parametrize("bank,h", BANKS)
def test_bank_selection_brute_force(bank, h):
    rng = np.random.default_rng(bank * 10 + h)
    W = np.concatenate([workloads.bf16_bits(workloads.weights(12, 256, seed=bank + h)), tie_rows(rng, 6, 256)])
    w = oracle.sqf_weights(W, bank, h)
    for r in range(W.shape[0]):
        assert np.array_equal(w["hi_mask"][r], brute_mask(W[r], bank, h)), r
    per_bank = w["hi_mask"].reshape(W.shape[0], -1, bank).sum(axis=2)
    assert np.all(per_bank == h)
    # at most two high entries in any aligned group of four (the 2:4 storage relies on it)
    assert np.all(w["hi_mask"].reshape(W.shape[0], -1, 4).sum(axis=2) <= 2)


@pytest.mark.parametrize("bank,h", [(4, 2), (8, 1), (16, 2)])
def test_low_part_matches_exact_rational(bank, h):
    """The low part is the symmetric INT4 quantizer over the row's low entries (scale
    fl32(a/7), codes rint(fl32(x/s)) clamped), restated in exact rational arithmetic;
    the mask code -8 sits exactly at the high positions."""
    rng = np.random.default_rng(3)
    W = np.concatenate([workloads.bf16_bits(workloads.weights(10, 128, seed=9)), tie_rows(rng, 4, 128)])
    w = oracle.sqf_weights(W, bank, h)
    for r in range(W.shape[0]):
        xs = [Fraction(float(v)) for v in to_f32(W[r])]
        low = [k for k in range(128) if not w["hi_mask"][r, k]]
        s, codes = exact_quant_row(xs, low)
        assert Fraction(float(w["s_lo"][r])) == s
        assert [int(w["lo"][r, k]) for k in low] == codes
        assert np.all(w["lo"][r][w["hi_mask"][r] == 1] == -8)


@pytest.mark.parametrize("bank,h", [(4, 1), (8, 2), (16, 1)])
def test_high_part_matches_library_e4m3(bank, h):
    W = workloads.bf16_bits(workloads.weights(16, 512, seed=21))
    w = oracle.sqf_weights(W, bank, h)
    x = to_f32(W)
    for r in range(W.shape[0]):
        m = w["hi_mask"][r] == 1
        a = np.float32(np.abs(x[r][m]).max())
        s = np.float32(a / np.float32(448.0))
        assert w["s_hi"][r] == s
        t = (x[r][m] / s).astype(np.float32)
        ref = torch.from_numpy(t.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(w["hi"][r][m], ref)
        assert np.all(w["hi"][r][~m] == 0)
        # the row's largest high entry lands on +-448
        assert np.abs(oracle.e4m3_decode(w["hi"][r][m])).max() == 448.0


def _layer(bank, h, M=6, K=256, N=10, seed=31):
    X = workloads.activations(M, K, workloads.outlier_channels(K, 0), seed=seed)
    W = workloads.weights(N, K, seed=seed + 1)
    return workloads.bf16_bits(X), workloads.bf16_bits(W)


@pytest.mark.parametrize("bank,h", BANKS)
def test_layer_matches_numpy_split(bank, h):
    """y equals numpy fp64 matmuls of the masked low codes and the decoded high codes."""
    Xb, Wb = _layer(bank, h)
    r = oracle.sqf_linear(Xb, Wb, bank, h)
    mask = r["hi_mask"].astype(bool)
    lo = np.where(mask, 0, r["lo"]).astype(np.int64)
    acc_lo = r["qx4"].astype(np.int64) @ lo.T
    assert np.array_equal(acc_lo, r["acc_lo"])
    dx = oracle.e4m3_decode(r["qx8"]).reshape(r["qx8"].shape)
    dw = np.where(mask, oracle.e4m3_decode(r["hi"]).reshape(r["hi"].shape), 0.0)
    acc_hi = dx @ dw.T
    assert np.allclose(acc_hi, r["acc_hi"], rtol=1e-13, atol=1e-300)
    y = acc_lo * r["sx4"][:, None].astype(np.float64) * r["s_lo"][None, :].astype(np.float64) + \
        acc_hi * r["sx8"][:, None].astype(np.float64) * r["s_hi"][None, :].astype(np.float64)
    assert np.allclose(y, r["y"], rtol=1e-12, atol=1e-300)


def test_layer_exact_rational_tiny():
    Xb, Wb = _layer(8, 2, M=3, K=64, N=4, seed=41)
    r = oracle.sqf_linear(Xb, Wb, 8, 2)
    for m in range(3):
        for n in range(4):
            lo = sum(int(r["qx4"][m, k]) * int(r["lo"][n, k]) for k in range(64) if not r["hi_mask"][n, k])
            hi = sum(Fraction(float(oracle.e4m3_decode(np.uint8(r["qx8"][m, k]))[0])) *
                     Fraction(float(oracle.e4m3_decode(np.uint8(r["hi"][n, k]))[0]))
                     for k in range(64) if r["hi_mask"][n, k])
            assert r["acc_lo"][m, n] == lo
            assert Fraction(r["acc_hi"][m, n]) == hi
            y = Fraction(lo) * Fraction(float(r["sx4"][m])) * Fraction(float(r["s_lo"][n])) + \
                hi * Fraction(float(r["sx8"][m])) * Fraction(float(r["s_hi"][n]))
            assert abs(Fraction(r["y"][m, n]) - y) <= abs(y) * Fraction(1, 2 ** 50) + Fraction(1, 2 ** 200)


def test_zero_rows_and_invalid_banks():
    W = np.zeros((3, 64), np.uint16)
    W[1, 5] = workloads.bf16_bits(torch.tensor([[2.0]], dtype=torch.bfloat16))[0, 0]
    w = oracle.sqf_weights(W, 4, 1)
    assert w["s_lo"][0] == 0 and w["s_hi"][0] == 0 and np.all(w["hi"][0] == 0)
    assert np.all(w["lo"][0][w["hi_mask"][0] == 1] == -8) and np.all(w["lo"][0][w["hi_mask"][0] == 0] == 0)
    assert w["hi_mask"][1, 5] == 1 and w["s_lo"][1] == 0 and oracle.e4m3_decode(w["hi"][1, 5:6])[0] == 448.0
    for bank, h in [(4, 0), (4, 4), (3, 1)]:
        with pytest.raises(ValueError):
            oracle.sqf_weights(W, bank, h)   # h outside [1, bank), or K = 64 not a multiple of the bank


@pytest.mark.parametrize("bank,h", BANKS)
def test_compress_24_round_trip(bank, h):
    Wb = workloads.bf16_bits(workloads.weights(8, 128, seed=bank + 2 * h))
    w = oracle.sqf_weights(Wb, bank, h)
    vals, meta = oracle.compress_24(w["hi_mask"], w["hi"])
    for r in range(8):
        dense = np.zeros(128, np.uint8)
        for g in range(32):
            nib = (int(meta[r, g // 2]) >> (4 * (g % 2))) & 15
            i0, i1 = nib & 3, nib >> 2
            assert i0 < i1
            dense[4 * g + i0] = vals[r, 2 * g]
            dense[4 * g + i1] |= vals[r, 2 * g + 1]
        assert np.array_equal(dense, np.where(w["hi_mask"][r] == 1, w["hi"][r], 0))


def test_high_entries_cut_the_weight_error():
    """Method sanity (information): keeping the largest entry of every bank of 16 in E4M3
    cuts the reconstruction error of the weights against plain per-row INT4."""
    W = workloads.weights(64, 1024, seed=51).float()
    W[:, ::37] *= 20.0      # a few large entries per row
    Wb = workloads.bf16_bits(W.to(torch.bfloat16))
    x = to_f32(Wb).astype(np.float64)
    w = oracle.sqf_weights(Wb, 16, 1)
    mask = w["hi_mask"].astype(bool)
    rec = np.where(mask, oracle.e4m3_decode(w["hi"]).reshape(x.shape) * w["s_hi"][:, None],
                   w["lo"] * w["s_lo"][:, None].astype(np.float64))
    q, s, _ = oracle.quantize_rows(Wb, 1024, np.zeros(0, np.int32))
    plain = q * s[:, None].astype(np.float64)
    e_sqf = np.linalg.norm(rec - x) / np.linalg.norm(x)
    e_int4 = np.linalg.norm(plain - x) / np.linalg.norm(x)
    assert e_sqf < 0.5 * e_int4
