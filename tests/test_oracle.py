"""Pins for the CPU oracle (no GPU).

Each test ties the oracle to something other than itself: hand-worked golden
cases, exact rational arithmetic, closed-form reductions to library routines
(numpy integer / fp64 matmul), brute force on tiny inputs, and invariants of
the quantizer (bound, split reconstruction, power-of-two scaling, sign
symmetry, channel-permutation invariance).
"""
from __future__ import annotations

import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------- helpers
def bf16_bits_of(values) -> np.ndarray:
    t = torch.tensor(values, dtype=torch.float32)
    b = t.to(torch.bfloat16)
    assert torch.equal(b.float(), t), "golden values must be exact in bf16"
    return b.view(torch.int16).numpy().view(np.uint16)


def bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f32_round(q: Fraction) -> Fraction:
    """Round a rational to the nearest IEEE binary32 value, ties to even."""
    if q == 0:
        return Fraction(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -126)
    quantum = Fraction(2) ** (e - 23)
    n = a / quantum
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * fl * quantum


def exact_quant_row(xs: list[Fraction], normal: list[int]):
    """Independent statement of the quantizer in exact rational arithmetic."""
    a = max((abs(xs[k]) for k in normal), default=Fraction(0))
    if a == 0:
        return Fraction(0), [0] * len(normal)
    s = f32_round(a / 7)
    codes = []
    for k in normal:
        t = f32_round(xs[k] / s)
        q = round(t)  # Fraction.__round__ rounds half to even
        codes.append(max(-7, min(7, q)))
    return s, codes


def parse_cases(path):
    cases, cur = [], None
    for raw in open(path):
        line = raw.split("#", 1)[0].strip()
        if not line:
            continue
        key, *rest = line.split()
        if key == "case":
            cur = {"name": rest[0]}
            cases.append(cur)
        else:
            cur[key] = rest
    return cases


# ----------------------------------------------------------------- golden
@pytest.mark.parametrize("case", parse_cases(os.path.join(GOLDEN, "quant_rows.txt")),
                         ids=lambda c: c["name"])
def test_golden_quant_rows(case):
    K = int(case["K"][0])
    O = [int(v) for v in case.get("O", [])]
    x = [float(v) for v in case["x"]]
    codes, scale, outl = oracle.quantize_rows(bf16_bits_of([x]), K, O)
    assert scale[0] == np.float32(float.fromhex(case["scale"][0]))
    assert codes[0].tolist() == [int(v) for v in case.get("codes", [])]
    assert outl[0].tolist() == bf16_bits_of([[float(v) for v in case.get("outl", [])]] if case.get("outl") else [[]]).reshape(-1).tolist()


def test_golden_dual_linear():
    case = {}
    for raw in open(os.path.join(GOLDEN, "dual_linear.txt")):
        line = raw.split("#", 1)[0].strip()
        if line:
            key, *rest = line.split()
            case.setdefault(key, []).append(rest)
    K = int(case["K"][0][0])
    O = [int(v) for v in case["O"][0]]
    X = bf16_bits_of([[float(v) for v in r] for r in case["X"]])
    W = bf16_bits_of([[float(v) for v in r] for r in case["W"]])
    r = oracle.linear(X, W, O)
    assert r["acc_i"].tolist() == [[int(v) for v in row] for row in case["acc_i"]]
    assert r["y"].tolist() == [[float(v) for v in row] for row in case["y"]]
    assert K == X.shape[1]


# ----------------------------------------------------------------- exact arithmetic
def _tie_heavy_rows(rng, rows, K):
    """bf16 rows whose entries sit on or next to rounding ties of x/s."""
    out = []
    for _ in range(rows):
        a = float(2.0 ** rng.integers(-6, 6)) * float(rng.choice([1.0, 1.5, 1.25, 1.75]))
        halves = rng.integers(-14, 15, size=K).astype(np.float64) / 2.0  # multiples of 0.5 in [-7, 7]
        xs = halves * (a / 7.0)
        xs[rng.integers(0, K)] = a * rng.choice([-1.0, 1.0])
        out.append(xs)
    b = torch.tensor(np.array(out), dtype=torch.float32).to(torch.bfloat16)
    return b.view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("kind", ["gauss", "ties"])
def test_quantizer_matches_exact_rational(kind):
    rng = np.random.default_rng(7)
    K, nO = 48, 5
    O = np.sort(rng.choice(K, nO, replace=False)).astype(np.int32)
    if kind == "gauss":
        bits = workloads.bf16_bits(workloads.activations(64, K, torch.from_numpy(O), sigma=30.0, seed=11))
    else:
        bits = _tie_heavy_rows(rng, 64, K)
    codes, scale, outl = oracle.quantize_rows(bits, K, O)
    normal = [k for k in range(K) if k not in set(O.tolist())]
    xf = bits_to_f64(bits)
    for r in range(bits.shape[0]):
        xs = [Fraction(float(v)) for v in xf[r]]
        s, q = exact_quant_row(xs, normal)
        assert Fraction(float(scale[r])) == s
        assert codes[r].tolist() == q
        assert outl[r].tolist() == bits[r, O].tolist()


# ----------------------------------------------------------------- invariants
def _tiny():
    w = workloads.TINY
    O, X, W = workloads.make(w)
    return w, O.numpy(), workloads.bf16_bits(X), workloads.bf16_bits(W)


def test_quantizer_bound_and_range():
    w, O, Xb, Wb = _tiny()
    for bits in (Xb, Wb):
        codes, scale, _ = oracle.quantize_rows(bits, w.K, O)
        normal = np.setdiff1d(np.arange(w.K), O)
        x = bits_to_f64(bits)[:, normal]
        s = scale.astype(np.float64)[:, None]
        assert codes.min() >= -7 and codes.max() <= 7
        err = np.abs(x - s * codes)
        assert np.all(err <= s / 2 * (1 + 2.0 ** -20))
        amax = np.argmax(np.abs(x), axis=1)
        assert np.all(np.abs(codes[np.arange(len(x)), amax]) == 7)


def test_split_reconstruction_is_exact():
    w, O, Xb, _ = _tiny()
    codes, scale, outl = oracle.quantize_rows(Xb, w.K, O)
    # Scatter the compact outlier tensor back: bit-identical to X on O.
    back = np.zeros_like(Xb)
    back[:, O] = outl
    assert np.array_equal(back[:, O], Xb[:, O])
    assert np.all(back[:, np.setdiff1d(np.arange(w.K), O)] == 0)
    # Every channel lands in exactly one part.
    assert codes.shape[1] + outl.shape[1] == w.K
    # Scatter the dequantized normal part back: it approximates X off O
    # (within half a step) and is exactly zero on O.
    normal = np.setdiff1d(np.arange(w.K), O)
    deq = np.zeros((Xb.shape[0], w.K))
    deq[:, normal] = scale[:, None].astype(np.float64) * codes
    x = bits_to_f64(Xb)
    assert np.all(deq[:, O] == 0)
    assert np.all(np.abs(deq[:, normal] - x[:, normal]) <= scale[:, None] / 2 * (1 + 2.0 ** -20))


@pytest.mark.parametrize("e", [-3, 1, 5])
def test_power_of_two_scaling(e):
    w, O, Xb, _ = _tiny()
    codes, scale, _ = oracle.quantize_rows(Xb, w.K, O)
    Xs = (torch.from_numpy(Xb.view(np.int16)).view(torch.bfloat16).float() * 2.0 ** e).to(torch.bfloat16)
    codes2, scale2, _ = oracle.quantize_rows(workloads.bf16_bits(Xs), w.K, O)
    assert np.array_equal(codes, codes2)
    assert np.array_equal(scale.astype(np.float64) * 2.0 ** e, scale2.astype(np.float64))


def test_sign_symmetry():
    w, O, Xb, _ = _tiny()
    codes, scale, outl = oracle.quantize_rows(Xb, w.K, O)
    neg = Xb ^ np.uint16(0x8000)
    codes_n, scale_n, outl_n = oracle.quantize_rows(neg, w.K, O)
    assert np.array_equal(codes_n, -codes)
    assert np.array_equal(scale_n, scale)
    assert np.array_equal(outl_n, outl ^ np.uint16(0x8000))


def test_channel_permutation_invariance():
    w, O, Xb, Wb = _tiny()
    r0 = oracle.linear(Xb, Wb, O)
    perm = np.random.default_rng(3).permutation(w.K)          # new channel j <- old perm[j]
    inv = np.argsort(perm)
    O2 = np.sort(inv[O]).astype(np.int32)
    r1 = oracle.linear(Xb[:, perm], Wb[:, perm], O2)
    assert np.array_equal(r0["acc_i"], r1["acc_i"])
    assert np.array_equal(r0["sx"], r1["sx"]) and np.array_equal(r0["sw"], r1["sw"])
    np.testing.assert_allclose(r1["y"], r0["y"], rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------- reductions
def test_empty_outlier_set_is_plain_w4a4():
    w = workloads.Workload("t", 32, 128, 48, 0)
    O, X, W = workloads.make(w)
    Xb, Wb = workloads.bf16_bits(X), workloads.bf16_bits(W)
    r = oracle.linear(Xb, Wb, O.numpy())
    assert r["xo"].shape == (32, 0) and r["wo"].shape == (48, 0)
    ref = r["qx"].astype(np.int64) @ r["qw"].astype(np.int64).T
    assert np.array_equal(r["acc_i"], ref)
    assert np.all(r["acc_o"] == 0)
    y = ref.astype(np.float64) * r["sx"].astype(np.float64)[:, None] * r["sw"].astype(np.float64)[None, :]
    assert np.array_equal(r["y"], y)


def test_all_channels_outliers_is_bf16_gemm():
    w = workloads.Workload("t", 24, 64, 40, 64)
    O, X, W = workloads.make(w)
    Xb, Wb = workloads.bf16_bits(X), workloads.bf16_bits(W)
    r = oracle.linear(Xb, Wb, O.numpy())
    assert r["qx"].shape == (24, 0) and np.all(r["sx"] == 0) and np.all(r["sw"] == 0)
    ref = bits_to_f64(Xb) @ bits_to_f64(Wb).T
    np.testing.assert_allclose(r["y"], ref, rtol=1e-12, atol=1e-12)


def test_bruteforce_triple_loop():
    rng = np.random.default_rng(5)
    M, N, K = 3, 4, 16
    O = np.sort(rng.choice(K, 3, replace=False)).astype(np.int32)
    X = torch.from_numpy(rng.standard_normal((M, K)).astype(np.float32)).to(torch.bfloat16)
    W = torch.from_numpy(rng.standard_normal((N, K)).astype(np.float32)).to(torch.bfloat16)
    Xb, Wb = workloads.bf16_bits(X), workloads.bf16_bits(W)
    r = oracle.linear(Xb, Wb, O)
    x, wt = bits_to_f64(Xb), bits_to_f64(Wb)
    normal = [k for k in range(K) if k not in set(O.tolist())]
    for m in range(M):
        sx, qx = exact_quant_row([Fraction(float(v)) for v in x[m]], normal)
        for n in range(N):
            sw, qw = exact_quant_row([Fraction(float(v)) for v in wt[n]], normal)
            low = sum(qx[j] * qw[j] for j in range(len(normal)))
            high = sum(Fraction(float(x[m, k])) * Fraction(float(wt[n, k])) for k in O)
            exact = Fraction(low) * sx * sw + high
            assert r["acc_i"][m, n] == low
            assert abs(r["y"][m, n] - float(exact)) <= 1e-12 * max(1.0, abs(float(exact)))


# ----------------------------------------------------------------- storage formats
def test_pack_layout_matches_definition():
    rng = np.random.default_rng(1)
    codes = rng.integers(-7, 8, size=(5, 37)).astype(np.int8)
    packed = oracle.pack_int4(codes, 64)
    for r in range(5):
        expect = bytearray(64)
        for j, c in enumerate(codes[r].tolist()):
            nib = c & 0xF
            expect[j // 2] |= nib if j % 2 == 0 else nib << 4
        assert bytes(packed[r]) == bytes(expect)
    # two's complement nibbles: 0x9 is -7, 0x8 (-8) never appears
    lo = (packed & 0xF).astype(np.int16)
    assert not np.any((lo == 8))


def test_chan_table_definition():
    K = 64
    O = [0, 5, 7, 8, 31, 32, 63]
    tab = oracle.chan_table(O, K)
    for c in range(K // 8):
        below = sum(1 for o in O if o < 8 * c)
        mask = sum(1 << (o - 8 * c) for o in O if 8 * c <= o < 8 * c + 8)
        assert int(tab[c]) == (below << 8) | mask


def decode_chan_map(tab: np.ndarray, K: int) -> np.ndarray:
    """The per-channel map the channel table stands for: >= 0 is the channel's rank among
    the normal channels, -(1+j) marks outlier j (its rank in O)."""
    out = np.zeros(K, np.int64)
    for k in range(K):
        word = int(tab[k // 8])
        below, mask = word >> 8, word & 0xFF
        before = below + bin(mask & ((1 << (k % 8)) - 1)).count("1")   # outliers below k
        out[k] = -(1 + before) if mask >> (k % 8) & 1 else k - before
    return out


@pytest.mark.parametrize("K,nO,seed", [(64, 7, 0), (4096, 256, 1), (2048, 0, 2), (1024, 1024, 3), (14336, 1792, 4)])
def test_chan_table_decodes_to_rank_and_outlier_map(K, nO, seed):
    """The compact table (one word per 8 channels) holds exactly the per-channel
    map chan_map[k] = normal rank, or -(1+j) for outlier j, for a random O."""
    O = np.sort(np.random.default_rng(seed).choice(K, nO, replace=False)).astype(np.int32)
    want = np.zeros(K, np.int64)
    normal = np.setdiff1d(np.arange(K), O)
    want[normal] = np.arange(normal.size)
    want[O] = -(1 + np.arange(nO))
    assert np.array_equal(decode_chan_map(oracle.chan_table(O, K), K), want)


def test_outlier_set_validation():
    assert oracle.validate_outliers([1, 4, 9], 10)
    assert oracle.validate_outliers([], 10)
    assert not oracle.validate_outliers([4, 1], 10)
    assert not oracle.validate_outliers([1, 1], 10)
    assert not oracle.validate_outliers([10], 10)
    assert not oracle.validate_outliers([-1], 10)
    with pytest.raises(ValueError):
        oracle.quantize_rows(np.zeros((1, 8), np.uint16), 8, [3, 2])


# ----------------------------------------------------------------- method sanity
def test_outlier_channels_reduce_error():
    """Routing the true outlier channels through the 16-bit branch must cut the
    error against the exact fp64 product (the point of the channel split)."""
    w = workloads.TINY
    O, X, W = workloads.make(w)
    Xb, Wb = workloads.bf16_bits(X), workloads.bf16_bits(W)
    exact = bits_to_f64(Xb) @ bits_to_f64(Wb).T
    err = {}
    for name, o in (("none", np.zeros(0, np.int32)), ("true", O.numpy())):
        y = oracle.linear(Xb, Wb, o)["y"]
        err[name] = np.linalg.norm(y - exact) / np.linalg.norm(exact)
    assert err["true"] < 0.25 * err["none"]
    assert err["true"] < 0.2


# ----------------------------------------------------------------- FP8 low path (OSC: FP8 fallback for W2 inputs)
def _finite_e4m3_codes():
    c = np.arange(256, dtype=np.uint8)
    return c[(c & 0x7F) != 0x7F]  # 0x7F / 0xFF are NaN in E4M3


def test_e4m3_decode_matches_library():
    """Every finite E4M3 code decodes to the value torch's float8_e4m3fn gives it."""
    c = _finite_e4m3_codes()
    ref = torch.from_numpy(c.copy()).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(oracle.e4m3_decode(c), ref)
    assert oracle.e4m3_decode(np.array([0x7E], np.uint8))[0] == 448.0
    assert oracle.e4m3_decode(np.array([0x01], np.uint8))[0] == 2.0 ** -9


def test_e4m3_encode_matches_library():
    """Nearest-even encoding of in-range values agrees with torch's conversion,
    including every midpoint between neighbouring codes (the ties)."""
    vals = oracle.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    rng = np.random.default_rng(7)
    rnd = np.concatenate([rng.standard_normal(50000) * 30, rng.standard_normal(20000) * 2.0 ** -7,
                          rng.uniform(-448, 448, 20000)]).astype(np.float32)
    t = np.concatenate([mids, -mids, vals.astype(np.float32), rnd])
    t = t[np.abs(t) <= 448]
    ref = torch.from_numpy(t.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(t), ref)


def test_e4m3_ties_saturation_and_signed_zero():
    t = np.array([1.0625, 1.1875, 448.5, 1000.0, -1000.0, 2.0 ** -10, 3 * 2.0 ** -10, -2.0 ** -11, 0.0, -0.0],
                 np.float32)
    want = [0x38,  # tie between 1.0 (m=0) and 1.125 (m=1): even code
            0x3A,  # tie between 1.125 and 1.25: 1.25 (m=2)
            0x7E, 0x7E, 0xFE,  # saturation to +-448
            0x00,  # tie between 0 and 2^-9: even code 0
            0x02,  # tie between 2^-9 (code 1) and 2^-8 (code 2): code 2
            0x80,  # negative value rounding to zero keeps its sign
            0x00, 0x80]
    assert list(oracle.e4m3_encode(t)) == want


def _fp8_case(M=48, K=512, nO=24, seed=3):
    O = workloads.outlier_channels(K, nO, seed=seed)
    X = workloads.activations(M, K, O, seed=seed + 1)
    return O.numpy(), workloads.bf16_bits(X)


def test_fp8_quantizer_invariants():
    O, Xb = _fp8_case()
    K = Xb.shape[1]
    q, s, xo = oracle.quantize_rows_fp8(Xb, K, O)
    normal = np.setdiff1d(np.arange(K), O)
    x = (Xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)[:, normal]
    d = oracle.e4m3_decode(q).reshape(q.shape)
    # the absolute-maximum element of each row lands on +-448 exactly
    am = np.argmax(np.abs(x), axis=1)
    assert np.all(np.abs(d[np.arange(len(am)), am]) == 448.0)
    assert np.all(np.abs(d) <= 448.0)
    # error of a 3-bit mantissa: half an ulp relative (normals), 2^-10 s absolute (subnormals)
    err = np.abs(d * s[:, None].astype(np.float64) - x)
    assert np.all(err <= 2.0 ** -4 * np.abs(x) * (1 + 2.0 ** -20) + 2.0 ** -10 * s[:, None] * (1 + 2.0 ** -20))
    # outliers are exact bit copies
    assert np.array_equal(xo, Xb[:, O])


@pytest.mark.parametrize("e", [-20, -3, 5, 30])
def test_fp8_power_of_two_scaling(e):
    O, Xb = _fp8_case(seed=5)
    K = Xb.shape[1]
    x = (Xb.astype(np.uint32) << 16).view(np.float32) * np.float32(2.0 ** e)
    Xe = (x.view(np.uint32) >> 16).astype(np.uint16)
    q0, s0, _ = oracle.quantize_rows_fp8(Xb, K, O)
    q1, s1, _ = oracle.quantize_rows_fp8(Xe, K, O)
    assert np.array_equal(q0, q1)
    assert np.array_equal(s1, (s0 * np.float32(2.0 ** e)).astype(np.float32))


def test_fp8_sign_symmetry():
    O, Xb = _fp8_case(seed=9)
    K = Xb.shape[1]
    q0, s0, _ = oracle.quantize_rows_fp8(Xb, K, O)
    q1, s1, _ = oracle.quantize_rows_fp8(Xb ^ np.uint16(0x8000), K, O)
    assert np.array_equal(s0, s1)
    assert np.array_equal(q1, q0 ^ np.uint8(0x80))


def test_fp8_products_exact_rational():
    """acc_8 equals the exact rational sum of decoded products (small K: exact in fp64)."""
    O, Xb = _fp8_case(M=6, K=256, nO=8, seed=11)
    Wb = workloads.bf16_bits(workloads.weights(5, 256, seed=12))
    ref = oracle.linear_fp8(Xb, Wb, O)
    for m in range(6):
        for n in range(5):
            exact = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in
                        zip(oracle.e4m3_decode(ref["qx"][m]), oracle.e4m3_decode(ref["qw"][n])))
            assert Fraction(ref["acc_8"][m, n]) == exact


def test_fp8_reductions():
    """nO = 0: a plain FP8 GEMM (numpy matmul of the decoded codes); nO = K: a plain bf16 GEMM."""
    M, K, N = 32, 384, 40
    X = workloads.activations(M, K, workloads.outlier_channels(K, 0, seed=1), seed=2)
    W = workloads.weights(N, K, seed=3)
    Xb, Wb = workloads.bf16_bits(X), workloads.bf16_bits(W)
    r0 = oracle.linear_fp8(Xb, Wb, np.zeros(0, np.int32))
    dx = oracle.e4m3_decode(r0["qx"]).reshape(r0["qx"].shape)
    dw = oracle.e4m3_decode(r0["qw"]).reshape(r0["qw"].shape)
    y0 = (dx @ dw.T) * r0["sx"][:, None].astype(np.float64) * r0["sw"][None, :].astype(np.float64)
    assert np.allclose(r0["y"], y0, rtol=1e-12, atol=1e-12)
    rK = oracle.linear_fp8(Xb, Wb, np.arange(K, dtype=np.int32))
    xf = (Xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    wf = (Wb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.allclose(rK["y"], xf @ wf.T, rtol=1e-12, atol=1e-12)
    assert np.all(rK["sx"] == 0) and rK["qx"].shape == (M, 0)


def test_fp8_path_tracks_the_exact_product():
    """Method sanity (information): on a down-projection-like input (products of
    two Gaussians, outlier channels x40) the FP8 low path with the outlier
    branch stays within a few percent of the exact X W^T, closer than INT4."""
    w = workloads.Workload("t", 64, 1024, 96, 128, x_kind="swiglu", sigma=40.0)
    O, X, W = workloads.make(w)
    Xb, Wb = workloads.bf16_bits(X), workloads.bf16_bits(W)
    exact = (Xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64) @ \
        (Wb.astype(np.uint32) << 16).view(np.float32).astype(np.float64).T
    e8 = np.linalg.norm(oracle.linear_fp8(Xb, Wb, O.numpy())["y"] - exact) / np.linalg.norm(exact)
    e4 = np.linalg.norm(oracle.linear(Xb, Wb, O.numpy())["y"] - exact) / np.linalg.norm(exact)
    assert e8 < 0.05 and e8 < e4


# ----------------------------------------------------------------- static outlier selection (write-up §5, §9; OSC)
def _bf(t):
    return workloads.bf16_bits(t.to(torch.bfloat16))


def _f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _sel_case(Mc=300, K=256, N=96, seed=0):
    g = torch.Generator().manual_seed(seed)
    X = torch.randn(Mc, K, generator=g)
    W = torch.randn(N, K, generator=g) / 16
    return X, W


def test_selection_scores_match_library():
    """score = mean |X| per column x L2 norm of the weight column (numpy, another summation order)."""
    X, W = _sel_case(Mc=2500, N=1100)
    Xb, Wb = _bf(X), _bf(W)
    O, sc = oracle.select_outliers(Xb, Wb, 16)
    ref = np.mean(np.abs(_f64(Xb)), axis=0) * np.linalg.norm(_f64(Wb), axis=0)
    assert np.allclose(sc, ref, rtol=1e-13, atol=0)
    want = np.sort(np.argsort(-ref, kind="stable")[:16])
    assert np.array_equal(O, want.astype(np.int32))


def test_selection_scores_within_the_bound_of_the_exact_score():
    """Against exact rationals: S1 = sum |x| and S2 = sum w^2 over each column, summed
    exactly; score = (S1 / Mc) * sqrt(S2) evaluated to 40 digits.  fp64 sums of n
    nonnegative terms are within (n-1)*2^-53 of the exact sum, relative; the square
    root halves that, and the division, root and product add one rounding each."""
    from decimal import Decimal, getcontext
    from fractions import Fraction
    getcontext().prec = 40
    X, W = _sel_case(Mc=97, K=24, N=53, seed=12)
    X[5] *= 2.0 ** 30        # rows of very different size: the sums round
    X[6] *= 2.0 ** -30
    W[7] *= 2.0 ** 20
    Xb, Wb = _bf(X), _bf(W)
    _, sc = oracle.select_outliers(Xb, Wb, 4)
    xf, wf = _f64(Xb), _f64(Wb)
    Mc, N = xf.shape[0], wf.shape[0]
    bound = ((Mc - 1) + (N - 1) / 2 + 4) * 2.0 ** -53
    for k in range(xf.shape[1]):
        s1 = sum((Fraction(abs(float(v))) for v in xf[:, k]), Fraction(0))
        s2 = sum((Fraction(float(v)) ** 2 for v in wf[:, k]), Fraction(0))
        exact = (Decimal(s1.numerator) / Decimal(s1.denominator) / Mc) * \
            (Decimal(s2.numerator) / Decimal(s2.denominator)).sqrt()
        rel = abs(Decimal(float(sc[k])) - exact) / exact
        assert rel <= Decimal(bound), (k, float(rel), bound)


def test_selection_finds_planted_channels():
    """Channels amplified in the calibration activations, or whose weight column is
    large, are selected; a large weight column with tiny activations is not."""
    X, W = _sel_case(K=128, seed=1)
    X[:, [7, 30, 101]] *= 40.0
    W[:, 64] *= 50.0           # large weights, ordinary activations: contribution x50
    W[:, 90] *= 50.0
    X[:, 90] *= 1e-4           # ...but no activation: contribution tiny
    O, _ = oracle.select_outliers(_bf(X), _bf(W), 4)
    assert list(O) == [7, 30, 64, 101]


def test_selection_ties_go_to_the_lower_index():
    X, W = _sel_case(K=32, seed=2)
    for c in (3, 9, 20):       # three identical, dominant columns
        X[:, c] = X[:, 0] * 30.0
        W[:, c] = W[:, 0]
    O, sc = oracle.select_outliers(_bf(X), _bf(W), 2)
    assert sc[3] == sc[9] == sc[20]
    assert list(O) == [3, 9]


def test_selection_group_aligned():
    """Groups of G consecutive channels ranked by summed score; whole groups selected."""
    X, W = _sel_case(K=256, seed=3)
    X[:, 70] *= 50.0           # group 70 // 8 = 8
    X[:, 200:203] *= 12.0      # group 25
    Xb, Wb = _bf(X), _bf(W)
    O, sc = oracle.select_outliers(Xb, Wb, 16, group=8)
    gs = sc.reshape(-1, 8).sum(axis=1)
    top = np.sort(np.argsort(-gs, kind="stable")[:2])
    assert list(top) == [8, 25]
    assert np.array_equal(O, np.concatenate([np.arange(64, 72), np.arange(200, 208)]).astype(np.int32))
    with pytest.raises(ValueError):
        oracle.select_outliers(Xb, Wb, 12, group=8)


def test_selection_permutation_and_scaling_invariance():
    X, W = _sel_case(K=192, seed=4)
    Xb, Wb = _bf(X), _bf(W)
    O, sc = oracle.select_outliers(Xb, Wb, 24)
    perm = np.random.default_rng(5).permutation(192)
    Op, scp = oracle.select_outliers(Xb[:, perm], Wb[:, perm], 24)
    assert np.array_equal(scp, sc[perm])
    assert np.array_equal(np.sort(perm[Op]), O)
    # a power-of-two scale of X scales every score exactly and keeps the selection
    O2, sc2 = oracle.select_outliers(_bf(X * 4.0), Wb, 24)
    assert np.array_equal(sc2, 4.0 * sc) and np.array_equal(O2, O)


def test_selection_edge_cases():
    X, W = _sel_case(K=64, seed=6)
    Xb, Wb = _bf(X), _bf(W)
    O, _ = oracle.select_outliers(Xb, Wb, 0)
    assert O.size == 0
    O, _ = oracle.select_outliers(Xb, Wb, 64)
    assert np.array_equal(O, np.arange(64, dtype=np.int32))
