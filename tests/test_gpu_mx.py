"""GPU parity of the micro-scaling FP4 (MXFP4) low path against the CPU oracle.

Packed E2M1 codes, the tiled E8M0 block scales, the compact outlier tensor
and the channel table must be bit-exact.  The GEMM accumulates the
block-scaled E2M1 products (tcgen05 kind::mxf4, scales applied by the tensor
core) and the bf16 branch into one fp32 accumulator, compared with the
oracle's exact fp64 sums within 2^-12 of the sum of absolute products; Y
within |dY| <= 1e-2 * max(|Y_ref|, rms(Y_ref)) elementwise.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads
import mixed_precision_gemm_b200 as sq

pytestmark = pytest.mark.gpu

Y_TOL = 1e-2
ACC_REL = 2.0 ** -12
E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def dequant_abs(codes: np.ndarray, e8: np.ndarray) -> np.ndarray:
    """|code value| * 2^E, float32 (exact: E2M1 magnitudes times a power of two in range); only bounds use it."""
    R, KN = codes.shape
    return E2M1.astype(np.float32)[codes & 7] * np.exp2(
        np.repeat(e8.astype(np.float32) - 127, 32, axis=1)[:, :KN])


def check_quant_mx(O, src: torch.Tensor, codes_dev, S_dev, XO_dev, K):
    rows = src.shape[0]
    codes, e8, outl = oracle.quantize_rows_mx(workloads.bf16_bits(src), K, O)
    kn_pad = sq.sq_kn_pad_mx(K, len(O))
    got = codes_dev.cpu().numpy()
    want = oracle.pack_fp4(codes, kn_pad // 2)
    assert got.shape == want.shape
    bad = got != want
    assert not bad.any(), f"E2M1 bytes differ in {int(bad.sum())} places (first at {np.argwhere(bad)[0]})"
    if kn_pad:
        nbytes = sq.sq_mx_scale_bytes(rows, K, len(O))
        want_s = oracle.mx_scale_tiles(e8, (rows + 127) // 128 * 128, kn_pad // 32)
        got_s = S_dev.cpu().numpy()[:nbytes]
        assert got_s.size == want_s.size
        bad = got_s != want_s
        assert not bad.any(), f"block scales differ in {int(bad.sum())} places"
    if len(O):
        go = bits(XO_dev)
        assert np.array_equal(go[:, :len(O)], outl), "compact outlier tensor differs"
        assert np.all(go[:, len(O):] == 0), "outlier padding not zero"
    return codes, e8


def check_layer_mx(O, X, W, rows=None, ldy_extra=0):
    O = np.asarray(O, dtype=np.int32)
    K = X.shape[1]
    M, N = X.shape[0], W.shape[0]
    dev = torch.device("cuda")
    pw = sq.prepare_weights(W.to(dev), O, mx=True)
    X_N4, S_X, X_O = sq.quant_gather(X.to(dev), pw)
    guard = torch.full((M + 1, N + ldy_extra), -1024.0, dtype=torch.bfloat16, device=dev)
    Y = guard[:M, :N]
    _, _, acc = sq.gemm(X_N4, S_X, X_O, pw, Y=Y, debug=True)
    torch.cuda.synchronize()
    sq.sq_check()
    g = guard.float().cpu()
    assert torch.all(g[M] == -1024.0) and torch.all(g[:, N:] == -1024.0), "write outside Y"

    assert np.array_equal(pw.chan_tab.cpu().numpy().view(np.uint32), oracle.chan_table(O, K))
    check_quant_mx(O, W, pw.W_N, pw.s_w, pw.W_O, K)
    check_quant_mx(O, X, X_N4, S_X, X_O, K)

    Xb, Wb = workloads.bf16_bits(X), workloads.bf16_bits(W)
    sel = np.arange(M) if rows is None else np.asarray(rows)
    ref = oracle.linear_mx(Xb, Wb, O, rows=sel)
    absum = (dequant_abs(ref["qx"], ref["ex"]) @ dequant_abs(ref["qw"], ref["ew"]).T).astype(np.float64)
    if len(O):
        xo = (ref["xo"].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        wo = (ref["wo"].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        absum = absum + np.abs(xo) @ np.abs(wo).T
    err = np.abs(acc.cpu().numpy()[sel].astype(np.float64) - (ref["acc_mx"] + ref["acc_o"]))
    assert np.all(err <= ACC_REL * absum + 1e-30), \
        f"accumulator off: worst {float((err / np.maximum(absum, 1e-300)).max()):.3g} of sum|products|"
    y = Y.float().cpu().numpy().astype(np.float64)[sel]
    yr = ref["y"]
    rms = float(np.sqrt(np.mean(yr ** 2))) if yr.size else 0.0
    bad = np.abs(y - yr) > Y_TOL * np.maximum(np.abs(yr), rms)
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} Y entries out of tolerance"


def sampled_rows(M, n=24, seed=321):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([rng.choice(M, size=min(n, M), replace=False), [0, M - 1]]))


SHAPES = [
    # (M, K, N, nO): several tiles with ragged tails, partial scale blocks, tiny M
    (300, 1024, 520, 40),
    (1000, 2048, 1288, 0),
    (520, 768, 264, 768),        # every channel an outlier: plain bf16 GEMM
    (257, 1040, 392, 24),        # K - nO = 1016: partial last block, kn_pad_mx = 1024
    (16, 4096, 2048, 256),
    (5, 1024, 136, 3),
    (40, 2048, 384, 0),
    (100, 3072, 1152, 320),
    (128, 14336, 512, 1792),
    # few tokens: the split-K kernel (one W tile -> 8 K ranges crossing the E2M1 / bf16 boundary)
    (16, 4096, 128, 256),
    (64, 8192, 256, 512),
    (1, 1024, 64, 8),
    (33, 2048, 1032, 0),
    # 632 pair tiles on 74 clusters (several tiles per cluster: the accumulator handed back before
    # Y is stored, the scale slots reused across tiles), ragged last M and N tiles
    (1800, 1024, 20000, 64),
]


@pytest.mark.parametrize("M,K,N,nO", SHAPES, ids=lambda v: str(v))
def test_mx_shapes(M, K, N, nO):
    O = workloads.outlier_channels(K, nO, seed=M + K + 11)
    X = workloads.activations(M, K, O, kind="gauss", sigma=30.0, seed=M + 11)
    W = workloads.weights(N, K, seed=N + 11)
    rows = None if M * N * K <= 2 ** 31 else sampled_rows(M)
    check_layer_mx(O.numpy(), X, W, rows=rows, ldy_extra=8)


def test_mx_ties_signed_zero_and_zero_blocks():
    """Entries exactly between two E2M1 values at their block's scale, -0 and
    small negatives that round to zero, an all-zero row and all-zero blocks,
    rows whose scale clamps (subnormal and tiny values), and large values."""
    M, K, N, nO = 24, 512, 128, 16
    O = workloads.outlier_channels(K, nO, seed=31)
    X = workloads.activations(M, K, O, seed=32).float()
    normal = torch.tensor(np.setdiff1d(np.arange(K), O.numpy()))
    X[0] = 0.0
    X[1, :] = 0.0
    X[1, O.long()] = 3.0
    # block absmax 6 -> E = 0: the quotients are the values themselves
    ties = [6.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.0, 0.0, -0.1, 4.0, -6.0, 3.0, 0.5]
    X[2, normal] = torch.tensor(np.resize(ties, normal.numel()), dtype=torch.float32)
    X[3, normal] = X[2, normal] * 2.0 ** -40
    X[4, normal] = X[2, normal] * 2.0 ** 60
    X[5, normal[:64]] = 0.0                     # two zero blocks
    X[6, normal] = 2.0 ** -130                  # bf16 subnormals: scale clamps at 2^-127
    X[7, normal] = X[2, normal] * 2.0 ** -120   # scale near the bottom of the range
    W = workloads.weights(N, K, seed=33).float()
    W[5] = 0.0
    check_layer_mx(O.numpy(), X.to(torch.bfloat16), W.to(torch.bfloat16))


def test_mx_decode_sweep_point():
    """M = 16 tokens against an 8192 x 8192 layer with nO = K/16 (a sweep point), every row."""
    w = workloads.CONFIGS["sweep_M16_o1/16"]
    O, X, W = workloads.make(w)
    check_layer_mx(O.numpy(), X, W)


def test_mx_quant_padded_ld_and_wide_rows():
    """X with a row stride above K, and rows wider than any configuration."""
    dev = torch.device("cuda")
    for M, K, nO, ld in [(130, 2048, 64, 2056), (9, 40960, 512, 40960)]:
        O = workloads.outlier_channels(K, nO, seed=K)
        X = workloads.activations(M, K, O, seed=K + 1)
        Xp = torch.zeros(M, ld, dtype=torch.bfloat16)
        Xp[:, :K] = X
        Xd = Xp.to(dev)[:, :K]
        W = workloads.weights(8, K, seed=K + 2)
        pw = sq.prepare_weights(W.to(dev), O.numpy(), mx=True)
        X_N4, S_X, X_O = sq.quant_gather(Xd, pw)
        torch.cuda.synchronize()
        sq.sq_check()
        check_quant_mx(O.numpy(), X, X_N4, S_X, X_O, K)


def test_mx_linear_matches_two_calls():
    w = workloads.Workload("t", 257, 2048, 640, 96, x_kind="gauss", sigma=30.0)
    O, X, W = workloads.make(w)
    dev = torch.device("cuda")
    layer = sq.SQLinear(W.to(dev), O, mx=True)
    Xd = X.to(dev)
    y1 = layer(Xd)
    X_N4, S_X, X_O = sq.quant_gather(Xd, layer.weights)
    y2 = sq.gemm(X_N4, S_X, X_O, layer.weights)
    torch.cuda.synchronize()
    sq.sq_check()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_mx_argument_errors():
    dev = torch.device("cuda")
    W = torch.zeros(16, 256, dtype=torch.bfloat16, device=dev)
    with pytest.raises(sq.SQError) as e:
        sq.prepare_weights(W, [5, 3], mx=True)
    assert e.value.status == sq.SQ_ERR_INVALID_ARG
    pw = sq.prepare_weights(W, [1, 2], mx=True)
    X = torch.zeros(4, 256, dtype=torch.bfloat16, device=dev)
    X_N4, S_X, X_O = sq.quant_gather(X, pw)
    with pytest.raises(sq.SQError) as e:
        sq.sq_gemm_mx(X_N4, S_X, X_O, pw.W_N, pw.s_w, pw.W_O, 4, 12, 256, 2,
                      torch.zeros(4, 16, dtype=torch.bfloat16, device=dev))
    assert e.value.status == sq.SQ_ERR_INVALID_ARG
