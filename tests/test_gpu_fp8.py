"""GPU parity of the FP8 low path (OSC's FP8 fallback for the inputs of W2)
against the CPU oracle.

E4M3 codes, scales, the compact outlier tensor and the channel table must be
bit-exact.  The low-path accumulator is fp32 on the tensor cores (E4M3 x E4M3,
kind::f8f6f4) and is compared with the oracle's exact fp64 sum within
2^-12 of the sum of absolute products; the 16-bit branch as for INT4; Y
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
ACC8_REL = 2.0 ** -12


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def check_quant_fp8(O, Xc: torch.Tensor, X_N8, s_x, X_O, K):
    Xb = workloads.bf16_bits(Xc)
    codes, scale, outl = oracle.quantize_rows_fp8(Xb, K, O)
    KN = K - len(O)
    got = X_N8.cpu().numpy()
    assert np.array_equal(got[:, :KN], codes), \
        f"E4M3 codes differ in {int((got[:, :KN] != codes).sum())} places"
    assert np.all(got[:, KN:] == 0), "code padding not zero"
    assert np.array_equal(s_x.cpu().numpy().view(np.uint32), scale.view(np.uint32)), "scales differ"
    if len(O):
        go = bits(X_O)
        assert np.array_equal(go[:, :len(O)], outl), "compact outlier tensor differs"
        assert np.all(go[:, len(O):] == 0), "outlier padding not zero"


def check_layer_fp8(O, X, W, rows=None, ldy_extra=0):
    O = np.asarray(O, dtype=np.int32)
    K = X.shape[1]
    M, N = X.shape[0], W.shape[0]
    dev = torch.device("cuda")
    pw = sq.prepare_weights(W.to(dev), O, fp8=True)
    X_N8, s_x, X_O = sq.quant_gather(X.to(dev), pw)
    guard = torch.full((M + 1, N + ldy_extra), -1024.0, dtype=torch.bfloat16, device=dev)
    Y = guard[:M, :N]
    _, acc8, accf = sq.gemm(X_N8, s_x, X_O, pw, Y=Y, debug=True)
    torch.cuda.synchronize()
    sq.sq_check()
    g = guard.float().cpu()
    assert torch.all(g[M] == -1024.0) and torch.all(g[:, N:] == -1024.0), "write outside Y"

    assert np.array_equal(pw.chan_tab.cpu().numpy().view(np.uint32), oracle.chan_table(O, K))
    check_quant_fp8(O, W, pw.W_N, pw.s_w, pw.W_O, K)
    check_quant_fp8(O, X, X_N8, s_x, X_O, K)

    Xb, Wb = workloads.bf16_bits(X), workloads.bf16_bits(W)
    sel = np.arange(M) if rows is None else np.asarray(rows)
    ref = oracle.linear_fp8(Xb, Wb, O, rows=sel)
    dx = np.abs(oracle.e4m3_decode(ref["qx"]).reshape(ref["qx"].shape))
    dw = np.abs(oracle.e4m3_decode(ref["qw"]).reshape(ref["qw"].shape))
    absum8 = dx @ dw.T
    err8 = np.abs(acc8.cpu().numpy()[sel].astype(np.float64) - ref["acc_8"])
    assert np.all(err8 <= ACC8_REL * absum8 + 1e-30), \
        f"low-path accumulator off: worst {float((err8 / np.maximum(absum8, 1e-300)).max()):.3g} of sum|products|"
    if len(O):
        xo = (ref["xo"].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        wo = (ref["wo"].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        absum = np.abs(xo) @ np.abs(wo).T
        errf = np.abs(accf.cpu().numpy()[sel].astype(np.float64) - ref["acc_o"])
        assert np.all(errf <= 2.0 ** -20 * absum + 1e-30), "16-bit branch accumulator off"
    y = Y.float().cpu().numpy().astype(np.float64)[sel]
    yr = ref["y"]
    rms = float(np.sqrt(np.mean(yr ** 2))) if yr.size else 0.0
    bad = np.abs(y - yr) > Y_TOL * np.maximum(np.abs(yr), rms)
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} Y entries out of tolerance"


def sampled_rows(M, n=24, seed=321):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([rng.choice(M, size=min(n, M), replace=False), [0, M - 1]]))


SHAPES = [
    # (M, K, N, nO): pair kernel (M > 128) and every skinny token class
    (300, 1024, 520, 40),
    (1000, 2048, 1288, 0),
    (520, 768, 264, 768),        # every channel an outlier: plain bf16 GEMM
    (16, 4096, 2048, 256),
    (5, 1024, 136, 3),
    (40, 2048, 384, 0),
    (100, 3072, 1152, 320),
    (128, 14336, 512, 1792),
]


@pytest.mark.parametrize("M,K,N,nO", SHAPES, ids=lambda v: str(v))
def test_fp8_shapes(M, K, N, nO):
    O = workloads.outlier_channels(K, nO, seed=M + K + 7)
    X = workloads.activations(M, K, O, kind="swiglu", sigma=40.0, seed=M + 7)
    W = workloads.weights(N, K, seed=N + 7)
    rows = None if M * N * K <= 2 ** 31 else sampled_rows(M)
    check_layer_fp8(O.numpy(), X, W, rows=rows, ldy_extra=8)


def test_fp8_ties_signed_zero_and_zero_rows():
    """Quotients exactly between two E4M3 codes (normal and subnormal range),
    negative values that round to -0, a zero row and a row whose normal part is
    zero: codes bit-exact."""
    M, K, N, nO = 24, 512, 128, 16
    O = workloads.outlier_channels(K, nO, seed=21)
    X = workloads.activations(M, K, O, seed=22).float()
    normal = torch.tensor(np.setdiff1d(np.arange(K), O.numpy()))
    X[0] = 0.0
    X[1, :] = 0.0
    X[1, O.long()] = 3.0
    # a = 448 -> s = 1: the quotients are the values themselves
    ties = [448.0, 1.0625, 1.1875, -2.125, 3.25, -13.0, 2.0 ** -10, 3 * 2.0 ** -10, -2.0 ** -11, -2.0 ** -12, 0.0, -0.0]
    X[2, normal] = torch.tensor(np.resize(ties, normal.numel()), dtype=torch.float32)
    X[3, normal] = X[2, normal] * 2.0 ** -40
    W = workloads.weights(N, K, seed=23).float()
    W[5] = 0.0
    check_layer_fp8(O.numpy(), X.to(torch.bfloat16), W.to(torch.bfloat16))


def test_fp8_linear_matches_two_calls():
    w = workloads.Workload("t", 257, 2048, 640, 96, x_kind="swiglu", sigma=40.0)
    O, X, W = workloads.make(w)
    dev = torch.device("cuda")
    layer = sq.SQLinear(W.to(dev), O, fp8=True)
    Xd = X.to(dev)
    y1 = layer(Xd)
    X_N8, s_x, X_O = sq.quant_gather(Xd, layer.weights)
    y2 = sq.gemm(X_N8, s_x, X_O, layer.weights)
    torch.cuda.synchronize()
    sq.sq_check()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_fp8_wide_rows_rejected():
    dev = torch.device("cuda")
    W = torch.zeros(16, 20480, dtype=torch.bfloat16, device=dev)
    with pytest.raises(sq.SQError) as e:
        sq.prepare_weights(W, [1, 2], fp8=True)
    assert e.value.status == sq.SQ_ERR_UNSUPPORTED
