"""GPU parity: the CUDA path against the CPU oracle, element by element.

Integer, byte and index outputs (packed codes, scales, compact outlier
tensors, channel table, int32 accumulators) must be bit-exact.  The 16-bit
branch accumulator must match the fp64 oracle within fp32 summation error,
and Y within |dY| <= 1e-2 * max(|Y_ref|, rms(Y_ref)) elementwise.
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


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().float().numpy().astype(np.float64)


def check_y(Y_gpu: np.ndarray, y_ref: np.ndarray):
    rms = float(np.sqrt(np.mean(y_ref ** 2))) if y_ref.size else 0.0
    bound = Y_TOL * np.maximum(np.abs(y_ref), rms)
    err = np.abs(Y_gpu - y_ref)
    bad = err > bound
    assert not bad.any(), (f"{int(bad.sum())} of {bad.size} Y entries out of tolerance; "
                           f"worst ratio {float((err / np.maximum(bound, 1e-300)).max()):.3g}")


def check_quant(O, Xc: torch.Tensor, X_N, s_x, X_O, K, rows=None):
    """Bit-exact check of the quantize-and-gather outputs for all (or the given) rows."""
    Xb = workloads.bf16_bits(Xc)
    sel = np.arange(Xb.shape[0]) if rows is None else np.asarray(rows)
    codes, scale, outl = oracle.quantize_rows(Xb[sel], K, O)
    nO = len(O)
    kn_pad, no_pad = sq.sq_kn_pad(K, nO), sq.sq_no_pad(nO)
    packed = oracle.pack_int4(codes, kn_pad // 2)
    got_n = X_N.cpu().numpy()[sel] if kn_pad else np.zeros((len(sel), 0), np.uint8)
    assert np.array_equal(got_n, packed), "packed INT4 codes differ"
    got_s = s_x.cpu().numpy()[sel]
    assert np.array_equal(got_s.view(np.uint32), scale.view(np.uint32)), "scales differ"
    if nO:
        got_o = bits(X_O)[sel]
        assert np.array_equal(got_o[:, :nO], outl), "compact outlier tensor differs"
        assert np.all(got_o[:, nO:] == 0), "outlier padding not zero"


def run_gpu(O, X: torch.Tensor, W: torch.Tensor, ldy_extra: int = 0):
    dev = torch.device("cuda")
    pw = sq.prepare_weights(W.to(dev), O)
    Xd = X.to(dev)
    X_N, s_x, X_O = sq.quant_gather(Xd, pw)
    M, N = X.shape[0], W.shape[0]
    guard = torch.full((M + 1, N + ldy_extra), -1024.0, dtype=torch.bfloat16, device=dev)
    Y = guard[:M, :N]
    _, dbg_i, dbg_f = sq.gemm(X_N, s_x, X_O, pw, Y=Y, debug=True)
    torch.cuda.synchronize()
    sq.sq_check()
    g = guard.float().cpu()
    assert torch.all(g[M] == -1024.0) and torch.all(g[:, N:] == -1024.0), "write outside Y"
    return pw, (X_N, s_x, X_O), Y, dbg_i, dbg_f


def check_layer(O, X, W, rows=None, ldy_extra=0):
    K = X.shape[1]
    O = np.asarray(O, dtype=np.int32)
    pw, (X_N, s_x, X_O), Y, dbg_i, dbg_f = run_gpu(O, X, W, ldy_extra)
    # offline artefacts
    assert np.array_equal(pw.chan_tab.cpu().numpy().view(np.uint32), oracle.chan_table(O, K))
    check_quant(O, W, pw.W_N, pw.s_w, pw.W_O, K)
    # online quantize-and-gather: every row
    check_quant(O, X, X_N, s_x, X_O, K)
    # products on the selected rows
    Xb, Wb = workloads.bf16_bits(X), workloads.bf16_bits(W)
    sel = np.arange(X.shape[0]) if rows is None else np.asarray(rows)
    ref = oracle.linear(Xb, Wb, O, rows=sel)
    assert np.array_equal(dbg_i.cpu().numpy()[sel].astype(np.int64), ref["acc_i"]), "int32 accumulators differ"
    nO = len(O)
    if nO:
        xo = ref["xo"].astype(np.uint32) << 16
        wo = ref["wo"].astype(np.uint32) << 16
        absum = np.abs(xo.view(np.float32).astype(np.float64)) @ np.abs(wo.view(np.float32).astype(np.float64)).T
        err = np.abs(dbg_f.cpu().numpy()[sel].astype(np.float64) - ref["acc_o"])
        assert np.all(err <= 2.0 ** -20 * absum + 1e-30), "16-bit branch accumulator off"
    else:
        assert np.all(dbg_f.cpu().numpy()[sel] == 0)
    check_y(bf16_to_f64(Y)[sel], ref["y"])
    return Y


# ----------------------------------------------------------------- small shapes
def test_tiny_config_full():
    w = workloads.TINY
    O, X, W = workloads.make(w)
    check_layer(O.numpy(), X, W, ldy_extra=8)


EDGE = [
    # (M, K, N, nO)
    (1, 256, 64, 8),
    (17, 512, 128, 1),
    (127, 384, 192, 0),
    (128, 256, 256, 256),     # every channel an outlier: plain bf16 GEMM
    (129, 1024, 320, 64),
    (300, 200, 136, 3),       # K - nO odd, N not a multiple of 64
    (64, 1024, 512, 1000),    # K - nO = 24 < one block
    (257, 2048, 264, 128),
]


@pytest.mark.parametrize("M,K,N,nO", EDGE, ids=lambda v: str(v))
def test_edge_shapes(M, K, N, nO):
    O = workloads.outlier_channels(K, nO, seed=M + K)
    X = workloads.activations(M, K, O, seed=M)
    W = workloads.weights(N, K, seed=N)
    check_layer(O.numpy(), X, W, ldy_extra=16)


# Shapes that take the CTA-pair kernel (256 x 256 tiles over two SMs): ragged
# M and N, more outlier blocks than ring slots, and both degenerate outlier sets.
PAIR_EDGE = [
    # (M, K, N, nO)
    (1000, 768, 4872, 200),
    (520, 2048, 9480, 1500),
    (512, 256, 9728, 256),
    (768, 512, 6400, 0),
]


@pytest.mark.parametrize("M,K,N,nO", PAIR_EDGE, ids=lambda v: str(v))
def test_pair_kernel_edge_shapes(M, K, N, nO):
    O = workloads.outlier_channels(K, nO, seed=M + K + 1)
    X = workloads.activations(M, K, O, seed=M + 1)
    W = workloads.weights(N, K, seed=N + 1)
    rows = np.unique(np.concatenate([sampled_rows(M, 40), np.arange(248, 264), np.arange(M - 8, M)]))
    check_layer(O.numpy(), X, W, rows=rows, ldy_extra=8)


# Shapes that take the swapped-operand split-K kernel (M <= 128): every token
# width class (16, 32, 64, 128), K split over clusters of 2..8 CTAs, ragged N,
# a single K-block, and both degenerate outlier sets.
SKINNY_EDGE = [
    # (M, K, N, nO)
    (16, 8192, 8192, 4096),
    (5, 4096, 1040, 100),
    (2, 64, 16, 0),
    (32, 1024, 384, 0),
    (33, 2048, 640, 2048),
    (100, 3072, 2176, 320),
    (128, 14336, 4096, 1792),
]


@pytest.mark.parametrize("M,K,N,nO", SKINNY_EDGE, ids=lambda v: str(v))
def test_skinny_kernel_edge_shapes(M, K, N, nO):
    O = workloads.outlier_channels(K, nO, seed=M + K + 2)
    X = workloads.activations(M, K, O, seed=M + 2)
    W = workloads.weights(N, K, seed=N + 2)
    rows = None if M * N * K <= 2 ** 31 else np.unique(np.concatenate([sampled_rows(M, 24), [M - 1]]))
    check_layer(O.numpy(), X, W, rows=rows, ldy_extra=8)


# Rows wider than 16384 channels take the register-resident quantizer (a group
# of 16 warps per row); narrower rows are streamed through shared memory.
WIDE_K = [
    # (M, K, N, nO)
    (40, 20480, 256, 300),
    (24, 40960, 128, 5000),
]


@pytest.mark.parametrize("M,K,N,nO", WIDE_K, ids=lambda v: str(v))
def test_wide_rows(M, K, N, nO):
    O = workloads.outlier_channels(K, nO, seed=K + 5)
    X = workloads.activations(M, K, O, seed=M + 5)
    W = workloads.weights(N, K, seed=N + 5)
    check_layer(O.numpy(), X, W, ldy_extra=8)


def test_zero_rows_and_ties():
    M, K, N, nO = 40, 512, 128, 16
    O = workloads.outlier_channels(K, nO, seed=3)
    X = workloads.activations(M, K, O, seed=4).float()
    X[0] = 0.0                                   # zero row
    X[1, :] = 0.0
    X[1, O.long()] = 5.0                         # zero normal part, nonzero outliers
    normal = torch.tensor(np.setdiff1d(np.arange(K), O.numpy()))
    # ties: a = 7 -> s = 1, entries on half-integers
    X[2, normal] = torch.tensor(np.resize([0.5, 1.5, 2.5, -3.5, 7.0, -6.5], normal.numel()), dtype=torch.float32)
    X[3, normal] = X[2, normal] * 0.125
    W = workloads.weights(N, K, seed=5).float()
    W[7] = 0.0
    check_layer(O.numpy(), X.to(torch.bfloat16), W.to(torch.bfloat16))


def test_tiny_and_huge_row_scales():
    """Rows scaled by powers of two from the bf16 subnormal range (scale below
    2^-100: the quantizer's prescaled path) up to 2^100: codes and scales
    bit-exact, and Y within tolerance."""
    exps = [-140, -136, -133, -130, -127, -124, -120, -112, -104, -100, -96, -60, 0, 40, 80, 100]
    M, K, N, nO = len(exps) * 2, 1024, 128, 40
    O = workloads.outlier_channels(K, nO, seed=11)
    X = workloads.activations(M, K, O, seed=12).float()
    for i, e in enumerate(exps):
        X[2 * i] *= 2.0 ** e
        X[2 * i + 1] *= 2.0 ** e
        X[2 * i + 1, O.long()] = 1.0     # outliers of ordinary size beside a tiny or huge normal part
    W = workloads.weights(N, K, seed=13).float()
    W[3] *= 2.0 ** -120
    W[4] *= 2.0 ** -133
    check_layer(O.numpy(), X.to(torch.bfloat16), W.to(torch.bfloat16))


def test_linear_matches_two_calls_and_is_deterministic():
    w = workloads.Workload("t", 333, 1024, 384, 64)
    O, X, W = workloads.make(w)
    dev = torch.device("cuda")
    layer = sq.SQLinear(W.to(dev), O)
    Xd = X.to(dev)
    y1 = layer(Xd)
    y2 = layer(Xd)
    X_N, s_x, X_O = sq.quant_gather(Xd, layer.weights)
    y3 = sq.gemm(X_N, s_x, X_O, layer.weights)
    torch.cuda.synchronize()
    sq.sq_check()
    assert torch.equal(bits_t(y1), bits_t(y2))
    assert torch.equal(bits_t(y1), bits_t(y3))


def bits_t(t):
    return t.view(torch.int16)


# ----------------------------------------------------------------- full-size workloads
def sampled_rows(M, n=64, seed=123):
    rng = np.random.default_rng(seed)
    rows = rng.choice(M, size=min(n, M), replace=False)
    return np.sort(np.concatenate([rows, [0, M - 1]]).astype(np.int64))


# The full-size configurations and every sweep point are checked through
# sq_linear in test_gpu_linear.py.


# ----------------------------------------------------------------- failure detection
def test_watchdog_times_out_cleanly_and_context_survives():
    sq.sq_selftest_watchdog(50)
    with pytest.raises(sq.SQError) as ei:
        sq.sq_check()
    assert ei.value.status == sq.SQ_ERR_TIMEOUT
    sq.sq_check()  # the error word was cleared
    w = workloads.Workload("t", 64, 256, 64, 8)
    O, X, W = workloads.make(w)
    check_layer(O.numpy(), X, W)


def test_misaligned_device_pointer_rejected():
    dev = torch.device("cuda")
    w = workloads.Workload("t", 8, 256, 64, 8)
    O, X, W = workloads.make(w)
    pw = sq.prepare_weights(W.to(dev), O)
    buf = torch.zeros(8 * 256 + 8, dtype=torch.bfloat16, device=dev)
    Xmis = buf[4:4 + 8 * 256].view(8, 256)
    X_N = torch.empty(8, 128, dtype=torch.uint8, device=dev)
    s_x = torch.empty(8, dtype=torch.float32, device=dev)
    X_O = torch.empty(8, 64, dtype=torch.bfloat16, device=dev)
    with pytest.raises(sq.SQError) as ei:
        sq.sq_quant_gather(Xmis, pw.chan_tab, 8, X_N, s_x, X_O)
    assert ei.value.status == sq.SQ_ERR_MISALIGNED
