"""GPU parity of the element-level SQ-format path against the CPU oracle.

Bit-exact: the packed INT4 low part with its mask code -8, the row scales,
the 2:4-compressed E4M3 high part and its metadata, the all-zero channel
table, the tokens' INT4 and E4M3 codes and scales, and the exact int32 sums of
the low part.  The high part P (2:4 sparse tensor cores, fp32 accumulation,
then the two scales) is compared with the oracle's fp64 value within 2^-12 of
the sum of absolute products; Y within |dY| <= 1e-2 * max(|Y_ref|, rms(Y_ref)).
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


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def check_sqf(X, W, bank, h, rows=None, ldy_extra=0):
    M, K = X.shape
    N = W.shape[0]
    dev = torch.device("cuda")
    pw = sq.prepare_weights_sqf(W.to(dev), bank, h)
    X_N, s_x4, X_8, s_x8 = sq.quant_gather_sqf(X.to(dev), pw)
    guard = torch.full((M + 1, N + ldy_extra), -1024.0, dtype=torch.bfloat16, device=dev)
    Y = guard[:M, :N]
    _, acc_lo, P = sq.gemm_sqf(X_N, s_x4, X_8, s_x8, pw, Y=Y, debug=True)
    torch.cuda.synchronize()
    sq.sq_check()
    g = guard.float().cpu()
    assert torch.all(g[M] == -1024.0) and torch.all(g[:, N:] == -1024.0), "write outside Y"

    Xb, Wb = workloads.bf16_bits(X), workloads.bf16_bits(W)
    # weights
    w = oracle.sqf_weights(Wb, bank, h)
    assert np.array_equal(pw.W_N.cpu().numpy(), oracle.pack_int4(w["lo"], K // 2)), "low part differs"
    assert np.array_equal(pw.s_lo.cpu().numpy().view(np.uint32), w["s_lo"].view(np.uint32)), "s_lo differs"
    vals, meta = oracle.compress_24(w["hi_mask"], w["hi"])
    assert np.array_equal(pw.W_H.cpu().numpy(), vals), "2:4 high values differ"
    assert np.array_equal(pw.W_E.cpu().numpy(), meta), "2:4 metadata differs"
    assert np.array_equal(pw.s_hi.cpu().numpy().view(np.uint32), w["s_hi"].view(np.uint32)), "s_hi differs"
    assert torch.all(pw.chan_tab == 0)
    # tokens
    none = np.zeros(0, np.int32)
    q4, sx4, _ = oracle.quantize_rows(Xb, K, none)
    q8, sx8, _ = oracle.quantize_rows_fp8(Xb, K, none)
    assert np.array_equal(X_N.cpu().numpy(), oracle.pack_int4(q4, K // 2))
    assert np.array_equal(s_x4.cpu().numpy().view(np.uint32), sx4.view(np.uint32))
    assert np.array_equal(X_8.cpu().numpy(), q8)
    assert np.array_equal(s_x8.cpu().numpy().view(np.uint32), sx8.view(np.uint32))
    # products
    sel = np.arange(M) if rows is None else np.asarray(rows)
    ref = oracle.sqf_linear(Xb, Wb, bank, h, rows=sel)
    assert np.array_equal(acc_lo.cpu().numpy()[sel].astype(np.int64), ref["acc_lo"]), "low-part sums differ"
    # |decoded codes| in float32 (E4M3 values are exact in fp32); only the bound uses them
    e4 = np.abs(oracle.e4m3_decode(np.arange(256, dtype=np.uint8))).astype(np.float32)
    dx = e4[ref["qx8"]]
    dw = np.where(ref["hi_mask"] == 1, e4[ref["hi"]], np.float32(0))
    scale = ref["sx8"][:, None].astype(np.float64) * ref["s_hi"][None, :].astype(np.float64)
    p_ref = ref["acc_hi"] * scale
    bound = ACC_REL * (dx @ dw.T).astype(np.float64) * scale + 2.0 ** -20 * np.abs(p_ref) + 1e-30
    err = np.abs(P.cpu().numpy()[sel].astype(np.float64) - p_ref)
    assert np.all(err <= bound), f"high part off: worst {float((err / bound).max()):.3g} of the bound"
    y = Y.float().cpu().numpy().astype(np.float64)[sel]
    yr = ref["y"]
    rms = float(np.sqrt(np.mean(yr ** 2))) if yr.size else 0.0
    bad = np.abs(y - yr) > Y_TOL * np.maximum(np.abs(yr), rms)
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} Y entries out of tolerance"


SHAPES = [
    # (M, K, N, bank, h): the pair kernel (M > 128) and every split-K token class, both high-part tile
    # sizes; for M <= 128 the high part splits each tile's K stages over two CTAs unless the tiles
    # already fill half of the SMs
    (300, 1024, 520, 8, 2),
    (1000, 2048, 1288, 16, 1),
    (130, 512, 264, 8, 1),
    (16, 4096, 2048, 4, 2),
    (5, 1024, 136, 4, 1),
    (40, 2048, 384, 16, 2),
    (100, 3072, 1152, 4, 2),
    (128, 1024, 512, 16, 1),
    # more W tiles than half the SMs: one CTA per tile (no K split), both token tile sizes
    (16, 1024, 10240, 16, 1),
    (100, 1024, 9728, 8, 2),
]


@pytest.mark.parametrize("M,K,N,bank,h", SHAPES, ids=lambda v: str(v))
def test_sqf_shapes(M, K, N, bank, h):
    O = workloads.outlier_channels(K, K // 32, seed=M + K)
    X = workloads.activations(M, K, O, kind="gauss", sigma=30.0, seed=M + 5)
    W = workloads.weights(N, K, seed=N + 5)
    check_sqf(X, W, bank, h, ldy_extra=8)


def test_sqf_zero_rows_ties_and_large_entries():
    M, K, N = 24, 512, 136
    X = workloads.activations(M, K, workloads.outlier_channels(K, 0), seed=61).float()
    X[0] = 0.0
    X[1, ::3] = 0.0
    W = workloads.weights(N, K, seed=62).float()
    W[0] = 0.0                                   # zero row: both scales 0
    W[1] = 0.5                                   # all ties: the first h of every bank
    W[2, ::16] = 3.0                             # one large entry per bank of 16
    W[3, ::5] = -2.0
    check_sqf(X.to(torch.bfloat16), W.to(torch.bfloat16), 16, 2)


def test_sqf_qkv_sampled():
    """Llama-3-8B QKV shape (2048 x 4096 x 6144), banks of 16 with one high entry, sampled rows."""
    w = workloads.LLAMA8B_QKV
    X = workloads.activations(w.M, w.K, workloads.outlier_channels(w.K, w.nO), seed=71)
    W = workloads.weights(w.N, w.K, seed=72)
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([rng.choice(w.M, 12, replace=False), [0, w.M - 1]]))
    check_sqf(X, W, 16, 1, rows=rows)


def test_sqf_many_tiles_per_cluster():
    """632 high-part pair tiles on 74 clusters (the persistent kernel walks several tiles per
    cluster, its staging ring and accumulator hand-back running across them), ragged last M and
    N tiles; sampled rows, including the last."""
    M, K, N = 1800, 1024, 20000
    X = workloads.activations(M, K, workloads.outlier_channels(K, 0), seed=91)
    W = workloads.weights(N, K, seed=92)
    rng = np.random.default_rng(9)
    rows = np.unique(np.concatenate([rng.choice(M, 10, replace=False), [0, 255, 256, 1791, M - 1]]))
    check_sqf(X, W, 16, 1, rows=rows)


def test_sqf_linear_matches_calls():
    M, K, N = 257, 1024, 392
    X = workloads.activations(M, K, workloads.outlier_channels(K, 0), seed=81).to("cuda")
    W = workloads.weights(N, K, seed=82).to("cuda")
    pw = sq.prepare_weights_sqf(W, 8, 2)
    Y1 = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(sq.sq_linear_workspace_bytes_sqf(M, N, K), dtype=torch.uint8, device="cuda")
    sq.sq_linear_sqf(X, pw.chan_tab, pw.W_N, pw.s_lo, pw.W_H, pw.W_E, pw.s_hi, N, Y1, ws)
    Y2 = sq.gemm_sqf(*sq.quant_gather_sqf(X, pw), pw)
    torch.cuda.synchronize()
    sq.sq_check()
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))


def test_sqf_argument_errors():
    dev = torch.device("cuda")
    W = torch.zeros(16, 512, dtype=torch.bfloat16, device=dev)
    for bank, h in [(3, 1), (8, 3), (32, 1)]:
        with pytest.raises(sq.SQError) as e:
            sq.prepare_weights_sqf(W, bank, h)
        assert e.value.status == sq.SQ_ERR_INVALID_ARG
    with pytest.raises(sq.SQError) as e:
        sq.prepare_weights_sqf(torch.zeros(16, 384, dtype=torch.bfloat16, device=dev), 8, 1)
    assert e.value.status == sq.SQ_ERR_INVALID_ARG


@pytest.mark.parametrize("name,bank,h", [("llama3_8b_down_4096x14336x4096_o1792", 8, 2),
                                         ("llama3_70b_gateup_8192x8192x57344_o512", 16, 1),
                                         ("sweep_M8192_o0", 4, 1)])
def test_sqf_full_size_sampled(name, bank, h):
    """Full-size configurations with element-level SQ-format weights, sampled GEMM rows."""
    w = workloads.CONFIGS[name]
    X = workloads.activations(w.M, w.K, workloads.outlier_channels(w.K, w.nO), kind=w.x_kind, sigma=w.sigma, seed=91)
    W = workloads.weights(w.N, w.K, seed=92)
    rng = np.random.default_rng(7)
    rows = np.unique(np.concatenate([rng.choice(w.M, 6, replace=False), [0, w.M - 1]]))
    check_sqf(X, W, bank, h, rows=rows)
