"""sq_linear_noalloc: the layer for callers that cannot allocate a workspace.

Plugins and inference servers that own all device memory through their own
pool (and forbid allocations once running), or latency-bound serving loops
where cudaMalloc/cudaFree would stall the device, cannot lend sq_linear a
workspace.  sq_linear_noalloc keeps that scratch in a fixed array inside the
library instead.  These tests call it through the C ABI and check it against
sq_linear (with a caller workspace) on two calls in a row, with different
inputs, so the second call runs on scratch the first one left behind.  Both
entry points run the same kernels on the same inputs, so Y must agree bit for
bit; one case is also compared with the CPU oracle.

The cases cover the few-token kernel (M = 16), the CTA-pair kernel (M = 512)
and the largest M whose scratch fits the array exactly.

This file is named so that pytest collects it last.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import mixed_precision_gemm_b200 as sq
import oracle
import workloads

LIMIT = 16 * 1024 * 1024     # SQ_NOALLOC_WS_BYTES
Y_TOL = 1e-2                 # the Y tolerance of the parity tests
K, N, nO = 4096, 1024, 256


def largest_m_that_fits() -> int:
    lo, hi = 1, 1 << 20
    while lo < hi:                      # largest M with workspace <= LIMIT
        mid = (lo + hi + 1) // 2
        if sq.sq_linear_workspace_bytes(mid, K, nO) <= LIMIT:
            lo = mid
        else:
            hi = mid - 1
    return lo


@pytest.mark.gpu
@pytest.mark.parametrize("M", [16, 512, "max"])
def test_noalloc_matches_sq_linear_on_two_calls_in_a_row(M):
    dev = torch.device("cuda")
    if M == "max":
        M = largest_m_that_fits()
        assert sq.sq_linear_workspace_bytes(M + 1, K, nO) > LIMIT
    assert sq.sq_linear_workspace_bytes(M, K, nO) <= LIMIT
    O = workloads.outlier_channels(K, nO)
    W = workloads.weights(N, K)
    pw = sq.prepare_weights(W.to(dev), O)
    ws = torch.empty(sq.sq_linear_workspace_bytes(M, K, nO), dtype=torch.uint8, device=dev)
    for seed in (11, 12):
        X = workloads.activations(M, K, O, seed=seed + M)
        Xd = X.to(dev)
        Y_ref = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        sq.sq_linear(Xd, pw.chan_tab, pw.W_N, pw.s_w, pw.W_O, N, nO, Y_ref, ws)
        Y = torch.full((M, N), -1024.0, dtype=torch.bfloat16, device=dev)
        sq.sq_linear_noalloc(Xd, pw.chan_tab, pw.W_N, pw.s_w, pw.W_O, N, nO, Y)
        torch.cuda.synchronize()
        sq.sq_check()
        assert torch.equal(Y.view(torch.int16), Y_ref.view(torch.int16)), "noalloc Y differs from sq_linear's"
    if M == 512:
        # the last call against the oracle on a sample of rows
        rows = np.array([0, 1, 100, 257, 511])
        ref = oracle.linear(workloads.bf16_bits(X), workloads.bf16_bits(W), O.numpy(), rows=rows)
        y = Y[torch.as_tensor(rows, device=dev)].float().cpu().numpy().astype(np.float64)
        rms = float(np.sqrt(np.mean(ref["y"] ** 2)))
        assert np.all(np.abs(y - ref["y"]) <= Y_TOL * np.maximum(np.abs(ref["y"]), rms))


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = sq.load()
    M, K_, nO_ = 65536, 8192, 512
    assert sq.sq_linear_workspace_bytes(M, K_, nO_) > LIMIT
    P = ctypes.c_void_p
    st = lib.sq_linear_noalloc(P(0x1000), M, K_, K_, P(0x2000), P(0x3000), P(0x4000), P(0x5000), 64, nO_,
                               P(0x6000), 64, None)
    assert st == sq.SQ_ERR_UNSUPPORTED
    assert b"scratch" in lib.sq_last_error_detail()
