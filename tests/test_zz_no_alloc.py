"""sq_linear_noalloc: the layer for callers that cannot allocate a workspace.

Plugins and inference servers that own all device memory through their own
pool (and forbid allocations once running), or latency-bound serving loops
where cudaMalloc/cudaFree would stall the device, cannot lend sq_linear a
workspace.  sq_linear_noalloc keeps that scratch in a fixed array inside the
library instead.  These tests call it through the C ABI and check it against
sq_linear (with a caller workspace) on two calls in a row, with different
inputs, so the second call runs on scratch the first one left behind.

This file is named so that pytest collects it last.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import mixed_precision_gemm_b200 as sq
import workloads

Y_TOL = 1e-2  # the Y tolerance of the parity tests


def _within_tolerance(Y: torch.Tensor, Y_ref: torch.Tensor):
    y = Y.float().cpu().numpy().astype(np.float64)
    r = Y_ref.float().cpu().numpy().astype(np.float64)
    rms = float(np.sqrt(np.mean(r ** 2)))
    assert np.all(np.abs(y - r) <= Y_TOL * np.maximum(np.abs(r), rms))


@pytest.mark.gpu
def test_noalloc_matches_sq_linear_on_two_calls_in_a_row():
    dev = torch.device("cuda")
    M, K, N, nO = 512, 4096, 1024, 256
    assert sq.sq_linear_workspace_bytes(M, K, nO) <= 16 * 1024 * 1024
    O = workloads.outlier_channels(K, nO)
    W = workloads.weights(N, K)
    pw = sq.prepare_weights(W.to(dev), O)
    ws = torch.empty(sq.sq_linear_workspace_bytes(M, K, nO), dtype=torch.uint8, device=dev)
    for call, seed in enumerate((11, 12)):
        X = workloads.activations(M, K, O, seed=seed).to(dev)
        Y_ref = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        sq.sq_linear(X, pw.chan_tab, pw.W_N, pw.s_w, pw.W_O, N, nO, Y_ref, ws)
        Y = torch.full((M, N), -1024.0, dtype=torch.bfloat16, device=dev)
        sq.sq_linear_noalloc(X, pw.chan_tab, pw.W_N, pw.s_w, pw.W_O, N, nO, Y)
        torch.cuda.synchronize()
        sq.sq_check()
        _within_tolerance(Y, Y_ref)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = sq.load()
    M, K, nO = 65536, 8192, 512
    assert sq.sq_linear_workspace_bytes(M, K, nO) > 16 * 1024 * 1024
    P = __import__("ctypes").c_void_p
    st = lib.sq_linear_noalloc(P(0x1000), M, K, K, P(0x2000), P(0x3000), P(0x4000), P(0x5000), 64, nO,
                               P(0x6000), 64, None)
    assert st == sq.SQ_ERR_UNSUPPORTED
    assert b"scratch" in lib.sq_last_error_detail()
