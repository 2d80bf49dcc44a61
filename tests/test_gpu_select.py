"""GPU parity of the static outlier-channel selection against the CPU oracle:
the selected channel list and the per-channel fp64 scores are bit-exact (the
score's summation order is part of its definition)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads
import mixed_precision_gemm_b200 as sq

pytestmark = pytest.mark.gpu


def run(X, W, nO, group=1):
    dev = torch.device("cuda")
    O, sc = sq.select_outliers(X.to(dev), W.to(dev), nO, group)
    torch.cuda.synchronize()
    sq.sq_check()
    O_ref, sc_ref = oracle.select_outliers(workloads.bf16_bits(X), workloads.bf16_bits(W), nO, group)
    assert np.array_equal(sc.cpu().numpy().view(np.uint64), sc_ref.view(np.uint64)), "scores differ"
    assert np.array_equal(O.cpu().numpy(), O_ref), "selected channels differ"
    return O_ref


@pytest.mark.parametrize("Mc,K,N,nO,group", [
    (300, 256, 96, 16, 1),
    (2500, 1024, 1100, 64, 1),      # several 256-row blocks on both sides
    (512, 4096, 6144, 256, 1),      # Llama-3-8B QKV weights, 512 calibration tokens
    (512, 14336, 1024, 1792, 8),    # down-projection width, group-aligned
    (64, 8192, 2048, 512, 64),
    (100, 200, 40, 0, 1),
    (100, 200, 40, 200, 4),
])
def test_selection_matches_oracle(Mc, K, N, nO, group):
    O = workloads.outlier_channels(K, min(K, 32), seed=K)
    X = workloads.activations(Mc, K, O, kind="swiglu", sigma=20.0, seed=Mc)
    W = workloads.weights(N, K, seed=N)
    run(X, W, nO, group)


def test_selection_ties_and_planted_channels():
    g = torch.Generator().manual_seed(9)
    X = torch.randn(700, 512, generator=g)
    W = torch.randn(300, 512, generator=g) / 16
    for c in (11, 40, 333, 400):      # identical dominant columns: equal scores
        X[:, c] = X[:, 0] * 25.0
        W[:, c] = W[:, 0]
    X[:, 100] *= 60.0
    O = run(X.to(torch.bfloat16), W.to(torch.bfloat16), 3)
    assert list(O) == [11, 40, 100]


def test_selection_rejects_bad_groups():
    dev = torch.device("cuda")
    X = torch.zeros(8, 64, dtype=torch.bfloat16, device=dev)
    W = torch.zeros(8, 64, dtype=torch.bfloat16, device=dev)
    with pytest.raises(sq.SQError):
        sq.select_outliers(X, W, 12, group=8)
