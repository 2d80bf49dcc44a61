"""Seeded synthetic workloads for the dual-path sparse-quantized linear layer.

This module only draws inputs.  It holds none of the layer's arithmetic
(no scales, no codes, no products), so both the CPU oracle's tests and the
CUDA path's tests and benchmark can take their inputs from here without the
two sides sharing any computation.

Workload shapes follow the LLM projection layers that the SQ-format page
(arXiv:2512.05409, sections 4 and 8: Llama-3-8B / Llama-3-70B prefill) and the
OSC page (arXiv:2604.12782, abstract: Qwen3, down-projection "W2" inputs) use.
No model weights or text datasets are involved: activations and weights are
Gaussian draws with the statistics below, which stand in for the pages'
WikiText / Qwen3 evaluations.

Recipe (all draws on the torch CPU generator, fp32, then rounded to bf16 with
round-to-nearest-even):
  * O: ``torch.randperm(K)`` with seed 0, first ``nO`` entries, sorted
    ascending -- a uniform draw without replacement, the same for every token
    (the token-persistent outlier channels of the OSC abstract).
  * X (seed 1): N(0,1) everywhere, outlier channels multiplied by ``sigma``
    (so they are N(0, sigma^2)).  The "swiglu" kind instead draws two N(0,1)
    matrices a, b and uses a*b (a post-SwiGLU-like product), with the outlier
    channels multiplied by ``sigma``.
  * W (seed 2): N(0, 1/K).
"""
from __future__ import annotations

import dataclasses
import math

import torch

SEED_O = 0
SEED_X = 1
SEED_W = 2


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    M: int
    K: int
    N: int
    nO: int
    x_kind: str = "gauss"      # "gauss" or "swiglu"
    sigma: float = 30.0        # outlier-channel multiplier

    @property
    def KN(self) -> int:
        return self.K - self.nO

    def describe(self) -> dict:
        return {"workload": self.name, "M": self.M, "K": self.K, "N": self.N,
                "nO": self.nO, "x_kind": self.x_kind, "outlier_sigma": self.sigma}


TINY = Workload("tiny_64x256x256_o8", 64, 256, 256, 8)
LLAMA8B_QKV = Workload("llama3_8b_qkv_2048x4096x6144_o256", 2048, 4096, 6144, 256)
LLAMA8B_DOWN = Workload("llama3_8b_down_4096x14336x4096_o1792", 4096, 14336, 4096, 1792,
                        x_kind="swiglu", sigma=40.0)
LLAMA70B_GATEUP = Workload("llama3_70b_gateup_8192x8192x57344_o512", 8192, 8192, 57344, 512,
                           sigma=50.0)


def sweep_workloads() -> list[Workload]:
    """K = N = 8192 square layer; M in {16, 512, 8192} x nO/K in {1/2,1/4,1/8,1/16,0}."""
    out = []
    for M in (16, 512, 8192):
        for den in (2, 4, 8, 16, 0):
            nO = 0 if den == 0 else 8192 // den
            tag = "0" if den == 0 else f"1/{den}"
            out.append(Workload(f"sweep_M{M}_o{tag}", M, 8192, 8192, nO))
    return out


CONFIGS = {w.name: w for w in [TINY, LLAMA8B_QKV, LLAMA8B_DOWN, LLAMA70B_GATEUP] + sweep_workloads()}


def outlier_channels(K: int, nO: int, seed: int = SEED_O) -> torch.Tensor:
    """Sorted int32 tensor of nO distinct channels drawn uniformly from [0, K)."""
    if nO == 0:
        return torch.zeros(0, dtype=torch.int32)
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(K, generator=g)[:nO]
    return torch.sort(perm).values.to(torch.int32)


def _randn(shape, seed: int) -> torch.Tensor:
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g, dtype=torch.float32)


def activations(M: int, K: int, O: torch.Tensor, kind: str = "gauss", sigma: float = 30.0,
                seed: int = SEED_X) -> torch.Tensor:
    """bf16 [M, K] activations with the outlier channels O amplified by ``sigma``."""
    if kind == "gauss":
        x = _randn((M, K), seed)
    elif kind == "swiglu":
        g = torch.Generator().manual_seed(seed)
        a = torch.randn(M, K, generator=g, dtype=torch.float32)
        b = torch.randn(M, K, generator=g, dtype=torch.float32)
        x = a.mul_(b)
        del b
    else:
        raise ValueError(f"unknown activation kind {kind!r}")
    if O.numel():
        x[:, O.long()] *= sigma
    return x.to(torch.bfloat16)


def weights(N: int, K: int, seed: int = SEED_W) -> torch.Tensor:
    """bf16 [N, K] weights ~ N(0, 1/K)."""
    w = _randn((N, K), seed)
    w.mul_(1.0 / math.sqrt(K))
    return w.to(torch.bfloat16)


def make(w: Workload, with_weights: bool = True):
    """(O, X, W) for a workload; W is None when ``with_weights`` is False."""
    O = outlier_channels(w.K, w.nO)
    X = activations(w.M, w.K, O, w.x_kind, w.sigma)
    W = weights(w.N, w.K) if with_weights else None
    return O, X, W


def bf16_bits(t: torch.Tensor):
    """uint16 numpy view of a bf16 CPU tensor (the exact bit patterns)."""
    assert t.dtype == torch.bfloat16 and t.device.type == "cpu"
    return t.contiguous().view(torch.int16).numpy().view("uint16")
