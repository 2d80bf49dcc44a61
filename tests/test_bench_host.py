"""Host logic of bench.py (no GPU): the source hash that keys the recorded ncu
traffic, and the algorithmic byte counts of the two kernels."""
from __future__ import annotations

import json

import bench


def test_code_only_drops_comments_keeps_code_and_strings():
    src = 'int a = 1;  // note\n/* block\n comment */ const char *s = "x//y /*z*/";\nchar q = \'"\';\n'
    assert bench._code_only(src) == 'int a = 1; const char *s = "x//y /*z*/"; char q = \'"\';'
    # whitespace and comment edits leave the code text unchanged; a code edit does not
    assert bench._code_only("a  =\n b; // x") == bench._code_only("a = b;  /* y */")
    assert bench._code_only("a = b;") != bench._code_only("a = c;")


def test_recorded_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    d = tmp_path / "profiles"
    d.mkdir()
    rec = {"source_hash": bench.source_hash(),
           "workloads": {"w": {"dual_gemm": 123.0}, "w|mx": {"dual_gemm": 456.0}}}
    (d / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "source_hash", lambda: rec["source_hash"])
    assert bench.recorded_traffic("w", "dual_gemm") == 123.0
    assert bench.recorded_traffic("w", "dual_gemm", "mx") == 456.0
    assert bench.recorded_traffic("w", "rowquant") is None
    monkeypatch.setattr(bench, "source_hash", lambda: "0" * 16)   # kernels changed since the capture
    assert bench.recorded_traffic("w", "dual_gemm") is None


def test_algorithmic_bytes():
    # Llama-3-8B QKV: 2048 x 4096 x 6144, 256 outlier channels
    M, K, N, nO = 2048, 4096, 6144, 256
    KN = K - nO
    assert bench.quant_gather_bytes(M, K, nO) == 2 * M * K + M * KN // 2 + 2 * M * nO + 4 * M
    g = bench.gemm_bytes(M, N, K, nO)
    assert g == N * KN // 2 + 2 * N * nO + 4 * N + M * KN // 2 + 2 * M * nO + 4 * M + 2 * M * N
    # E4M3 codes are one byte each, MX codes half a byte plus one scale byte per 32
    assert bench.gemm_bytes(M, N, K, nO, cb=1.0) - g == (N + M) * KN // 2


def test_both_arms_describe_the_same_config():
    """The GPU arm and the reference arm print the same `config` dict for a run."""
    import argparse
    import workloads
    args = argparse.Namespace(low="int4", bank=16, high=1)
    w = workloads.LLAMA70B_GATEUP
    c = bench.run_config(w, args, 1)
    assert c["workload"] == w.name and c["M"] == 8192 and c["N"] == 57344 and c["nO"] == 512
    assert c["parallelism"] == "single" and bench.run_config(w, args, 2)["parallelism"] == "dp2"
    assert bench.DEFAULT_WORKLOAD == w.name
