"""sq_linear (and its FP8, MXFP4 and SQ-format forms) against the CPU oracle on
every configuration of the layer: the tiny layer, the Llama-3-8B QKV and down
projections, the Llama-3-70B gate+up projection, and all fifteen points of
the K = N = 8192 sweep (M in {16, 512, 8192} x nO/K in {1/2, 1/4, 1/8, 1/16, 0}).

Each case calls the whole-layer entry point through the C ABI with a caller
workspace, in the launch configuration the benchmark times, and then checks:
  * the quantize-and-gather outputs that sq_linear left in its workspace
    (codes, scales, compact outlier channels), bit-exact on every token row;
  * Y on a seeded sample of rows, within |dY| <= 1e-2 * max(|Y_ref|, rms(Y_ref));
  * the GEMM alone on that same workspace gives sq_linear's Y bit for bit;
  * the GEMM's accumulators on the same rows, from a debug run of the GEMM on
    that workspace: the int32 sums exactly, the fp32 sums within the fp32
    summation bound of the oracle's exact fp64 sums, and its Y (which adds
    the two sums outside the tensor core) within the Y tolerance too;
  * nothing written outside Y (a guard row and guard columns).
"""
from __future__ import annotations

import functools

import numpy as np
import pytest
import torch

import oracle
import workloads
import mixed_precision_gemm_b200 as sq
from test_gpu_fp8 import check_quant_fp8
from test_gpu_mx import check_quant_mx, dequant_abs
from test_gpu_parity import check_quant

pytestmark = pytest.mark.gpu

Y_TOL = 1e-2
ACC_F_REL = 2.0 ** -20    # bf16 x bf16 products summed in fp32 (16-bit branch)
ACC_8_REL = 2.0 ** -12    # E4M3 / E2M1 products summed by the tensor core in fp32
GUARD = -1024.0

NAMES = [workloads.TINY.name, workloads.LLAMA8B_QKV.name, workloads.LLAMA8B_DOWN.name,
         workloads.LLAMA70B_GATEUP.name] + [w.name for w in workloads.sweep_workloads()]
CASES = [(n, low) for n in NAMES for low in ("int4", "fp8", "mx")]
SQF_CASES = [workloads.TINY.name, workloads.LLAMA8B_QKV.name, workloads.LLAMA8B_DOWN.name,
             workloads.LLAMA70B_GATEUP.name, "sweep_M16_o0", "sweep_M512_o0", "sweep_M8192_o0"]


@functools.lru_cache(maxsize=1)
def inputs(name):
    """(O numpy, X, W) for a configuration; cached so the low paths of one configuration share one draw."""
    O, X, W = workloads.make(workloads.CONFIGS[name])
    return O.numpy(), X, W


def sample(M: int, n: int = 24, seed: int = 99) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([rng.choice(M, size=min(n, M), replace=False), [0, M - 1]]))


def rup(v: int, a: int = 256) -> int:
    return (v + a - 1) // a * a


def guarded_y(M, N, dev):
    g = torch.full((M + 1, N + 8), GUARD, dtype=torch.bfloat16, device=dev)
    return g, g[:M, :N]


def check_guard(g, M, N):
    assert bool(torch.all(g[M] == GUARD)) and bool(torch.all(g[:, N:] == GUARD)), "write outside Y"


def check_y(Y_rows: np.ndarray, y_ref: np.ndarray):
    rms = float(np.sqrt(np.mean(y_ref ** 2))) if y_ref.size else 0.0
    err = np.abs(Y_rows - y_ref)
    bound = Y_TOL * np.maximum(np.abs(y_ref), rms)
    bad = err > bound
    assert not bad.any(), (f"{int(bad.sum())} of {bad.size} Y entries out of tolerance; "
                           f"worst {float((err / np.maximum(bound, 1e-300)).max()):.3g} of the bound")


def f64_of_bits(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def rows_of(t: torch.Tensor, sel: np.ndarray) -> np.ndarray:
    return t[torch.as_tensor(sel, device=t.device)].float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("name,low", CASES, ids=[f"{n}-{low}" for n, low in CASES])
def test_linear_matches_oracle(name, low):
    w = workloads.CONFIGS[name]
    O, X, W = inputs(name)
    M, K, N, nO = w.M, w.K, w.N, w.nO
    dev = torch.device("cuda")
    fp8, mx = low == "fp8", low == "mx"
    pw = sq.prepare_weights(W.to(dev), O, fp8=fp8, mx=mx)
    Xd = X.to(dev)
    g, Y = guarded_y(M, N, dev)
    if mx:
        ws = torch.zeros(sq.sq_linear_workspace_bytes_mx(M, K, nO), dtype=torch.uint8, device=dev)
        sq.sq_linear_mx(Xd, pw.chan_tab, pw.W_N, pw.s_w, pw.W_O, N, nO, Y, ws)
    elif fp8:
        ws = torch.zeros(sq.sq_linear_workspace_bytes_fp8(M, K, nO), dtype=torch.uint8, device=dev)
        sq.sq_linear_fp8(Xd, pw.chan_tab, pw.W_N, pw.s_w, pw.W_O, N, nO, Y, ws)
    else:
        ws = torch.zeros(sq.sq_linear_workspace_bytes(M, K, nO), dtype=torch.uint8, device=dev)
        sq.sq_linear(Xd, pw.chan_tab, pw.W_N, pw.s_w, pw.W_O, N, nO, Y, ws)
    torch.cuda.synchronize()
    sq.sq_check()
    check_guard(g, M, N)

    # the workspace as the header lays it out: codes, scales, compact X_O, each 256-byte aligned
    no_pad = sq.sq_no_pad(nO)
    code_bytes = pw.code_bytes(K)
    off_s = rup(M * code_bytes)
    s_bytes = sq.sq_mx_scale_bytes(M, K, nO) if mx else 4 * M
    off_o = off_s + rup(s_bytes)
    X_N = ws[:M * code_bytes].view(M, code_bytes)
    s_x = ws[off_s:off_s + s_bytes] if mx else ws[off_s:off_s + s_bytes].view(torch.float32)
    X_O = ws[off_o:off_o + 2 * M * no_pad].view(torch.bfloat16).view(M, no_pad)
    # the offline weight step and every token row of the quantize-and-gather step, bit-exact
    assert np.array_equal(pw.chan_tab.cpu().numpy().view(np.uint32), oracle.chan_table(O, K))
    chk = check_quant_mx if mx else check_quant_fp8 if fp8 else check_quant
    chk(O, W, pw.W_N, pw.s_w, pw.W_O, K)
    chk(O, X, X_N, s_x, X_O, K)

    # the GEMM alone on that workspace: same Y, bit for bit; then with its accumulators exposed
    g2, Y2 = guarded_y(M, N, dev)
    sq.gemm(X_N, s_x, X_O, pw, Y=Y2)
    g3, Y3 = guarded_y(M, N, dev)
    _, dbg_a, dbg_b = sq.gemm(X_N, s_x, X_O, pw, Y=Y3, debug=True)
    torch.cuda.synchronize()
    sq.sq_check()
    check_guard(g2, M, N)
    check_guard(g3, M, N)
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16)), "sq_linear and the GEMM on its workspace differ"

    sel = sample(M, 16 if N > 10000 else 24)
    Xb, Wb = workloads.bf16_bits(X), workloads.bf16_bits(W)
    if mx:
        ref = oracle.linear_mx(Xb, Wb, O, rows=sel)
        absum = (dequant_abs(ref["qx"], ref["ex"]) @ dequant_abs(ref["qw"], ref["ew"]).T).astype(np.float64)
        if nO:
            absum += np.abs(f64_of_bits(ref["xo"])) @ np.abs(f64_of_bits(ref["wo"])).T
        err = np.abs(rows_of(dbg_b, sel) - (ref["acc_mx"] + ref["acc_o"]))
        assert np.all(err <= ACC_8_REL * absum + 1e-30), "accumulator off"
    else:
        ref = (oracle.linear_fp8 if fp8 else oracle.linear)(Xb, Wb, O, rows=sel)
        if fp8:
            dx = np.abs(oracle.e4m3_decode(ref["qx"]).reshape(ref["qx"].shape))
            dw = np.abs(oracle.e4m3_decode(ref["qw"]).reshape(ref["qw"].shape))
            err8 = np.abs(rows_of(dbg_a, sel) - ref["acc_8"])
            assert np.all(err8 <= ACC_8_REL * (dx @ dw.T) + 1e-30), "E4M3 accumulator off"
        else:
            got_i = dbg_a[torch.as_tensor(sel, device=dev)].cpu().numpy().astype(np.int64)
            assert np.array_equal(got_i, ref["acc_i"]), "int32 accumulators differ"
        if nO:
            absum = np.abs(f64_of_bits(ref["xo"])) @ np.abs(f64_of_bits(ref["wo"])).T
            errf = np.abs(rows_of(dbg_b, sel) - ref["acc_o"])
            assert np.all(errf <= ACC_F_REL * absum + 1e-30), "16-bit branch accumulator off"
        else:
            assert np.all(rows_of(dbg_b, sel) == 0)
    check_y(rows_of(Y, sel), ref["y"])
    check_y(rows_of(Y3, sel), ref["y"])


@pytest.mark.parametrize("name", SQF_CASES)
def test_linear_sqf_matches_oracle(name):
    """Element-level SQ-format weights (banks of 16 channels, one E4M3 entry each; no
    outlier channels) through sq_linear_sqf."""
    w = workloads.CONFIGS[name]
    _, X, W = inputs(name)
    M, K, N = w.M, w.K, w.N
    bank, h = 16, 1
    dev = torch.device("cuda")
    pw = sq.prepare_weights_sqf(W.to(dev), bank, h)
    Xd = X.to(dev)
    g, Y = guarded_y(M, N, dev)
    ws = torch.zeros(sq.sq_linear_workspace_bytes_sqf(M, N, K), dtype=torch.uint8, device=dev)
    sq.sq_linear_sqf(Xd, pw.chan_tab, pw.W_N, pw.s_lo, pw.W_H, pw.W_E, pw.s_hi, N, Y, ws)
    torch.cuda.synchronize()
    sq.sq_check()
    check_guard(g, M, N)

    # workspace: X_N [M, K/2], s_x4 [M], X_8 [M, K], s_x8 [M], P [M, N], each 256-byte aligned
    o1 = rup(M * K // 2)
    o2 = o1 + rup(4 * M)
    o3 = o2 + rup(M * K)
    X_N = ws[:M * K // 2].view(M, K // 2)
    s_x4 = ws[o1:o1 + 4 * M].view(torch.float32)
    X_8 = ws[o2:o2 + M * K].view(M, K)
    s_x8 = ws[o3:o3 + 4 * M].view(torch.float32)
    Xb, Wb = workloads.bf16_bits(X), workloads.bf16_bits(W)
    none = np.zeros(0, np.int32)
    q4, sx4, _ = oracle.quantize_rows(Xb, K, none)
    q8, sx8, _ = oracle.quantize_rows_fp8(Xb, K, none)
    assert np.array_equal(X_N.cpu().numpy(), oracle.pack_int4(q4, K // 2)), "token INT4 codes differ"
    assert np.array_equal(s_x4.cpu().numpy().view(np.uint32), sx4.view(np.uint32)), "s_x4 differs"
    assert np.array_equal(X_8.cpu().numpy(), q8), "token E4M3 codes differ"
    assert np.array_equal(s_x8.cpu().numpy().view(np.uint32), sx8.view(np.uint32)), "s_x8 differs"

    g2, Y2 = guarded_y(M, N, dev)
    sq.gemm_sqf(X_N, s_x4, X_8, s_x8, pw, Y=Y2)
    g3, Y3 = guarded_y(M, N, dev)
    _, acc_lo, P = sq.gemm_sqf(X_N, s_x4, X_8, s_x8, pw, Y=Y3, debug=True)
    torch.cuda.synchronize()
    sq.sq_check()
    check_guard(g2, M, N)
    check_guard(g3, M, N)
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16)), "sq_linear_sqf and the GEMM differ"

    sel = sample(M, 8 if N > 10000 else 16)
    ref = oracle.sqf_linear(Xb, Wb, bank, h, rows=sel)
    got_lo = acc_lo[torch.as_tensor(sel, device=dev)].cpu().numpy().astype(np.int64)
    assert np.array_equal(got_lo, ref["acc_lo"]), "low-part sums differ"
    e4 = np.abs(oracle.e4m3_decode(np.arange(256, dtype=np.uint8))).astype(np.float32)
    dx = e4[ref["qx8"]]
    dw = np.where(ref["hi_mask"] == 1, e4[ref["hi"]], np.float32(0))
    scale = ref["sx8"][:, None].astype(np.float64) * ref["s_hi"][None, :].astype(np.float64)
    p_ref = ref["acc_hi"] * scale
    bound = ACC_8_REL * (dx @ dw.T).astype(np.float64) * scale + 2.0 ** -20 * np.abs(p_ref) + 1e-30
    assert np.all(np.abs(rows_of(P, sel) - p_ref) <= bound), "high part off"
    check_y(rows_of(Y, sel), ref["y"])
    check_y(rows_of(Y3, sel), ref["y"])
