"""GPU parity: NF4-LoRA linear forward / backward against the fp64 oracle."""
import dataclasses

import numpy as np
import pytest
import torch

from oracle import lora
from quantized_lora_fine_b200 import api, synth
from tests.gpu_helpers import assert_close, f64_of_bf16, gpu_case, oracle_qweight, oracle_what

pytestmark = pytest.mark.gpu


def run_and_compare(case: synth.LinearCase, protected=False, rows=None, need_dX=True, save_T=True):
    d = case.make()
    s = case.scale
    if protected:
        What = f64_of_bf16(d["W"])
    else:
        What = oracle_what(oracle_qweight(d["W"], case.double_quant))
    X, L1, L2, dY = (f64_of_bf16(d[k]) for k in ("X", "L1", "L2", "dY"))
    g, w = gpu_case(d, case.double_quant, protected)
    Y, T = api.linear_fwd(w, g["X"], g["L1"], g["L2"], s, save_T=save_T)
    dX, dL1, dL2 = api.linear_bwd(w, g["X"], g["dY"], g["L1"], g["L2"], s, T=T, need_dX=need_dX)
    torch.cuda.synchronize()
    assert api.status() == 0
    sel = np.arange(case.M) if rows is None else rows
    Yref, Tref = lora.forward(X[sel], What, L1, L2, s)
    out = {}
    out["Y"] = assert_close(f64_of_bf16(Y)[sel], Yref, "Y")
    if T is not None:
        out["T"] = assert_close(f64_of_bf16(T)[sel], Tref, "T")
    # gradients: dL1/dL2 reduce over all M rows; dX is checked on the sampled rows
    T_full = X @ L1
    U_full = dY @ L2.T
    out["dL2"] = assert_close(dL2.cpu().numpy(), s * (T_full.T @ dY), "dL2")
    out["dL1"] = assert_close(dL1.cpu().numpy(), s * (X.T @ U_full), "dL1")
    if need_dX:
        dXref = dY[sel] @ What + s * (U_full[sel] @ L1.T)
        out["dX"] = assert_close(f64_of_bf16(dX)[sel], dXref, "dX")
    else:
        assert dX is None
    return out


def test_small_case_fwd_bwd(cuda_device):
    run_and_compare(synth.case_small())


@pytest.mark.parametrize("M", [1, 77, 200, 384])
def test_ragged_token_counts(cuda_device, M):
    run_and_compare(dataclasses.replace(synth.case_small(), M=M))


@pytest.mark.parametrize("r", [8, 16, 32, 64, 128, 256])
def test_ranks(cuda_device, r):
    c = dataclasses.replace(synth.case_small(), M=256, out=768, inp=512, r=r, alpha=2.0 * r, double_quant=(r % 16 == 0))
    run_and_compare(c)


@pytest.mark.parametrize("pairs", [1, 2, 3, 4, 5, 7])
def test_split_last_round_schedules(cuda_device, monkeypatch, pairs):
    """The GEMMs' schedule with the co-resident pairs capped: whole rounds of 512 x 256
    tiles, then the remaining tiles cut into step ranges over the pairs (a tile in up
    to four parts, finished by the pair holding its first step) or run whole. Six
    output tiles of 1024 x 768 with 9 steps each (8 K steps + the LoRA step) give a
    different mix of whole rounds and split tiles for every cap; ragged M covers a
    box wholly past the last row."""
    monkeypatch.setenv("QLORA_B200_MAX_PAIRS", str(pairs))
    c = dataclasses.replace(synth.case_small(), M=1024, out=768, inp=512, r=16, alpha=32.0, double_quant=True)
    run_and_compare(c)
    run_and_compare(dataclasses.replace(c, M=700))


_ENGINE_CHECK = """
import dataclasses, sys
sys.path.insert(0, {root!r})
from quantized_lora_fine_b200 import synth
from tests.test_gpu_linear import run_and_compare
c = dataclasses.replace(synth.case_small(), M=700, out=768, inp=512, r=16, alpha=32.0, double_quant=True)
run_and_compare(c)
print("ok")
"""


@pytest.mark.parametrize("env", [{"QLORA_B200_PAIR2": "4x2"}, {"QLORA_B200_GEMM": "pair256"},
                                 {"QLORA_B200_GEMM": "1cta"}])
def test_other_gemm_engines(cuda_device, env):
    """The NF4 GEMM engines kept for measurement (4 ring slots with 2 staging buffers,
    the 256 x 256 pair kernel, the single-CTA kernel) give the same products within
    the tolerances. The engine is chosen once per process, so each runs in a child."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    res = subprocess.run([sys.executable, "-c", _ENGINE_CHECK.format(root=root)], env={**os.environ, **env},
                         capture_output=True, text=True, timeout=300)
    assert res.returncode == 0 and res.stdout.strip().endswith("ok"), res.stdout[-2000:] + res.stderr[-2000:]


def test_protected_bf16_layer(cuda_device):
    c = dataclasses.replace(synth.case_small(), M=300, out=512, inp=768, r=16, alpha=32.0)
    run_and_compare(c, protected=True)


def test_early_stop_and_recompute_T(cuda_device):
    c = dataclasses.replace(synth.case_small(), M=192, r=16, alpha=32.0)
    run_and_compare(c, need_dX=False, save_T=False)


def test_zero_adapter_is_plain_gemm(cuda_device):
    c = synth.case_small()
    d = c.make()
    d["L2"] = torch.zeros_like(d["L2"])
    g, w = gpu_case(d, False)
    Y, _ = api.linear_fwd(w, g["X"], g["L1"], g["L2"], c.scale)
    What = oracle_what(oracle_qweight(d["W"], False))
    assert_close(f64_of_bf16(Y), f64_of_bf16(d["X"]) @ What.T, "Y(L2=0)")


def test_deterministic_gradients(cuda_device):
    c = dataclasses.replace(synth.case_small(), M=512, r=16, alpha=32.0)
    d = c.make()
    g, w = gpu_case(d, False)
    a = api.linear_bwd(w, g["X"], g["dY"], g["L1"], g["L2"], c.scale)
    b = api.linear_bwd(w, g["X"], g["dY"], g["L1"], g["L2"], c.scale)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_q_proj_full_size_sampled(cuda_device):
    """Llama-7B q_proj shape at full size (M=8192, 4096^2, DQ, r=16): Y and dX on
    sampled rows, dL1 / dL2 over all rows."""
    rows = np.random.default_rng(0).choice(8192, 192, replace=False)
    rows.sort()
    run_and_compare(synth.case_q_proj(), rows=rows)


@pytest.mark.parametrize("idx", [0, 1, 2])   # gate, up, down
def test_mlp_full_size_sampled(cuda_device, idx):
    rows = np.random.default_rng(1).choice(8192, 96, replace=False)
    rows.sort()
    run_and_compare(synth.cases_mlp()[idx], rows=rows)


@pytest.mark.parametrize("kind,r", [("q", 16), ("gate", 32), ("down", 64), ("q", 128)])
def test_14b_shapes_full_size_sampled(cuda_device, kind, r):
    """14B-shaped linears (hidden 5120, intermediate 13824), double quant, X of
    16384 tokens, the sweep's ranks: Y and dX on sampled rows, dL1 / dL2 over all
    rows."""
    case = synth.cases_14b(r, kinds=(kind,))[0]
    rows = np.random.default_rng(2).choice(case.M, 48, replace=False)
    rows.sort()
    run_and_compare(case, rows=rows)


def test_14b_protected_layer_full_size_sampled(cuda_device):
    """A layer the allocation keeps in bf16 (no dequantization) at the 14B gate shape."""
    case = synth.cases_14b(16, kinds=("gate",))[0]
    rows = np.random.default_rng(3).choice(case.M, 32, replace=False)
    rows.sort()
    run_and_compare(case, protected=True, rows=rows)


def test_two_part_forward_matches_forward(cuda_device, monkeypatch):
    """lora_down + linear_fwd(T=...) is the forward split in two: the same bits as
    the one-call forward when that one computes T in its own pass (same kernels,
    same T)."""
    monkeypatch.setenv("QLORA_B200_FUSED_T", "0")
    case = synth.case_small()
    d = case.make()
    g, w = gpu_case(d, case.double_quant, False)
    Y1, T1 = api.linear_fwd(w, g["X"], g["L1"], g["L2"], case.scale)
    T2 = api.lora_down(g["X"], g["L1"])
    Y2, T2r = api.linear_fwd(w, g["X"], g["L1"], g["L2"], case.scale, T=T2)
    torch.cuda.synchronize()
    assert api.status() == 0
    assert T2r is T2
    assert torch.equal(T1, T2)
    assert torch.equal(Y1, Y2)


def test_quantize_on_side_stream_beside_lora_down(cuda_device, monkeypatch):
    """The allocation pass on a second stream while T = X L1 runs on the first (each
    stream has its own workspace): the same codes, scales and outputs as in order."""
    monkeypatch.setenv("QLORA_B200_FUSED_T", "0")
    case = synth.case_small()
    d = case.make()
    g = {k: v.cuda() for k, v in d.items()}
    ref_w = api.quantize(g["W"], double_quant=True)
    Yref, Tref = api.linear_fwd(ref_w, g["X"], g["L1"], g["L2"], case.scale)
    main = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    side.wait_stream(main)
    with torch.cuda.stream(side):
        _, _, _, (w,) = api.quantize_error_rank([g["W"]], 0, double_quant=True)
    T = api.lora_down(g["X"], g["L1"])
    main.wait_stream(side)
    for t in (w.codes, w.absmax_q, w.absmax2):
        t.record_stream(main)
    Y, _ = api.linear_fwd(w, g["X"], g["L1"], g["L2"], case.scale, T=T)
    torch.cuda.synchronize()
    assert api.status() == 0
    assert torch.equal(w.codes, ref_w.codes) and torch.equal(w.absmax_q, ref_w.absmax_q)
    assert torch.equal(w.absmax2, ref_w.absmax2)
    assert torch.equal(T, Tref) and torch.equal(Y, Yref)


@pytest.mark.parametrize("M,r,pairs", [(1300, 16, None), (1300, 72, None), (600, 256, None), (2048, 64, None),
                                       (1300, 16, 3), (2048, 64, 5)])
def test_fused_t_tiles(cuda_device, monkeypatch, M, r, pairs):
    """The forward GEMM computes T = X L1 itself: one extra tile per 512-row block
    (A = the X rows, B = L1), whose rows the output tiles' LoRA step waits for. T and
    Y are within the oracle's tolerance, and T differs from the separate T = X L1
    pass by at most one bf16 rounding (the fp32 sums are added in another order).
    Ragged M and r (a partial 64-column chunk of T), r = 256 (four chunks), and a
    capped pair count (T tiles cut into step ranges) are covered."""
    if pairs is not None:
        monkeypatch.setenv("QLORA_B200_MAX_PAIRS", str(pairs))
    c = dataclasses.replace(synth.case_small(), M=M, out=768, inp=512, r=r, alpha=2.0 * r, double_quant=True)
    monkeypatch.delenv("QLORA_B200_FUSED_T", raising=False)
    run_and_compare(c)
    d = c.make()
    g, w = gpu_case(d, c.double_quant, False)
    Yf, Tf = api.linear_fwd(w, g["X"], g["L1"], g["L2"], c.scale)
    monkeypatch.setenv("QLORA_B200_FUSED_T", "0")
    Yu, Tu = api.linear_fwd(w, g["X"], g["L1"], g["L2"], c.scale)
    torch.cuda.synchronize()
    assert api.status() == 0
    tf, tu = Tf.double(), Tu.double()
    # one bf16 rounding, plus fp32 summation-order slack where T nearly cancels
    slack = 2.0 ** -7 * tu.abs() + 2.0 ** -16 * tu.abs().max()
    assert torch.all((tf - tu).abs() <= slack), "fused T off by more than one rounding"
    assert_close(f64_of_bf16(Yf), f64_of_bf16(Yu), "Y fused vs separate T")


@pytest.mark.parametrize("M,r,pairs", [(1300, 16, None), (1300, 72, None), (600, 256, None), (2048, 64, None),
                                       (1300, 16, 3), (2048, 128, 5)])
def test_fused_u_tiles(cuda_device, monkeypatch, M, r, pairs):
    """The dX GEMM computes U = dY L2^T itself (forced on: by default only for outputs
    of at least 32 column tiles, as the full-size MLP down and 14B down cases are):
    one extra tile per 512-row block (A = the dY rows, B = L2 read K-major) that
    stores U and s.U, whose rows the output tiles' LoRA step waits for; dL1 and dL2
    run after it. Gradients are within the
    oracle's tolerance, dL2 (which does not read U) has the same bits as with U as
    its own pass, and dX and dL1 agree with that path within one bf16 rounding of U."""
    if pairs is not None:
        monkeypatch.setenv("QLORA_B200_MAX_PAIRS", str(pairs))
    c = dataclasses.replace(synth.case_small(), M=M, out=768, inp=512, r=r, alpha=2.0 * r, double_quant=True)
    monkeypatch.setenv("QLORA_B200_FUSED_U", "1")   # by default only outputs of >= 32 column tiles
    monkeypatch.delenv("QLORA_B200_BWD", raising=False)
    run_and_compare(c)
    d = c.make()
    g, w = gpu_case(d, c.double_quant, False)
    _, T = api.linear_fwd(w, g["X"], g["L1"], g["L2"], c.scale)
    fused = api.linear_bwd(w, g["X"], g["dY"], g["L1"], g["L2"], c.scale, T=T)
    monkeypatch.setenv("QLORA_B200_FUSED_U", "0")
    sep = api.linear_bwd(w, g["X"], g["dY"], g["L1"], g["L2"], c.scale, T=T)
    torch.cuda.synchronize()
    assert api.status() == 0
    assert torch.equal(fused[2], sep[2]), "dL2 does not read U"
    assert_close(f64_of_bf16(fused[0]), f64_of_bf16(sep[0]), "dX fused vs separate U")
    assert_close(fused[1].double().cpu().numpy(), sep[1].double().cpu().numpy(), "dL1 fused vs separate U")


@pytest.mark.parametrize("schedule", ["beside", "serial"])
def test_backward_schedules_give_the_same_bits(cuda_device, monkeypatch, schedule):
    """Both backward schedules (dX beside dL1 / dL2, or dL2 beside U and dL1 before
    dX) compute the same products with the same reductions: identical bits, and
    within the oracle's tolerance."""
    case = dataclasses.replace(synth.case_q_proj(seed=3, M=1024), double_quant=True)
    monkeypatch.delenv("QLORA_B200_BWD", raising=False)
    ref = run_and_compare(case, rows=np.arange(0, case.M, 97))
    monkeypatch.setenv("QLORA_B200_FUSED_U", "0")   # U as its own pass in every schedule
    d = case.make()
    g, w = gpu_case(d, case.double_quant, False)
    Y, T = api.linear_fwd(w, g["X"], g["L1"], g["L2"], case.scale)
    outs = {}
    for sch in ("auto", schedule):
        if sch == "auto":
            monkeypatch.delenv("QLORA_B200_BWD", raising=False)
        else:
            monkeypatch.setenv("QLORA_B200_BWD", sch)
        outs[sch] = api.linear_bwd(w, g["X"], g["dY"], g["L1"], g["L2"], case.scale, T=T)
    torch.cuda.synchronize()
    assert api.status() == 0
    for a, b in zip(outs["auto"], outs[schedule]):
        assert torch.equal(a, b)
    assert ref is not None
