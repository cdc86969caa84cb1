"""GPU parity: AQLoRA per-layer NF4 error (within 1e-6 relative) and ranks
(bit-exact) against the oracle."""
import numpy as np
import pytest
import torch

from oracle import layer_error, nf4
from quantized_lora_fine_b200 import api, synth
from tests import stack_pool
from tests.conftest import load_golden
from tests.gpu_helpers import bits

pytestmark = pytest.mark.gpu


def _compare(Ws, K, dq):
    ref_err = np.array([layer_error.layer_error(bits(W), dq) for W in Ws])
    ref_order = layer_error.rank_layers(ref_err)
    ref_keep = layer_error.keep_mask(ref_order, K)
    err, order, keep = api.layer_error_rank([W.cuda() for W in Ws], K, double_quant=dq)
    torch.cuda.synchronize()
    err = err.cpu().numpy()
    nz = ref_err > 0
    assert np.all(np.abs(err[nz] - ref_err[nz]) <= 1e-6 * ref_err[nz])
    assert np.all(err[~nz] == 0)
    assert np.array_equal(order.cpu().numpy(), ref_order)
    assert np.array_equal(keep.cpu().numpy(), ref_keep)
    assert api.status() == 0


@pytest.mark.parametrize("dq", [False, True])
def test_small_stack(cuda_device, dq):
    mats = synth.stack_matrices(n_layers=4, linears=(("a", 256, 512), ("b", 512, 256), ("c", 64, 320)))
    Ws = [synth.stack_weight(m) for m in mats]
    _compare(Ws, K=5, dq=dq)


def test_degenerate_layers(cuda_device):
    Ws = [torch.zeros((64, 64), dtype=torch.bfloat16),
          synth.normal_bf16((64, 128), 0.02, 0, 1, 0),
          synth.normal_bf16((64, 128), 0.02, 0, 1, 0),   # exact duplicate: tie resolved by index
          synth.student_t_bf16((128, 64), 3.0, 0.01, 0, 1, 1)]
    _compare(Ws, K=0, dq=False)
    _compare(Ws, K=4, dq=False)
    _compare(Ws, K=2, dq=True)


def test_llama_stack_sampled_layers(cuda_device):
    """A few full-size matrices of the 32-layer Llama-7B-shaped stack (per-layer
    Student-t with nu in [3,30], scale in [0.005,0.05]); K = 3."""
    mats = synth.stack_matrices()
    pick = [mats[i] for i in (0, 4, 6, 100, 223)]
    Ws = [synth.stack_weight(m) for m in pick]
    _compare(Ws, K=3, dq=False)


def _golden_stack(name, mats):
    """The oracle's errors, order and keep for a full stack (tests/golden, written by
    make_stack_rank_goldens.py from the host-drawn weights), and the same weights on
    the GPU, drawn on the host the same way."""
    gold = load_golden(name)
    assert [(m["out"], m["in"]) for m in gold["matrices"]] == [(m.out, m.inp) for m in mats]
    Ws = [None] * len(mats)
    for idx, b in stack_pool.stack_bits(mats):
        Ws[idx] = synth.from_bf16_bits(b, device="cuda")
    return gold, Ws


def _check_against_golden(gold, err, order, keep):
    ref = np.array(gold["err"], np.float64)
    e = err.cpu().numpy()
    assert np.all(ref > 0)
    rel = np.abs(e - ref) / ref
    assert rel.max() <= 1e-6, (int(rel.argmax()), float(rel.max()))
    assert np.array_equal(order.cpu().numpy(), np.array(gold["order"], np.int32))
    assert np.array_equal(keep.cpu().numpy(), np.array(gold["keep"], np.uint8))


@pytest.mark.parametrize("name,mats_of", [
    ("stack_rank_llama7b.json", lambda: synth.stack_matrices()),
    ("stack_rank_14b.json", lambda: synth.stack_matrices_14b())])
def test_full_stack_ranking_against_oracle_golden(cuda_device, name, mats_of):
    """Every matrix of the 224-matrix Llama-7B-shaped stack (fp32 absmax, K = 16) and
    of the 280-matrix 14B-shaped stack (double quant, K = 8): all errors within 1e-6
    relative of the oracle's, order and keep bit-exact, through the error pass and
    through the fused quantize + error pass."""
    gold, Ws = _golden_stack(name, mats_of())
    dq, K = gold["double_quant"], gold["K"]
    err, order, keep = api.layer_error_rank(Ws, K, double_quant=dq)
    torch.cuda.synchronize()
    assert api.status() == 0
    _check_against_golden(gold, err, order, keep)
    err, order, keep, outs = api.quantize_error_rank(Ws, K, double_quant=dq)
    torch.cuda.synchronize()
    assert api.status() == 0
    _check_against_golden(gold, err, order, keep)
    del Ws, outs
    torch.cuda.empty_cache()


def _compare_fused(Ws, K, dq):
    err, order, keep, outs = api.quantize_error_rank([W.cuda() for W in Ws], K, double_quant=dq, keep_absmax=dq)
    torch.cuda.synchronize()
    assert api.status() == 0
    ref_err = np.array([layer_error.layer_error(bits(W), dq) for W in Ws])
    ref_order = layer_error.rank_layers(ref_err)
    e = err.cpu().numpy()
    nz = ref_err > 0
    assert np.all(np.abs(e[nz] - ref_err[nz]) <= 1e-6 * ref_err[nz])
    assert np.all(e[~nz] == 0)
    assert np.array_equal(order.cpu().numpy(), ref_order)
    assert np.array_equal(keep.cpu().numpy(), layer_error.keep_mask(ref_order, K))
    for W, w in zip(Ws, outs):
        qw = nf4.quantize(nf4.f32_from_bf16_bits(bits(W)).reshape(W.shape), double_quant=dq)
        assert np.array_equal(w.codes.cpu().numpy(), qw["codes"]), "codes differ"
        assert np.array_equal(w.absmax.cpu().numpy().view(np.uint32), qw["absmax"].view(np.uint32))
        if dq:
            assert np.array_equal(w.absmax_q.cpu().numpy(), qw["absmax_q"])
            assert np.array_equal(w.absmax2.cpu().numpy().view(np.uint32), qw["absmax2"].view(np.uint32))


@pytest.mark.parametrize("dq", [False, True])
def test_fused_quantize_error_rank_small_stack(cuda_device, dq):
    """One pass: the same errors and ranks as the oracle's error pass and the same
    codes and scales as the oracle's quantizer, for every layer."""
    mats = synth.stack_matrices(n_layers=3, linears=(("a", 256, 512), ("b", 512, 256), ("c", 64, 320)))
    Ws = [synth.stack_weight(m) for m in mats]
    Ws.append(torch.zeros((64, 64), dtype=torch.bfloat16))
    _compare_fused(Ws, K=4, dq=dq)


def test_fused_quantize_error_rank_full_gate(cuda_device):
    mats = synth.stack_matrices()
    Ws = [synth.stack_weight(mats[i]) for i in (4, 7)]   # an 11008 x 4096 gate and a 4096^2 q
    _compare_fused(Ws, K=1, dq=True)


def _compare_budget(Ws, dq, budgets):
    ref_err = np.array([layer_error.layer_error(bits(W), dq) for W in Ws])
    ref_order = layer_error.rank_layers(ref_err)
    numel = [W.numel() for W in Ws]
    g = [W.cuda() for W in Ws]
    for budget in budgets:
        K_ref = layer_error.k_under_memory_budget(ref_order, numel, dq, budget)
        err, order, keep, K = api.layer_error_rank_budget(g, budget, double_quant=dq)
        torch.cuda.synchronize()
        assert int(K.item()) == K_ref, (budget, int(K.item()), K_ref)
        assert np.array_equal(order.cpu().numpy(), ref_order)
        assert np.array_equal(keep.cpu().numpy(), layer_error.keep_mask(ref_order, K_ref))
        nz = ref_err > 0
        assert np.all(np.abs(err.cpu().numpy()[nz] - ref_err[nz]) <= 1e-6 * ref_err[nz])
    assert api.status() == 0


@pytest.mark.parametrize("dq", [False, True])
def test_memory_budget_keep_rule(cuda_device, dq):
    """K from a byte budget: the budget at each exact prefix sum of the ranked costs
    keeps that prefix, one byte less keeps one layer fewer; zero keeps none and a
    large budget keeps all."""
    mats = synth.stack_matrices(n_layers=3, linears=(("a", 256, 512), ("b", 512, 256), ("c", 64, 320)))
    Ws = [synth.stack_weight(m) for m in mats]
    ref_err = np.array([layer_error.layer_error(bits(W), dq) for W in Ws])
    order = layer_error.rank_layers(ref_err)
    costs = np.cumsum([layer_error.protect_cost_bytes(Ws[l].numel(), dq) for l in order])
    budgets = [0, 1, int(costs[-1]) * 10] + [int(c) for c in costs[:5]] + [int(c) - 1 for c in costs[:5]]
    _compare_budget(Ws, dq, budgets)


def test_copy_wait_timeout_is_reported(cuda_device, monkeypatch):
    """Failure detection without a GPU fault: with the chunk kernel's bulk-copy wait
    limited to a single try, every chunk gives up before its copy lands. The call
    returns, the status word reads QLORA_ERR_TIMEOUT and the errors are NaN (each
    timed-out chunk writes a NaN partial); every copy still lands before its CTA exits,
    so after the status is cleared the same call with the normal limit matches the
    oracle on the same context."""
    mats = synth.stack_matrices(n_layers=2, linears=(("a", 256, 512), ("b", 512, 256)))
    Ws = [synth.stack_weight(m) for m in mats]
    g = [W.cuda() for W in Ws]
    monkeypatch.setenv("QLORA_B200_COPY_WAIT_NS", "0")
    err, order, keep = api.layer_error_rank(g, 2, double_quant=False)
    torch.cuda.synchronize()
    assert api.status() == 9          # QLORA_ERR_TIMEOUT
    assert np.all(np.isnan(err.cpu().numpy()))
    assert sorted(order.cpu().tolist()) == list(range(len(Ws)))   # still a permutation
    for ws in api.Workspace.all(torch.cuda.current_device()):
        api.reset_status(ws)
    monkeypatch.delenv("QLORA_B200_COPY_WAIT_NS")
    _compare(Ws, K=2, dq=False)


def test_rank_errors_alone_and_sharded_on_one_gpu(cuda_device):
    """The ranking step alone (nf4_rank_errors) on oracle errors gives the oracle's
    order and keep; the sharded pass with one rank (the library's error pass and
    ranking) gives the unsharded call's results."""
    from quantized_lora_fine_b200 import dist as qdist
    mats = synth.stack_matrices(n_layers=2, linears=(("a", 256, 512), ("b", 512, 256), ("c", 64, 320)))
    Ws = [synth.stack_weight(m) for m in mats]
    ref = np.array([layer_error.layer_error(bits(W), True) for W in Ws])
    ref_order = layer_error.rank_layers(ref)
    order, keep = api.rank_errors(torch.tensor(ref, dtype=torch.float64, device="cuda"), 3)
    torch.cuda.synchronize()
    assert np.array_equal(order.cpu().numpy(), ref_order)
    assert np.array_equal(keep.cpu().numpy(), layer_error.keep_mask(ref_order, 3))
    g = {i: W.cuda() for i, W in enumerate(Ws)}
    err, order, keep = qdist.sharded_layer_error_rank(g, [W.numel() for W in Ws], 3, double_quant=True)
    e1, o1, k1 = api.layer_error_rank(list(g.values()), 3, double_quant=True)
    torch.cuda.synchronize()
    assert torch.equal(err, e1) and torch.equal(order, o1) and torch.equal(keep, k1)
    assert api.status() == 0
