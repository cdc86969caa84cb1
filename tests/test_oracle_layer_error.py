"""Pins for the oracle's AQLoRA per-layer error, ranking and budget rule."""
import numpy as np
import pytest

from oracle import layer_error, nf4, storage
from tests.conftest import load_golden


def _bf16(x):
    return nf4.bf16_bits_from_f32(np.asarray(x, np.float32))


def test_zero_error_for_exact_code_weights():
    rng = np.random.default_rng(0)
    C = nf4.nf4_code_table()
    nb = 64
    a = nf4.f32_from_bf16_bits(_bf16(rng.uniform(0.01, 0.05, nb)))
    idx = rng.integers(0, 16, (nb, 64))
    idx[:, 0] = 15
    w = nf4.f32_from_bf16_bits(_bf16(C[idx] * a[:, None])).reshape(16, -1)
    assert layer_error.layer_error(_bf16(w)) == 0.0


def test_error_is_scale_invariant():
    rng = np.random.default_rng(1)
    w = _bf16(rng.standard_t(5, (64, 256)) * 0.02)
    e0 = layer_error.layer_error(w)
    for k in (-8, 3, 12):
        wk = _bf16(nf4.f32_from_bf16_bits(w) * np.float32(2.0 ** k))
        assert layer_error.layer_error(wk) == e0


def test_error_matches_library_norm():
    rng = np.random.default_rng(2)
    for dq in (False, True):
        w = _bf16(rng.standard_normal((32, 512)) * 0.02)
        qw = nf4.quantize(nf4.f32_from_bf16_bits(w), double_quant=dq)
        what = nf4.f32_from_bf16_bits(nf4.dequantize_bf16_bits(qw)).astype(np.float64)
        W = nf4.f32_from_bf16_bits(w).astype(np.float64)
        ref = np.linalg.norm(W - what) / np.linalg.norm(W)
        assert abs(layer_error.layer_error(w, dq) - ref) <= 1e-12 * ref


def test_error_bruteforce_tiny():
    rng = np.random.default_rng(3)
    w = _bf16(rng.standard_normal(128) * 0.1)
    W = nf4.f32_from_bf16_bits(w)
    C = nf4.nf4_code_table()
    num = den = 0.0
    for b in range(2):
        blk = W[b * 64:(b + 1) * 64]
        a = max(abs(float(x)) for x in blk)
        for x in blk:
            j = nf4.nearest_code_bruteforce(float(np.float32(np.float32(x) / np.float32(a))))
            xh = float(nf4.f32_from_bf16_bits(_bf16(np.float32(C[j]) * np.float32(a))))
            num += (float(x) - xh) ** 2
            den += float(x) ** 2
    assert abs(layer_error.layer_error(w) - np.sqrt(num / den)) < 1e-12


def test_rank_matches_lexsort_and_ties():
    rng = np.random.default_rng(4)
    e = rng.uniform(0, 1, 300)
    e[10] = e[20] = e[5]  # ties resolved by index
    order = layer_error.rank_layers(e)
    ref = np.lexsort((np.arange(300), -e))
    assert np.array_equal(order, ref)
    keep = layer_error.keep_mask(order, 16)
    assert keep.sum() == 16 and np.all(keep[ref[:16]] == 1)
    assert layer_error.keep_mask(order, 0).sum() == 0
    assert layer_error.keep_mask(order, 300).sum() == 300


def test_budget_golden():
    g = load_golden("aqlora_budget.json")
    assert layer_error.k_from_budget(g["rho"], g["n_linear_layers"]) == g["K"]


def test_zero_matrix_error_is_zero():
    assert layer_error.layer_error(np.zeros(128, np.uint16)) == 0.0


def test_storage_golden_65b():
    g = load_golden("storage_65b.json")
    n = g["n_weights"]
    assert n * 16 / 8 / 1e9 == g["gb_16bit"]
    assert n * 4 / 8 / 1e9 == g["gb_4bit"]
    assert float(storage.scale_bits_per_weight(False)) == g["scale_bits_nodq"]
    dq_bits = float(storage.scale_bits_per_weight(True))
    assert round(dq_bits, 3) == g["scale_bits_dq_approx"]
    assert round(float(storage.bits_per_weight(True)) * n / 8 / 1e9, 1) == g["gb_4bit_dq"]
    assert round(g["scale_bits_nodq"] * n / 8 / 1e9, 1) == g["gb_scales_nodq_approx"]
    assert round(dq_bits * n / 8 / 1e9) == g["gb_scales_dq_approx"]
    assert round(g["scale_bits_nodq"] - dq_bits, 2) == g["saving_bits_approx"]
    assert round((g["scale_bits_nodq"] - dq_bits) * n / 8 / 1e9) == g["saving_gb_approx"]
    bb = storage.buffer_bytes(64 * 256 * 10, True)
    assert bb == dict(codes=64 * 256 * 5, absmax_q=2560, absmax2=40, total=64 * 256 * 5 + 2600)


def test_storage_matches_oracle_buffers():
    rng = np.random.default_rng(5)
    w = rng.standard_normal((64, 1024)).astype(np.float32)
    for dq in (False, True):
        qw = nf4.quantize(w, double_quant=dq)
        bb = storage.buffer_bytes(w.size, dq)
        assert qw["codes"].nbytes == bb["codes"]
        if dq:
            assert qw["absmax_q"].nbytes == bb["absmax_q"] and qw["absmax2"].nbytes == bb["absmax2"]
        else:
            assert qw["absmax"].nbytes == bb["absmax"]


def test_memory_budget_rule_by_hand():
    """Three 64 x 64 layers without double quant: NF4 storage 2048 code bytes + 64
    fp32 scales = 2304 bytes, bf16 8192 bytes, so each kept layer adds 5888 bytes;
    with double quant 2048 + 64 + 4 = 2116 bytes, adding 6076. The budget is
    inclusive and the cut follows the ranking, not the layer ids."""
    assert layer_error.protect_cost_bytes(4096, False) == 5888
    assert layer_error.protect_cost_bytes(4096, True) == 6076
    order = [2, 0, 1]
    numel = [4096, 4096 * 4, 4096]
    # ranked costs: layer 2 -> 5888, layer 0 -> 5888, layer 1 (16384 weights) -> 4 * 5888
    for budget, K in [(0, 0), (5887, 0), (5888, 1), (11775, 1), (11776, 2), (11776 + 4 * 5888 - 1, 2),
                      (11776 + 4 * 5888, 3), (10 ** 12, 3)]:
        assert layer_error.k_under_memory_budget(order, numel, False, budget) == K, budget
    assert layer_error.k_under_memory_budget([1, 0, 2], numel, False, 4 * 5888 - 1) == 0   # big layer ranked first


def test_memory_budget_rule_is_monotone_and_a_prefix():
    rng = np.random.default_rng(3)
    numel = [int(64 * rng.integers(1, 5000)) for _ in range(40)]
    err = rng.random(40)
    order = layer_error.rank_layers(err)
    costs = [layer_error.protect_cost_bytes(n, True) for n in numel]
    prev = 0
    for budget in sorted(rng.integers(0, sum(costs) + 10, 200).tolist()):
        K = layer_error.k_under_memory_budget(order, numel, True, budget)
        assert K >= prev
        prev = K
        assert sum(costs[l] for l in order[:K]) <= budget
        assert K == len(order) or sum(costs[l] for l in order[:K + 1]) > budget
