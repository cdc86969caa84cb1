"""GPU parity: NF4 quantize / dequantize are bit-exact with the oracle."""
import numpy as np
import pytest
import torch

from oracle import nf4
from quantized_lora_fine_b200 import api, synth
from tests.gpu_helpers import bits

pytestmark = pytest.mark.gpu


def _check_quant(W: torch.Tensor, dq: bool):
    qw = nf4.quantize(nf4.f32_from_bf16_bits(bits(W)).reshape(W.shape), double_quant=dq)
    g = api.quantize(W.cuda(), double_quant=dq, keep_absmax=True)
    torch.cuda.synchronize()
    assert np.array_equal(g.codes.cpu().numpy(), qw["codes"]), "codes differ"
    assert np.array_equal(g.absmax.cpu().numpy().view(np.uint32), qw["absmax"].view(np.uint32)), "absmax differ"
    if dq:
        assert np.array_equal(g.absmax_q.cpu().numpy(), qw["absmax_q"]), "absmax_q differ"
        assert np.array_equal(g.absmax2.cpu().numpy().view(np.uint32), qw["absmax2"].view(np.uint32)), "absmax2 differ"
    deq = api.dequantize(g)
    torch.cuda.synchronize()
    assert np.array_equal(bits(deq).reshape(-1), nf4.dequantize_bf16_bits(qw).reshape(-1)), "dequantized values differ"
    assert api.status() == 0


def test_quant_small_case(cuda_device):
    d = synth.case_small().make()
    _check_quant(d["W"], dq=False)


@pytest.mark.parametrize("dq", [False, True])
def test_quant_q_proj_shape(cuda_device, dq):
    W = synth.normal_bf16((4096, 4096), 0.02, 0, synth.STREAM_W)
    _check_quant(W, dq)


def test_quant_student_t_ragged_groups(cuda_device):
    # 11008 x 256: 44032 blocks = 172 groups exactly; plus a shape whose last DQ group is partial
    _check_quant(synth.student_t_bf16((11008, 256), 5.0, 0.02, 0, synth.STREAM_W), dq=True)
    _check_quant(synth.student_t_bf16((300, 192), 3.0, 0.02, 1, synth.STREAM_W), dq=True)


def test_double_quant_hand_worked_group(cuda_device):
    """The hand-worked double-quant group of the oracle's pins (block maxima
    203 * 2^-20 and 49 * 2^-12): E4M3 scale bytes 0x4F and 0x7E, factor 7 * 2^-18,
    through the GPU quantizer and through the fused allocation pass."""
    W = torch.zeros((2, 64), dtype=torch.float32)
    W[0, 11] = -203 * 2.0 ** -20
    W[1, 40] = 49 * 2.0 ** -12
    W[0, 3] = 2.0 ** -20          # a smaller weight in each block, so the codes are not all zero
    W[1, 5] = -2.0 ** -9
    Wb = W.to(torch.bfloat16)
    g = api.quantize(Wb.cuda(), double_quant=True)
    torch.cuda.synchronize()
    assert g.absmax_q.cpu().tolist() == [0x4F, 0x7E]
    assert g.absmax2.cpu().tolist() == [7 * 2.0 ** -18]
    _check_quant(Wb, dq=True)
    _, _, _, outs = api.quantize_error_rank([Wb.cuda()], 0, double_quant=True)
    torch.cuda.synchronize()
    assert outs[0].absmax_q.cpu().tolist() == [0x4F, 0x7E]
    assert outs[0].absmax2.cpu().tolist() == [7 * 2.0 ** -18]


def test_quant_partial_tail_block(cuda_device):
    W = synth.normal_bf16((7, 38), 0.5, 2, synth.STREAM_W)   # 266 elements: 4 full blocks + 10
    _check_quant(W, dq=False)
    _check_quant(W, dq=True)


def test_quant_adversarial_blocks(cuda_device):
    C = nf4.nf4_code_table()
    mids = nf4.nf4_midpoints()
    rows = []
    rows.append(np.zeros(64, np.float32))                                   # all-zero block
    r = np.zeros(64, np.float32); r[5] = 3.0; rows.append(r)                 # one non-zero
    r = np.full(64, -0.0, np.float32); rows.append(r)                        # negative zeros
    r = np.concatenate([[1.0], mids, -mids, C, np.nextafter(mids, 2), np.nextafter(mids, -2)]).astype(np.float32)
    rows.append(np.resize(r, 64))
    rows.append(np.resize(np.concatenate([[1.0], np.nextafter(mids, 2)]), 64).astype(np.float32))
    r = (C[np.arange(64) % 16] * np.float32(0.75)).astype(np.float32); rows.append(r)
    r = np.full(64, 2.0 ** -130, np.float32); r[0] = 2.0 ** -126; rows.append(r)   # subnormal range
    r = np.linspace(-3e38, 3e38, 64).astype(np.float32); rows.append(r)            # huge
    W32 = np.stack(rows)
    Wb = synth.from_bf16_bits(nf4.bf16_bits_from_f32(W32))
    _check_quant(Wb, dq=False)
    _check_quant(Wb, dq=True)
    # fp32 input path
    qw = nf4.quantize(W32)
    g = api.quantize(torch.from_numpy(W32).cuda(), double_quant=False)
    assert np.array_equal(g.codes.cpu().numpy(), qw["codes"])


def test_nonfinite_sets_status(cuda_device):
    W = torch.zeros((4, 64), dtype=torch.bfloat16)
    W[2, 7] = float("nan")
    ws = api.Workspace.get(256, torch.device("cuda:0"))
    api.reset_status(ws)
    api.quantize(W.cuda())
    assert api.read_status(ws) == 8
    api.reset_status(ws)
    assert api.read_status(ws) == 0


def _exhaustive_blocks(exp: int, sigs) -> np.ndarray:
    """Blocks [a, x_1..x_63] for every bf16 x with |x| <= a, a = (1 + s/128) 2^exp."""
    allb = nf4.f32_from_bf16_bits(np.arange(65536, dtype=np.uint32).astype(np.uint16))
    allb = allb[np.isfinite(allb)]
    blocks = []
    for s in sigs:
        a = np.float32((1 + s / 128.0) * 2.0 ** exp)
        x = allb[np.abs(allb) <= a]
        pad = (-x.size) % 63
        x = np.concatenate([x, np.zeros(pad, np.float32)]).reshape(-1, 63)
        blocks.append(np.concatenate([np.full((x.shape[0], 1), a, np.float32), x], axis=1))
    return np.concatenate(blocks)


@pytest.mark.parametrize("exp,sigs", [(0, range(128)), (-120, range(0, 128, 9)), (-126, range(0, 128, 17)),
                                      (100, range(0, 128, 13)), (127, range(0, 128, 11))])
def test_quant_every_bf16_pair(cuda_device, exp, sigs):
    """Every (bf16 w, bf16 absmax) significand pair and exponent gap: the GPU's
    reciprocal-based quotient and cell-table code lookup give the oracle's codes
    (IEEE division, 15 midpoint comparisons); tiny (2^-126, 2^-120) and huge
    (2^100, 2^127) absmax take the rescaled path."""
    W32 = _exhaustive_blocks(exp, sigs)
    Wb = synth.from_bf16_bits(nf4.bf16_bits_from_f32(W32))
    _check_quant(Wb, dq=False)


def test_quant_stack_gate_matrix_full_size(cuda_device):
    """A full 11008 x 4096 gate matrix of the stack (scale * Student-t), with and
    without double quant."""
    m = synth.stack_matrices()[4]
    W = synth.stack_weight(m)
    _check_quant(W, dq=False)
    _check_quant(W, dq=True)


@pytest.mark.parametrize("dq", [False, True])
def test_quantize_batch_matches_single_calls(cuda_device, dq):
    """One batched launch over matrices of several shapes (one with a ragged last
    block, one smaller than a group) gives every matrix the bits of its own call."""
    shapes = [(512, 512), (11, 66), (3, 20000), (64, 256), (1, 6)]
    Ws = [synth.normal_bf16(sh, 0.02, 0, 1, i, device="cuda") for i, sh in enumerate(shapes)]
    outs = api.quantize_batch(Ws, double_quant=dq, keep_absmax=True)
    for W, o in zip(Ws, outs):
        ref = api.quantize(W, double_quant=dq, keep_absmax=True)
        assert torch.equal(o.codes, ref.codes)
        assert torch.equal(o.absmax.view(torch.int32), ref.absmax.view(torch.int32))
        if dq:
            assert torch.equal(o.absmax_q, ref.absmax_q)
            assert torch.equal(o.absmax2.view(torch.int32), ref.absmax2.view(torch.int32))
    assert api.status() == 0


def test_quantize_batch_stack_layer(cuda_device):
    """The seven matrices of one decoder layer of the 7B stack in one launch give the
    bits of seven single calls (which the tests above hold to the oracle)."""
    mats = synth.stack_matrices(n_layers=1)
    Ws = [synth.stack_weight(m, device="cuda") for m in mats]
    outs = api.quantize_batch(Ws, double_quant=True)
    for W, o in zip(Ws, outs):
        ref = api.quantize(W, double_quant=True)
        assert torch.equal(o.codes, ref.codes) and torch.equal(o.absmax_q, ref.absmax_q)
        assert torch.equal(o.absmax2.view(torch.int32), ref.absmax2.view(torch.int32))
    assert api.status() == 0
