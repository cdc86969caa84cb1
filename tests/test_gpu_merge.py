"""GPU parity: LoRA merge / unmerge into the stored weight, and merge + NF4
re-quantization, against the oracle.

Both sides form W_hat + s (L1 L2)^T in fp64 and round once to bf16. The rank
sums are of exact products of bf16 values, so the two fp64 results are equal
whenever the sums are exact, which is nearly always; otherwise they differ by
summation order in the last fp64 bits, which can change the bf16 rounding only
for an element within a few fp64 ulps of a bf16 rounding midpoint. Such
elements accept either neighbouring bf16 value; all others must match bit for
bit, and the seeded cases assert that none actually differ."""
import numpy as np
import pytest
import torch

from oracle import lora, nf4
from quantized_lora_fine_b200 import api, synth
from tests.gpu_helpers import bits, f64_of_bf16, gpu_case, oracle_qweight, oracle_what

pytestmark = pytest.mark.gpu


def _near_midpoint(m, mag):
    """Elements of the exact merge m within 2^-40 of the terms' magnitude mag of a
    bf16 rounding midpoint, with the two bf16 values they may round to."""
    a = np.abs(m)
    b = nf4.bf16_bits_from_f64(a).astype(np.int64)

    def val(k):
        return nf4.f32_from_bf16_bits(np.clip(k, 0, 0x7F7F).astype(np.uint16)).astype(np.float64)

    v = val(b)
    mid_up, mid_dn = (v + val(b + 1)) / 2, (v + val(b - 1)) / 2
    near_up = np.abs(a - mid_up) <= mag * 2.0 ** -40
    near_dn = np.abs(a - mid_dn) <= mag * 2.0 ** -40
    other = np.where(near_up, b + 1, np.where(near_dn, b - 1, b))
    sign = np.where(np.signbit(m), 0x8000, 0)
    return near_up | near_dn, (np.clip(other, 0, 0x7F7F) | sign).astype(np.uint16)


def _compare_merge(got, W_s, L1, L2, s):
    """Bit-exact outside the near-midpoint set; there, either neighbour. Returns the
    number of elements that took the other neighbour."""
    m = lora.merged_weight(W_s, L1, L2, s)
    ref = nf4.bf16_bits_from_f64(m)
    near, other = _near_midpoint(m, np.abs(W_s) + abs(s) * (np.abs(L1) @ np.abs(L2)).T)
    got = got.reshape(ref.shape)
    bad = (got != ref) & ~(near & (got == other))
    assert not bad.any(), f"{int(bad.sum())} merged elements differ (e.g. at {np.argwhere(bad)[:3].tolist()})"
    return int(((got != ref) & near).sum())


def _check_merge(case: synth.LinearCase, protected=False, s=None):
    d = case.make(with_dy=False)
    s = case.scale if s is None else s
    W_s = f64_of_bf16(d["W"]) if protected else oracle_what(oracle_qweight(d["W"], case.double_quant))
    L1, L2 = f64_of_bf16(d["L1"]), f64_of_bf16(d["L2"])
    ref = lora.merged_weight_bf16_bits(W_s, L1, L2, s)
    g, w = gpu_case(d, case.double_quant, protected)
    got = api.lora_merge(w, g["L1"], g["L2"], s)
    torch.cuda.synchronize()
    assert api.status() == 0
    flipped = _compare_merge(bits(got), W_s, L1, L2, s)
    assert flipped == 0, f"{flipped} near-midpoint elements rounded the other way"
    return d, g, w, W_s, L1, L2, ref


def test_merge_small_case(cuda_device):
    _check_merge(synth.case_small())


@pytest.mark.parametrize("dq", [False, True])
def test_merge_ragged_rows_and_ranks(cuda_device, dq):
    # out = 200 is not a multiple of the 64-row tile; r = 40 and 72 cross the 32-wide rank chunk
    for r in (40, 72):
        _check_merge(synth.LinearCase("merge-ragged", M=1, out=200, inp=320, r=r, alpha=16.0, double_quant=dq,
                                      seed=3))


@pytest.mark.parametrize("dq", [False, True])
def test_merge_unaligned_adapter_rows(cuda_device, dq):
    # r = 12 and out = 100: adapter rows are not whole 16-byte pieces (plain-load staging)
    case = synth.LinearCase("merge-odd", M=1, out=100, inp=192, r=12, alpha=24.0, double_quant=dq, seed=9)
    _check_merge(case)
    _check_requant(case, dq_out=dq, keep_absmax=True)


def test_merge_misaligned_adapter_pointers(cuda_device):
    """Adapters that start 2 bytes past a 16-byte boundary take the plain-load path and
    give the same bits."""
    case = synth.LinearCase("merge-misaligned", M=1, out=256, inp=256, r=16, alpha=32.0, double_quant=True, seed=10)
    d, g, w, W_s, L1, L2, ref = _check_merge(case)
    def shifted(t):
        buf = torch.empty(t.numel() + 1, dtype=t.dtype, device=t.device)
        v = buf[1:].view(t.shape)
        v.copy_(t)
        assert v.data_ptr() % 16 != 0
        return v
    got = api.lora_merge(w, shifted(g["L1"]), shifted(g["L2"]), case.scale)
    torch.cuda.synchronize()
    assert np.array_equal(bits(got).reshape(ref.shape), ref)


def test_merge_q_proj_shape(cuda_device):
    _check_merge(synth.LinearCase("merge-q_proj", M=1, out=4096, inp=4096, r=16, alpha=32.0, double_quant=True))


def test_merge_protected_bf16_weight(cuda_device):
    _check_merge(synth.LinearCase("merge-bf16", M=1, out=256, inp=512, r=8, alpha=16.0, double_quant=False, seed=4),
                 protected=True)


def test_unmerge_returns_the_weight(cuda_device):
    """Merging with s and then -s: both steps match the oracle bit for bit, and the
    unmerged weight is within one bf16 rounding of the original."""
    case = synth.LinearCase("merge-unmerge", M=1, out=256, inp=512, r=8, alpha=16.0, double_quant=False, seed=5)
    d, g, w, W_s, L1, L2, ref = _check_merge(case)
    merged = torch.from_numpy(np.ascontiguousarray(ref).view(np.int16)).view(torch.bfloat16).reshape(case.out, case.inp).cuda()
    back = api.lora_merge(api.NF4Weight.protected(merged), g["L1"], g["L2"], -case.scale)
    torch.cuda.synchronize()
    Wm = nf4.f32_from_bf16_bits(ref).astype(np.float64).reshape(case.out, case.inp)
    ref_back = lora.merged_weight_bf16_bits(Wm, L1, L2, -case.scale)
    assert _compare_merge(bits(back), Wm, L1, L2, -case.scale) == 0
    assert np.array_equal(bits(back).reshape(ref_back.shape), ref_back)
    err = np.abs(f64_of_bf16(back).reshape(W_s.shape) - W_s)
    assert np.all(err <= np.abs(W_s) * 2.0 ** -7 + abs(case.scale) * (np.abs(L1) @ np.abs(L2)).T * 2.0 ** -7 + 1e-30)


def _check_requant(case: synth.LinearCase, dq_out: bool, keep_absmax: bool, protected=False):
    """Codes and scales of the re-quantized merged weight equal the oracle's
    quantization of the oracle's merged bf16 weight."""
    d, g, w, W_s, L1, L2, ref = _check_merge(case, protected=protected)
    qw = nf4.quantize(nf4.f32_from_bf16_bits(ref).reshape(case.out, case.inp), double_quant=dq_out)
    o = api.lora_merge_requantize(w, g["L1"], g["L2"], case.scale, double_quant=dq_out, keep_absmax=keep_absmax)
    torch.cuda.synchronize()
    assert api.status() == 0
    assert np.array_equal(o.codes.cpu().numpy(), qw["codes"]), "codes differ"
    if keep_absmax or not dq_out:
        assert np.array_equal(o.absmax.cpu().numpy().view(np.uint32), qw["absmax"].view(np.uint32)), "absmax differ"
    else:
        assert o.absmax is None
    if dq_out:
        assert np.array_equal(o.absmax_q.cpu().numpy(), qw["absmax_q"]), "absmax_q differ"
        assert np.array_equal(o.absmax2.cpu().numpy().view(np.uint32), qw["absmax2"].view(np.uint32))
    return o


@pytest.mark.parametrize("dq", [False, True])
def test_merge_requantize_matches_oracle(cuda_device, dq):
    case = synth.LinearCase("merge-requant", M=1, out=384, inp=1024, r=16, alpha=32.0, double_quant=dq, seed=6)
    _check_requant(case, dq_out=dq, keep_absmax=True)
    _check_requant(case, dq_out=not dq, keep_absmax=False)


@pytest.mark.parametrize("r", [40, 72])
def test_merge_requantize_ragged(cuda_device, r):
    # 200 x 320: 1000 blocks, so the last double-quant group holds 232 scales; 200 rows
    # leave the second 128-row tile partly empty
    case = synth.LinearCase("merge-ragged", M=1, out=200, inp=320, r=r, alpha=16.0, double_quant=True, seed=3)
    _check_requant(case, dq_out=True, keep_absmax=False)
    _check_requant(case, dq_out=False, keep_absmax=False)


def test_merge_requantize_q_proj_shape(cuda_device):
    case = synth.LinearCase("merge-q_proj", M=1, out=4096, inp=4096, r=16, alpha=32.0, double_quant=True)
    _check_requant(case, dq_out=True, keep_absmax=True)


def test_merge_requantize_zero_blocks(cuda_device):
    """Rows whose weight and adapter rows are all zero merge to zero blocks: absmax 0,
    the zero code, and a double-quant group of such blocks gets a zero factor."""
    case = synth.LinearCase("merge-zero-rows", M=1, out=256, inp=1024, r=8, alpha=16.0, double_quant=False, seed=8)
    d = case.make(with_dy=False)
    d["W"][64:128] = 0           # 64 rows x 16 blocks = 1024 blocks: four whole double-quant groups
    d["L2"][:, 64:128] = 0
    W_s = f64_of_bf16(d["W"])
    L1, L2 = f64_of_bf16(d["L1"]), f64_of_bf16(d["L2"])
    ref = lora.merged_weight_bf16_bits(W_s, L1, L2, case.scale)
    qw = nf4.quantize(nf4.f32_from_bf16_bits(ref).reshape(case.out, case.inp), double_quant=True)
    assert np.all(qw["absmax"][64 * 16:128 * 16] == 0) and np.all(qw["absmax2"][4:8] == 0)
    g, w = gpu_case(d, False, protected=True)
    o = api.lora_merge_requantize(w, g["L1"], g["L2"], case.scale, double_quant=True, keep_absmax=True)
    torch.cuda.synchronize()
    assert api.status() == 0
    assert np.array_equal(o.codes.cpu().numpy(), qw["codes"])
    assert np.array_equal(o.absmax.cpu().numpy().view(np.uint32), qw["absmax"].view(np.uint32))
    assert np.array_equal(o.absmax_q.cpu().numpy(), qw["absmax_q"])
    assert np.array_equal(o.absmax2.cpu().numpy().view(np.uint32), qw["absmax2"].view(np.uint32))


def test_merge_requantize_nonfinite_sets_status(cuda_device):
    W = torch.zeros((128, 64), dtype=torch.bfloat16)
    W[5, 9] = float("inf")
    L1 = torch.zeros((64, 8), dtype=torch.bfloat16, device="cuda")
    L2 = torch.zeros((8, 128), dtype=torch.bfloat16, device="cuda")
    w = api.NF4Weight.protected(W.cuda())
    api.lora_merge_requantize(w, L1, L2, 2.0)
    torch.cuda.synchronize()
    assert api.status() == 8
    for ws in api.Workspace.all(torch.cuda.current_device()):
        api.reset_status(ws)
    assert api.status() == 0


def test_zero_adapter_merge_is_the_dequantized_weight(cuda_device):
    case = synth.LinearCase("merge-zero", M=1, out=128, inp=256, r=8, alpha=16.0, double_quant=True, seed=7)
    d = case.make(with_dy=False)
    g, w = gpu_case(d, True)
    z = torch.zeros_like(g["L2"])
    got = api.lora_merge(w, g["L1"], z, case.scale)
    torch.cuda.synchronize()
    assert np.array_equal(bits(got).reshape(-1), nf4.dequantize_bf16_bits(oracle_qweight(d["W"], True)).reshape(-1))


@pytest.mark.parametrize("exp,sigs", [(0, range(0, 128, 3)), (-120, range(0, 128, 9)), (-126, range(0, 128, 17)),
                                      (100, range(0, 128, 13)), (127, range(0, 128, 11))])
def test_merge_requantize_every_bf16_value(cuda_device, exp, sigs):
    """Blocks [a, x_1..x_63] holding every bf16 x with |x| <= a (a = (1 + s/128) 2^exp),
    merged with a zero adapter and re-quantized: codes and scales equal the oracle's
    quantization of the same values (this covers the power-of-two rescale that keeps
    the block reciprocal normal for tiny and huge blocks)."""
    from tests.test_gpu_codec import _exhaustive_blocks
    blocks = _exhaustive_blocks(exp, sigs)
    W = torch.from_numpy(nf4.bf16_bits_from_f32(blocks).view(np.int16)).view(torch.bfloat16).cuda()
    L1 = torch.zeros((64, 8), dtype=torch.bfloat16, device="cuda")
    L2 = torch.zeros((8, W.shape[0]), dtype=torch.bfloat16, device="cuda")
    qw = nf4.quantize(blocks, double_quant=False)
    o = api.lora_merge_requantize(api.NF4Weight.protected(W), L1, L2, 2.0, keep_absmax=True)
    torch.cuda.synchronize()
    assert api.status() == 0
    assert np.array_equal(o.codes.cpu().numpy(), qw["codes"])
    assert np.array_equal(o.absmax.cpu().numpy().view(np.uint32), qw["absmax"].view(np.uint32))


def test_linear_after_requantize_on_the_same_workspace(cuda_device):
    """Calls on one stream share one workspace: a merge + re-quantize (whose scratch
    holds fp32 scales) followed by the linear still gives the oracle's Y, i.e. the
    scratch stays clear of the split-K counters the linear relies on."""
    case = synth.LinearCase("after-requant", M=512, out=512, inp=768, r=16, alpha=32.0, double_quant=True, seed=11)
    d = case.make()
    g, w = gpu_case(d, True)
    api.lora_merge_requantize(w, g["L1"], g["L2"], case.scale, double_quant=True)
    Y, _ = api.linear_fwd(w, g["X"], g["L1"], g["L2"], case.scale)
    torch.cuda.synchronize()
    What = oracle_what(oracle_qweight(d["W"], True))
    X, L1, L2 = (f64_of_bf16(d[k]) for k in ("X", "L1", "L2"))
    Yref, _ = lora.forward(X, What, L1, L2, case.scale)
    from tests.gpu_helpers import assert_close
    assert_close(f64_of_bf16(Y), Yref, "Y")
