"""GPU parity: the residual NF4 second stage (codes and scales bit-exact) and the
two-stage reconstruction (bf16 bits exact) against the oracle; a two-stage layer
through the linear within the GEMM tolerances."""
import numpy as np
import pytest
import torch

from oracle import lora, nf4, residual
from quantized_lora_fine_b200 import api, synth
from tests.gpu_helpers import assert_close, bits, f64_of_bf16

pytestmark = pytest.mark.gpu


def _check(W: torch.Tensor, dq1: bool, dq2: bool):
    w32 = nf4.f32_from_bf16_bits(bits(W)).reshape(W.shape)
    qw1 = nf4.quantize(w32, double_quant=dq1)
    qw2 = residual.quantize_residual(w32, qw1, double_quant=dq2)
    g = W.cuda()
    w1 = api.quantize(g, double_quant=dq1)
    w2 = api.quantize_residual(g, w1, double_quant=dq2, keep_absmax=True)
    two = api.dequantize_two_stage(w1, w2)
    torch.cuda.synchronize()
    assert api.status() == 0
    assert np.array_equal(w2.codes.cpu().numpy(), qw2["codes"]), "stage-2 codes differ"
    assert np.array_equal(w2.absmax.cpu().numpy().view(np.uint32), qw2["absmax"].view(np.uint32))
    if dq2:
        assert np.array_equal(w2.absmax_q.cpu().numpy(), qw2["absmax_q"])
        assert np.array_equal(w2.absmax2.cpu().numpy().view(np.uint32), qw2["absmax2"].view(np.uint32))
    ref = residual.dequantize_two_stage_bf16_bits(qw1, qw2)
    assert np.array_equal(bits(two).reshape(-1), ref.reshape(-1)), "two-stage values differ"
    return w1, w2, two, ref


@pytest.mark.parametrize("dq1,dq2", [(False, False), (True, False), (False, True), (True, True)])
def test_residual_stage_small(cuda_device, dq1, dq2):
    _check(synth.student_t_bf16((256, 512), 5.0, 0.02, 0, synth.STREAM_W), dq1, dq2)


def test_residual_stage_ragged_groups(cuda_device):
    # 300 x 192 = 900 blocks: the last double-quant group holds 132 scales
    _check(synth.student_t_bf16((300, 192), 3.0, 0.02, 1, synth.STREAM_W), True, True)


def test_residual_stage_q_proj_shape(cuda_device):
    _check(synth.normal_bf16((4096, 4096), 0.02, 0, synth.STREAM_W), True, True)


def test_two_stage_layer_through_the_linear(cuda_device):
    """A layer stored as two NF4 stages runs through the protected (bf16) path on its
    two-stage reconstruction; Y and the gradients match the oracle on that weight."""
    case = synth.LinearCase("two-stage", M=512, out=512, inp=768, r=16, alpha=32.0, double_quant=True, seed=2)
    d = case.make()
    w1, w2, two, ref = _check(d["W"], True, True)
    g = {k: v.cuda() for k, v in d.items()}
    wp = api.NF4Weight.protected(two)
    Y, T = api.linear_fwd(wp, g["X"], g["L1"], g["L2"], case.scale)
    dX, dL1, dL2 = api.linear_bwd(wp, g["X"], g["dY"], g["L1"], g["L2"], case.scale, T=T)
    torch.cuda.synchronize()
    W2 = nf4.f32_from_bf16_bits(ref).astype(np.float64).reshape(case.out, case.inp)
    X, L1, L2, dY = (f64_of_bf16(d[k]) for k in ("X", "L1", "L2", "dY"))
    Yref, _ = lora.forward(X, W2, L1, L2, case.scale)
    gref = lora.backward(X, W2, L1, L2, dY, case.scale)
    assert_close(f64_of_bf16(Y), Yref, "Y")
    assert_close(f64_of_bf16(dX), gref["dX"], "dX")
    assert_close(dL1.cpu().numpy(), gref["dL1"], "dL1")
    assert_close(dL2.cpu().numpy(), gref["dL2"], "dL2")
