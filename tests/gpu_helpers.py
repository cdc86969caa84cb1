"""Shared helpers for the GPU parity tests: run the oracle and the CUDA path on
the same seeded inputs and compare."""
import numpy as np
import torch

from oracle import lora, nf4
from quantized_lora_fine_b200 import api, synth

REL_FRO_TOL = 5e-3          # relative Frobenius error bound for GEMM outputs / gradients
MAX_ABS_FRAC = 1e-2         # max |diff| <= 1e-2 * max |ref|


def bits(t: torch.Tensor) -> np.ndarray:
    return synth.bf16_bits(t)


def f64_of_bf16(t: torch.Tensor) -> np.ndarray:
    return nf4.f32_from_bf16_bits(bits(t)).astype(np.float64)


def assert_close(got, ref, name, rel=REL_FRO_TOL, frac=MAX_ABS_FRAC):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{name}: non-finite output"
    rf = lora.rel_frobenius(got, ref)
    mx = float(np.max(np.abs(got - ref))) if got.size else 0.0
    lim = frac * float(np.max(np.abs(ref))) if ref.size else 0.0
    assert rf <= rel, f"{name}: relative Frobenius error {rf:.3e} > {rel:.1e}"
    assert mx <= lim, f"{name}: max abs error {mx:.3e} > {lim:.3e}"
    return rf, mx


def oracle_qweight(W: torch.Tensor, dq: bool) -> dict:
    return nf4.quantize(nf4.f32_from_bf16_bits(bits(W)).reshape(W.shape), double_quant=dq)


def oracle_what(qw: dict) -> np.ndarray:
    return nf4.f32_from_bf16_bits(nf4.dequantize_bf16_bits(qw)).astype(np.float64).reshape(qw["shape"])


def gpu_case(d: dict, dq: bool, protected: bool = False):
    dev = torch.device("cuda:0")
    g = {k: (v.to(dev) if v is not None else None) for k, v in d.items()}
    w = api.NF4Weight.protected(g["W"]) if protected else api.quantize(g["W"], double_quant=dq)
    return g, w
