"""Residual NF4 second stage for protected layers (oracle).

TEST INFRASTRUCTURE ONLY -- see ``oracle/__init__.py``.

[AQLoRA] "Additional controls" and section 8: instead of keeping a protected layer
in 16-bit, a second NF4 stage quantizes what the first stage missed; it matched
plain 16-bit protection at +3.6 % step time. The page gives no formula.

Readings (where the page is silent):
* the residual is R = fp32_rn(w - v1) with v1 = fp32_rn(c1 * a1) the first stage's
  value before any bf16 rounding (the first stage as ``nf4.quantize``);
* the second stage is ``nf4.quantize`` of R (fp32 input, IEEE quotient), with the
  same block size and its own double-quant setting;
* the reconstruction the GEMM consumes is bf16_rn(fp32_rn(v1 + v2)), v2 =
  fp32_rn(c2 * a2): both stages in fp32, one sum, one rounding to bf16.
"""
from __future__ import annotations

import numpy as np

from . import nf4


def residual_f32(w32: np.ndarray, qw1: dict) -> np.ndarray:
    """R = fp32_rn(w - v1), elementwise, in the weight's shape."""
    w32 = np.asarray(w32, dtype=np.float32).reshape(qw1["shape"])
    return (w32 - nf4.dequantize_f32(qw1)).astype(np.float32)


def quantize_residual(w32: np.ndarray, qw1: dict, double_quant: bool = False) -> dict:
    """The second NF4 stage: nf4.quantize of the first stage's residual."""
    return nf4.quantize(residual_f32(w32, qw1), double_quant=double_quant)


def dequantize_two_stage_bf16_bits(qw1: dict, qw2: dict) -> np.ndarray:
    """bf16_rn(fp32_rn(v1 + v2)) as bf16 bit patterns."""
    v = (nf4.dequantize_f32(qw1) + nf4.dequantize_f32(qw2)).astype(np.float32)
    return nf4.bf16_bits_from_f32(v)
