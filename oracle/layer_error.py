"""AQLoRA per-layer NF4 reconstruction error, ranking and top-K selection (oracle).

TEST INFRASTRUCTURE ONLY -- see ``oracle/__init__.py``.

[AQLoRA] 3.1: one data-free pass evaluates each linear layer's weights in
64-element blocks (bitsandbytes' NF4 layout) and computes a per-layer NF4
reconstruction error (the equation itself is missing from the extracted page).
[AQLoRA] 3.2: layers are ranked by that error and a fixed top-K cut keeps the
highest-error layers in 16-bit; K comes from the protection budget rho.

Readings (where the pages are silent):
* error = relative Frobenius norm e = sqrt(sum (w - w_hat)^2 / sum w^2) over
  the whole matrix, w the bf16 input widened to fp64 and w_hat the bf16
  dequantized value the GEMM would consume, with the layer's double-quant
  setting; an all-zero matrix has e = 0;
* "layer" = one linear matrix (the page counts 144 linear layers in phi-1.5);
* ranking: error descending, ties by matrix index ascending;
* K from rho: round half up of rho * L (the only pin: 0.2 * 144 -> 29).
* K from a memory budget ([AQLoRA] keeps the top-K in 16-bit "under a memory
  budget"): the budget counts the bytes a kept layer adds to the all-NF4 model,
  i.e. its bf16 size minus its NF4 storage (codes and scales, as the format
  stores them); K is the longest prefix of the ranking whose added bytes fit.
"""
from __future__ import annotations

from fractions import Fraction
from typing import Sequence, Tuple

import numpy as np

from . import nf4, storage


def layer_sums(w_bf16_bits: np.ndarray, double_quant: bool = False) -> Tuple[float, float]:
    """(sum (w - w_hat)^2, sum w^2) in fp64 for one matrix given as bf16 bits."""
    w32 = nf4.f32_from_bf16_bits(w_bf16_bits)
    qw = nf4.quantize(w32, double_quant=double_quant)
    w_hat = nf4.f32_from_bf16_bits(nf4.dequantize_bf16_bits(qw)).astype(np.float64)
    w = w32.astype(np.float64).reshape(w_hat.shape)
    d = w - w_hat
    return float(np.sum(d * d)), float(np.sum(w * w))


def layer_error(w_bf16_bits: np.ndarray, double_quant: bool = False) -> float:
    sd, sw = layer_sums(w_bf16_bits, double_quant)
    return float(np.sqrt(sd / sw)) if sw > 0 else 0.0


def rank_layers(err: Sequence[float]) -> np.ndarray:
    """Layer indices sorted by (error descending, index ascending)."""
    e = list(err)
    return np.array(sorted(range(len(e)), key=lambda i: (-e[i], i)), dtype=np.int32)


def keep_mask(order: np.ndarray, K: int) -> np.ndarray:
    """keep[l] = 1 iff layer l is among the first K of ``order`` ([AQLoRA] 3.2)."""
    keep = np.zeros(len(order), dtype=np.uint8)
    keep[np.asarray(order[:max(0, K)], dtype=np.int64)] = 1
    return keep


def k_from_budget(rho, n_layers: int) -> int:
    """K = round half up of rho * L, in exact rational arithmetic."""
    x = Fraction(str(rho)) * n_layers
    return int((x + Fraction(1, 2)) // 1)


def protect_cost_bytes(numel: int, double_quant: bool) -> int:
    """Bytes that keeping one layer in bf16 adds to its NF4 storage."""
    return 2 * numel - storage.buffer_bytes(numel, double_quant)["total"]


def k_under_memory_budget(order: Sequence[int], numel: Sequence[int], double_quant: bool,
                          budget_bytes: int) -> int:
    """Largest K such that the top-K layers of ``order`` add at most budget_bytes."""
    used, K = 0, 0
    for l in order:
        used += protect_cost_bytes(int(numel[int(l)]), double_quant)
        if used > budget_bytes:
            break
        K += 1
    return K
