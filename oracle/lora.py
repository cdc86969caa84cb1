"""NF4-LoRA linear forward and backward in fp64 (oracle).

TEST INFRASTRUCTURE ONLY -- see ``oracle/__init__.py``.

Forward, [QLoRA-blog] "The algebra", eq. (3):  Y = X W + s X L1 L2, with the
frozen W of shape h x o, L1 of shape h x r, L2 of shape r x o; s = alpha / r
([LoRA-blog], eq. (3) with the alpha/r scaling made explicit).

Storage orientation (reading, nn.Linear layout used by the PEFT stack in
[QLoRA-notes]): the quantized weight is stored out x in, W_s = W^T, so
Y = X W_s^T + s T L2 with T = X L1.

Backward: the base is frozen -- gradient flows through the dequantized W to X
but no gradient is formed for W ([Lesson-17] warm-up: the 4-bit base is a
constant in the graph, read at high precision, no gradient stored;
[QLoRA-blog] "One training step"). With U = dY L2^T, differentiating eq. (3):
  dX  = dY W_s + s U L1^T
  dL2 = s T^T dY
  dL1 = s X^T U
All products are library matmuls in float64 on the exact bf16 input values.
"""
from __future__ import annotations

import numpy as np


def f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def forward(X, W_s, L1, L2, s: float):
    """Returns (Y, T) in fp64. X: M x h, W_s: o x h (dequantized), L1: h x r, L2: r x o."""
    X, W_s, L1, L2 = f64(X), f64(W_s), f64(L1), f64(L2)
    T = X @ L1
    Y = X @ W_s.T + s * (T @ L2)
    return Y, T


def backward(X, W_s, L1, L2, dY, s: float):
    """Returns dict(dX, dL1, dL2, U, T) in fp64 (no dW: the base is frozen)."""
    X, W_s, L1, L2, dY = f64(X), f64(W_s), f64(L1), f64(L2), f64(dY)
    T = X @ L1
    U = dY @ L2.T
    dX = dY @ W_s + s * (U @ L1.T)
    dL2 = s * (T.T @ dY)
    dL1 = s * (X.T @ U)
    return dict(dX=dX, dL1=dL1, dL2=dL2, U=U, T=T)


def merged_weight(W_s, L1, L2, s: float) -> np.ndarray:
    """Merged stored-layout weight W_s + s (L1 L2)^T ([LoRA-blog] "Serving models
    and switching tasks": W_merged = W_0 + (alpha/r) B A)."""
    return f64(W_s) + s * (f64(L1) @ f64(L2)).T


def merged_weight_bf16_bits(W_s, L1, L2, s: float) -> np.ndarray:
    """The merged weight stored in bf16: each element of merged_weight rounded once,
    to nearest even (reading: the merge is formed exactly and stored in the compute
    dtype; a negative s unmerges)."""
    from oracle import nf4
    return nf4.bf16_bits_from_f64(merged_weight(W_s, L1, L2, s))


def trainable_params(h: int, o: int, r: int) -> int:
    """LoRA parameter count r (h + o) ([LoRA-blog] "How much smaller is the trainable part?")."""
    return r * (h + o)


def rel_frobenius(a, ref) -> float:
    a, ref = f64(a), f64(ref)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(a - ref) / den) if den > 0 else float(np.linalg.norm(a))
