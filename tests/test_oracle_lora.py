"""Pins for the oracle's LoRA forward / backward (fp64).

Checks against: explicit scalar loops on tiny shapes (brute force), the merge
identity from the LoRA page, the zero-init special case, central finite
differences, adjoint identities and the pages' parameter counts.
"""
import numpy as np
import pytest

from oracle import lora, nf4
from tests.conftest import load_golden


def _tiny(seed=0, M=5, h=6, o=7, r=3):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((M, h)), rng.standard_normal((o, h)), rng.standard_normal((h, r)),
            rng.standard_normal((r, o)), rng.standard_normal((M, o)))


def pin_forward_loops(fwd=lora.forward):
    X, W, L1, L2, _ = _tiny()
    s = 1.75
    Y, T = fwd(X, W, L1, L2, s)
    M, h = X.shape
    o, r = W.shape[0], L1.shape[1]
    for i in range(M):
        for j in range(o):
            base = sum(X[i, k] * W[j, k] for k in range(h))
            ad = sum(sum(X[i, k] * L1[k, q] for k in range(h)) * L2[q, j] for q in range(r))
            assert abs(Y[i, j] - (base + s * ad)) < 1e-12 * (1 + abs(Y[i, j]))
    for i in range(M):
        for q in range(r):
            assert abs(T[i, q] - sum(X[i, k] * L1[k, q] for k in range(h))) < 1e-12


def pin_backward_fd(fwd=lora.forward, bwd=lora.backward):
    """Central differences of L = sum(Y * G) match the analytic gradients."""
    X, W, L1, L2, G = _tiny(1, M=4, h=5, o=6, r=2)
    s = 0.5
    g = bwd(X, W, L1, L2, G, s)
    eps = 1e-6

    def loss(X_, L1_, L2_):
        return float(np.sum(fwd(X_, W, L1_, L2_, s)[0] * G))

    for name, arr in (("dX", X), ("dL1", L1), ("dL2", L2)):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            p = arr.copy(); p[idx] += eps
            m = arr.copy(); m[idx] -= eps
            args_p = {"dX": (p, L1, L2), "dL1": (X, p, L2), "dL2": (X, L1, p)}[name]
            args_m = {"dX": (m, L1, L2), "dL1": (X, m, L2), "dL2": (X, L1, m)}[name]
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        err = np.max(np.abs(num - g[name])) / max(1e-30, np.max(np.abs(g[name])))
        assert err < 1e-8, (name, err)


def pin_merge_identity(fwd=lora.forward):
    X, W, L1, L2, _ = _tiny(2)
    s = 2.0
    Y, _ = fwd(X, W, L1, L2, s)
    Wm = lora.merged_weight(W, L1, L2, s)
    assert np.allclose(Y, X @ Wm.T, rtol=1e-12, atol=1e-12)


def test_forward_matches_scalar_loops():
    pin_forward_loops()


def test_backward_matches_finite_differences():
    pin_backward_fd()


def test_merge_identity():
    pin_merge_identity()


def test_zero_init_is_plain_gemm():
    X, W, L1, L2, _ = _tiny(3)
    Y, _ = lora.forward(X, W, L1, np.zeros_like(L2), 2.0)
    assert np.array_equal(Y, X @ W.T)
    Y0, _ = lora.forward(X, W, L1, L2, 0.0)
    assert np.array_equal(Y0, X @ W.T)


def test_linearity_in_x():
    X, W, L1, L2, _ = _tiny(4)
    X2 = np.random.default_rng(9).standard_normal(X.shape)
    a, b = 0.75, -1.5
    lhs = lora.forward(a * X + b * X2, W, L1, L2, 2.0)[0]
    rhs = a * lora.forward(X, W, L1, L2, 2.0)[0] + b * lora.forward(X2, W, L1, L2, 2.0)[0]
    assert np.allclose(lhs, rhs, rtol=1e-12, atol=1e-12)


def test_adjoint_identities():
    X, W, L1, L2, dY = _tiny(5, M=9, h=8, o=10, r=4)
    s = 3.0
    Y, T = lora.forward(X, W, L1, L2, s)
    g = lora.backward(X, W, L1, L2, dY, s)
    assert np.isclose(np.sum(dY * Y), np.sum(g["dX"] * X), rtol=1e-12)
    assert np.isclose(np.sum(g["dL2"] * L2), s * np.sum(dY * (T @ L2)), rtol=1e-12)
    assert np.isclose(np.sum(g["dL1"] * L1), s * np.sum(dY * (X @ L1 @ L2)), rtol=1e-12)


def test_no_weight_gradient_is_formed():
    X, W, L1, L2, dY = _tiny(6)
    g = lora.backward(X, W, L1, L2, dY, 1.0)
    assert set(g) == {"dX", "dL1", "dL2", "U", "T"}


def test_param_count_golden():
    gd = load_golden("lora_param_count.json")
    assert gd["r"] * gd["h"] == gd["lora_A"] and gd["r"] * gd["o"] == gd["lora_B"]
    assert lora.trainable_params(gd["h"], gd["o"], gd["r"]) == gd["both"]
    assert gd["h"] * gd["o"] == gd["full_matrix"] and gd["full_matrix"] // gd["both"] == gd["ratio"]
    pg = load_golden("peft_trainable_llama7b.json")
    total = pg["n_layers"] * pg["modules_per_layer"] * lora.trainable_params(pg["h"], pg["o"], pg["r"])
    assert total == pg["trainable_params"]


# ----------------------------------------------------------------- planted mistakes

def test_pins_catch_planted_mistakes():
    """Each pin fails when a plausible mistake is planted in the oracle (CPU only)."""
    def fwd_no_scale(X, W, L1, L2, s):
        Y, T = lora.forward(X, W, L1, L2, 1.0)
        return Y, T

    def fwd_wrong_index(X, W, L1, L2, s):
        X, W, L1, L2 = (np.asarray(a, np.float64) for a in (X, W, L1, L2))
        T = X @ L1
        return X @ W.T + s * (T @ L2[::-1]), T          # rank index reversed in L2

    def bwd_sign_slip(X, W, L1, L2, dY, s):
        g = lora.backward(X, W, L1, L2, dY, s)
        g = dict(g)
        g["dL1"] = -g["dL1"]
        return g

    def bwd_dropped_term(X, W, L1, L2, dY, s):
        g = dict(lora.backward(X, W, L1, L2, dY, s))
        U = np.asarray(dY, np.float64) @ np.asarray(L2, np.float64).T
        g["dX"] = g["dX"] - s * (U @ np.asarray(L1, np.float64).T)
        return g

    with pytest.raises(AssertionError):
        pin_merge_identity(fwd_no_scale)
    with pytest.raises(AssertionError):
        pin_forward_loops(fwd_wrong_index)
    with pytest.raises(AssertionError):
        pin_backward_fd(bwd=bwd_sign_slip)
    with pytest.raises(AssertionError):
        pin_backward_fd(bwd=bwd_dropped_term)


def test_merged_bf16_is_the_rounded_merge():
    """merged_weight_bf16_bits rounds merged_weight once; merging with s and then -s
    from an exact merge returns the weight; a zero adapter merges to the weight."""
    rng = np.random.default_rng(7)
    W = nf4.f32_from_bf16_bits(nf4.bf16_bits_from_f32(rng.standard_normal((32, 64)).astype(np.float32) * 0.02))
    L1 = nf4.f32_from_bf16_bits(nf4.bf16_bits_from_f32(rng.standard_normal((64, 4)).astype(np.float32) * 0.01))
    L2 = nf4.f32_from_bf16_bits(nf4.bf16_bits_from_f32(rng.standard_normal((4, 32)).astype(np.float32) * 0.01))
    Wm = lora.merged_weight(W, L1, L2, 2.0)
    assert np.array_equal(lora.merged_weight_bf16_bits(W, L1, L2, 2.0), nf4.bf16_bits_from_f64(Wm))
    assert np.array_equal(lora.merged_weight(Wm, L1, L2, -2.0), W.astype(np.float64))
    zero = np.zeros_like(L2)
    assert np.array_equal(lora.merged_weight_bf16_bits(W, L1, zero, 2.0), nf4.bf16_bits_from_f32(W))
