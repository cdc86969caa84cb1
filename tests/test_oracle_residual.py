"""Pins for the oracle's residual NF4 second stage."""
import numpy as np

from oracle import layer_error, nf4, residual


def _bf16(x):
    return nf4.f32_from_bf16_bits(nf4.bf16_bits_from_f32(np.asarray(x, np.float32)))


def test_exact_first_stage_leaves_a_zero_residual():
    """Weights that are exact first-stage values (code * a, a = the block's largest
    code value) have R = 0: the second stage is all zero codes with zero scales and
    the two-stage reconstruction equals the one-stage one."""
    c = nf4.nf4_code_table()
    rng = np.random.default_rng(0)
    idx = rng.integers(0, 16, (4, 64))
    idx[:, 0] = 15                                   # code 1.0 sets the absmax to a
    a = np.float32(0.0625)
    w = (c[idx] * a).astype(np.float32)              # products with a power of two: exact
    qw1 = nf4.quantize(w)
    assert np.array_equal(residual.residual_f32(w, qw1), np.zeros_like(w))
    qw2 = residual.quantize_residual(w, qw1)
    assert np.all(qw2["absmax"] == 0)
    assert np.all(nf4.unpack_nibbles(qw2["codes"], w.size) == nf4.ZERO_CODE)
    assert np.array_equal(residual.dequantize_two_stage_bf16_bits(qw1, qw2), nf4.dequantize_bf16_bits(qw1))


def _rn_f32(q):
    """Round an exact rational to the nearest fp32 (ties to even), by comparing the
    two fp32 neighbours found around a float approximation."""
    from fractions import Fraction
    x = np.float32(float(q))
    best = None
    for cand in (np.nextafter(x, np.float32(-np.inf)), x, np.nextafter(x, np.float32(np.inf))):
        d = abs(Fraction(float(cand)) - q)
        key = (d, int(np.float32(cand).view(np.uint32)) & 1)
        if best is None or key < best[0]:
            best = (key, cand)
    return np.float32(best[1])


def test_residual_and_two_stage_sum_follow_exact_rounding():
    """Every residual is the exact difference w - c1 a1 rounded once to fp32, and
    every two-stage value is the exact sum of the rounded stage values rounded once
    to fp32 and then to bf16 (exact rational arithmetic on a sample of elements)."""
    from fractions import Fraction
    rng = np.random.default_rng(1)
    w = _bf16(rng.standard_normal((16, 128)) * 0.03 * (1 + 9 * (rng.random((16, 128)) < 0.05)))
    qw1 = nf4.quantize(w)
    R = residual.residual_f32(w, qw1).reshape(-1)
    qw2 = residual.quantize_residual(w, qw1)
    two = residual.dequantize_two_stage_bf16_bits(qw1, qw2).reshape(-1)
    c = nf4.nf4_code_table()
    i1 = nf4.unpack_nibbles(qw1["codes"], w.size)
    i2 = nf4.unpack_nibbles(qw2["codes"], w.size)
    a1 = np.repeat(qw1["absmax"], 64)
    a2 = np.repeat(qw2["absmax"], 64)
    wf = w.reshape(-1)
    for e in rng.choice(w.size, 300, replace=False):
        v1 = _rn_f32(Fraction(float(c[i1[e]])) * Fraction(float(a1[e])))
        assert R[e] == _rn_f32(Fraction(float(wf[e])) - Fraction(float(v1))), e
        v2 = _rn_f32(Fraction(float(c[i2[e]])) * Fraction(float(a2[e])))
        s = _rn_f32(Fraction(float(v1)) + Fraction(float(v2)))
        assert two[e] == nf4.bf16_bits_from_f64(np.array([float(s)]))[0], e


def test_second_stage_reduces_the_error_on_normal_weights():
    """On N(0, 0.02^2) bf16 weights the two-stage reconstruction has a much smaller
    relative Frobenius error than one stage (the residual's blocks are rescaled
    to the full code range)."""
    rng = np.random.default_rng(2)
    w = _bf16(rng.standard_normal((128, 256)) * 0.02)
    qw1 = nf4.quantize(w)
    qw2 = residual.quantize_residual(w, qw1)
    one = nf4.f32_from_bf16_bits(nf4.dequantize_bf16_bits(qw1)).astype(np.float64).reshape(w.shape)
    two = nf4.f32_from_bf16_bits(residual.dequantize_two_stage_bf16_bits(qw1, qw2)).astype(np.float64).reshape(w.shape)
    w64 = w.astype(np.float64)
    e1 = np.linalg.norm(w64 - one) / np.linalg.norm(w64)
    e2 = np.linalg.norm(w64 - two) / np.linalg.norm(w64)
    assert e2 < e1 / 4, (e1, e2)
    assert abs(e1 - layer_error.layer_error(nf4.bf16_bits_from_f32(w))) < 1e-12
