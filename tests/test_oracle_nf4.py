"""Pins for the oracle's NF4 quantizer, double quantizer and dequantizer.

Every check here compares the oracle with something other than itself: the
defining quantile property via the forward normal CDF, exact rational brute
force, torch's CPU casts (bf16, float8_e4m3fn) as independent library
routines, closed-form identities and special cases.
"""
import numpy as np
import pytest
import scipy.special as sp
import torch

from oracle import nf4

C = nf4.nf4_code_table()
MID = nf4.nf4_midpoints()


# ----------------------------------------------------------------- pins (plain functions)

def pin_table_invariants():
    c = nf4.nf4_code_table()
    assert c.dtype == np.float32 and c.shape == (16,)
    assert np.all(np.diff(c) > 0), "codes must be strictly increasing"
    assert c[0] == -1.0 and c[15] == 1.0
    assert np.sum(c == 0.0) == 1 and c[nf4.ZERO_CODE] == 0.0
    assert np.sum(c < 0) == 7 and np.sum(c > 0) == 8


def pin_table_quantiles():
    """Positive codes sit at equally spaced probabilities between delta and 1/2
    (9-point grid), negative codes on the 8-point grid, through the forward CDF."""
    c = nf4.nf4_code_table().astype(np.float64)
    delta = 1.0 - 0.5 * (1.0 / 32 + 1.0 / 30)
    z = sp.ndtri(delta)  # normaliser, fixed by c[15] == 1
    p_pos = sp.ndtr(c[8:] * z)[::-1]          # from c15 down to c8
    grid_pos = np.linspace(delta, 0.5, 9)[:-1]
    assert np.allclose(p_pos, grid_pos, rtol=0, atol=2e-7), (p_pos, grid_pos)
    p_neg = sp.ndtr(-c[:7] * z)               # c0 .. c6
    grid_neg = np.linspace(delta, 0.5, 8)[:-1]
    assert np.allclose(p_neg, grid_neg, rtol=0, atol=2e-7), (p_neg, grid_neg)


def pin_bruteforce_codes(n_values):
    n_values = np.asarray(n_values, dtype=np.float32)
    w = n_values.reshape(-1)
    # absmax 1 via an explicit +1 element per block: append and quantize in blocks of 2
    blocks = np.stack([w, np.ones_like(w)], axis=1).reshape(-1)
    a = nf4.block_absmax(blocks, blocksize=2)
    idx = nf4.code_indices(blocks, a, blocksize=2)[0::2]
    mids = set(nf4.nf4_midpoints().tolist())
    for x, i in zip(w, idx):
        if float(x) in mids:
            # on an fp32 midpoint the rule n > m_j sends the value to the lower code
            j = sorted(mids).index(float(x))
            assert int(i) == j, (float(x), int(i))
        else:
            assert int(i) == nf4.nearest_code_bruteforce(float(x)), (float(x), int(i))


def pin_nibble_order():
    idx = np.array([1, 2, 15, 0, 7, 8], np.uint8)
    packed = nf4.pack_nibbles(idx)
    assert packed.tolist() == [0x12, 0xF0, 0x78]
    assert np.array_equal(nf4.unpack_nibbles(packed, 6), idx)


# ----------------------------------------------------------------- tests

def test_table_invariants():
    pin_table_invariants()


def test_table_quantile_property():
    pin_table_quantiles()


def test_table_independent_of_ndtri_route():
    d = 1 - (1 / 32 + 1 / 30) / 2
    pos = sp.ndtri(np.linspace(d, 0.5, 9)[:-1])
    neg = -sp.ndtri(np.linspace(d, 0.5, 8)[:-1])
    v = np.sort(np.concatenate([pos, neg, [0.0]])) / sp.ndtri(d)
    assert np.array_equal(v.astype(np.float32), C)


def test_midpoints_between_codes():
    assert MID.shape == (15,)
    assert np.all(C[:-1] < MID) and np.all(MID < C[1:])
    exact = (C[:-1].astype(np.float64) + C[1:].astype(np.float64)) / 2
    ulp = np.spacing(np.abs(MID)).astype(np.float64)
    assert np.all(np.abs(MID.astype(np.float64) - exact) <= ulp / 2)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * np.float32(3.0),
        (rng.standard_normal(50000) * 1e-38).astype(np.float32),            # subnormals
        np.array([0.0, -0.0, 1.0, -1.0, np.inf, -np.inf, 3.3895314e38, 1.00390625,
                  1.01171875, 1.0078125, 2.0 ** -133], np.float32),
        # exact ties: low 16 bits == 0x8000
        (rng.integers(0, 2 ** 31, 20000, dtype=np.uint32) & np.uint32(0xFFFF0000) | np.uint32(0x8000)).view(np.float32),
    ])
    x = x[np.isfinite(x) | np.isinf(x)]
    ours = nf4.bf16_bits_from_f32(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_e4m3_decode_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = nf4.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    both_nan = np.isnan(ours) & np.isnan(ref)
    assert np.all(both_nan | (ours == ref))
    assert np.sum(np.isnan(ours)) == 2


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(2)
    finite = nf4.e4m3_decode(np.arange(256, dtype=np.uint8))
    finite = finite[np.isfinite(finite)].astype(np.float64)
    pos = np.unique(np.abs(finite))
    ties = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)           # exact midpoints
    x = np.concatenate([
        (rng.uniform(-448, 448, 300000)).astype(np.float32),
        (rng.uniform(-0.03, 0.03, 100000)).astype(np.float32),      # subnormal range
        ties, -ties, finite.astype(np.float32),
        np.array([448.0, -448.0, 0.0, -0.0, 2.0 ** -10, 2.0 ** -11], np.float32),
    ])
    ours = nf4.e4m3_encode_satfinite(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_saturates():
    x = np.array([448.0, 449.0, 464.0, 480.0, 1e6, 3e38, -500.0], np.float32)
    assert nf4.e4m3_encode_satfinite(x).tolist() == [0x7E] * 6 + [0xFE]


def test_codes_match_rational_bruteforce():
    rng = np.random.default_rng(3)
    n = np.concatenate([rng.uniform(-1, 1, 3000), MID, -MID,
                        np.nextafter(MID, 2), np.nextafter(MID, -2), C]).astype(np.float32)
    n = n[np.abs(n) <= 1]
    pin_bruteforce_codes(n)


def test_exhaustive_bf16_sweep_against_bruteforce():
    """Block [a, x] for every bf16 x with |x| <= a, several a: threshold rule vs
    nearest code by exact distance; they may differ only where n equals an fp32
    midpoint that is not the exact midpoint."""
    all_bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    xs = nf4.f32_from_bf16_bits(all_bits)
    xs = xs[np.isfinite(xs)]
    exact_mid = (C[:-1].astype(np.float64) + C[1:].astype(np.float64)) / 2
    for a in (1.0, 0.0390625, 3.0, 2.0 ** -100, 1.5 * 2.0 ** 100):
        a32 = np.float32(a)
        x = xs[np.abs(xs) <= a32]
        blocks = np.stack([np.full_like(x, a32), x], axis=1).reshape(-1)
        am = nf4.block_absmax(blocks, blocksize=2)
        idx = nf4.code_indices(blocks, am, blocksize=2)[1::2].astype(np.int64)
        n = (x / a32).astype(np.float32).astype(np.float64)
        # brute force in fp64: nearest code; exact ties to the lower code
        d = np.abs(n[:, None] - C.astype(np.float64)[None, :])
        bf = np.argmin(d, axis=1)
        diff = idx != bf
        if diff.any():
            # only allowed where n sits exactly on an fp32 midpoint
            assert np.all(np.isin(n[diff].astype(np.float32), MID)), n[diff][:10]
        # rational check of near-ties (distances within 1e-12)
        srt = np.sort(d, axis=1)
        near = np.nonzero(srt[:, 1] - srt[:, 0] < 1e-12)[0]
        for k in near[:200]:
            assert idx[k] == nf4.nearest_code_bruteforce(float(n[k])) or np.float32(n[k]) in MID
        assert not np.any(np.isin(n.astype(np.float32), exact_mid[exact_mid == exact_mid.astype(np.float32)]) & diff)


def test_round_trip_identity_exact_codes():
    """dequant(quant(W)) == W for blocks of exact fp32 products c_i * a that
    contain a +-1 code (so the block absmax is a itself)."""
    rng = np.random.default_rng(4)
    nb = 512
    a = rng.uniform(0.01, 4.0, nb).astype(np.float32)
    idx = rng.integers(0, 16, (nb, 64)).astype(np.uint8)
    idx[:, 0] = rng.choice([0, 15], nb)
    w = (C[idx] * a[:, None]).astype(np.float32)
    qw = nf4.quantize(w.reshape(64, -1))
    assert np.array_equal(nf4.unpack_nibbles(qw["codes"], w.size), idx.reshape(-1))
    assert np.array_equal(qw["absmax"], a)
    assert np.array_equal(nf4.dequantize_f32(qw).reshape(-1), w.reshape(-1))
    assert np.array_equal(nf4.dequantize_bf16_bits(qw).reshape(-1), nf4.bf16_bits_from_f32(w.reshape(-1)))


def test_scale_invariance_power_of_two():
    rng = np.random.default_rng(5)
    w = (rng.standard_normal((32, 256)) * 0.02).astype(np.float32)
    base = nf4.quantize(w)
    for k in (-20, -3, 1, 7, 30):
        s = np.float32(2.0 ** k)
        qk = nf4.quantize(w * s)
        assert np.array_equal(qk["codes"], base["codes"])
        assert np.array_equal(qk["absmax"], base["absmax"] * s)


def test_zero_blocks_and_signed_zero():
    w = np.zeros((2, 64), np.float32)
    w[1, :] = -0.0
    qw = nf4.quantize(w)
    assert np.all(qw["absmax"] == 0)
    assert np.all(nf4.unpack_nibbles(qw["codes"], 128) == nf4.ZERO_CODE)
    assert np.all(nf4.dequantize_f32(qw) == 0)


def test_nonfinite_rejected():
    for bad in (np.nan, np.inf, -np.inf):
        w = np.zeros(64, np.float32)
        w[3] = bad
        with pytest.raises(ValueError):
            nf4.quantize(w)


def test_nibble_order():
    pin_nibble_order()


def test_partial_tail_block():
    rng = np.random.default_rng(6)
    w = rng.standard_normal(64 * 3 + 10).astype(np.float32)
    qw = nf4.quantize(w)
    assert qw["absmax"].shape == (4,)
    assert qw["absmax"][3] == np.abs(w[192:]).max()


def test_double_quant_group_structure():
    rng = np.random.default_rng(7)
    a = rng.uniform(0.001, 0.05, 256 * 3 + 17).astype(np.float32)
    a[300:512] = 0.0
    a[256:300] = 0.0          # group 1 all zero
    q, f = nf4.double_quantize(a)
    assert q.shape == a.shape and f.shape == (4,)
    for g in range(4):
        seg = a[g * 256:(g + 1) * 256]
        if seg.max() == 0:
            assert f[g] == 0 and np.all(q[g * 256:(g + 1) * 256] == 0)
            continue
        G = seg.max()
        assert f[g] == np.float32(G / np.float32(448))
        # the group maximum maps to the largest finite E4M3 code (or just below on rounding)
        assert q[g * 256 + int(np.argmax(seg))] in (0x7E, 0x7D)
    ahat = nf4.dq_scales(q, f)
    nz = a > 0.02 * a.max()
    # relative error of an E4M3 scale is at most 2^-4 (3 mantissa bits, RNE)
    assert np.all(np.abs(ahat[nz] - a[nz]) <= a[nz] * 2.0 ** -4 * 1.0001)


def pin_double_quant_hand_case():
    """A two-block group worked by hand in exact arithmetic (bf16 inputs).

    G = 49 * 2^-12 (bf16 0x3C44) is the group maximum and a = 203 * 2^-20 (bf16
    0x394B) the other scale.
      448 / G = 37449 + 1/7; fp32 spacing there is 2^-8, and 1/7 = 36.57 * 2^-8,
      so inv = fp32(448 / G) = 37449 + 37/256 (above 448 / G by 3/1792).
      a * inv = 7.25 + 87 * 2^-28 exactly; fp32 spacing in [4, 8) is 2^-21 =
      128 * 2^-28, so fp32(a * inv) = 7.25 + 2^-21. E4M3 spacing in [4, 8) is 0.5:
      7.25 is the midpoint of 7.0 and 7.5, and the value lies above it -> 7.5
      (exponent 2 + 7 = 9, mantissa 7: byte 0x4F).
      G * inv = 448.0000086 -> fp32 448.000030517578125 -> saturates to 448 (0x7E).
      f = fp32(G / 448) = 7 * 2^-18 exactly; a_hat = 7.5 * 7 * 2^-18 = 52.5 * 2^-18.
    Two plausible slips land exactly on the midpoint instead and round to the even
    neighbour 7.0 (0x4E): a * (448 / G) without rounding 448 / G first (= 7.25), and
    a / f (= 7.25)."""
    a = np.array([203 * 2.0 ** -20, 49 * 2.0 ** -12], np.float32)
    assert nf4.bf16_bits_from_f32(a).tolist() == [0x394B, 0x3C44]
    q, f = nf4.double_quantize(a)
    assert q.tolist() == [0x4F, 0x7E], [hex(v) for v in q]
    assert f.tolist() == [7 * 2.0 ** -18]
    assert nf4.dq_scales(q, f).tolist() == [52.5 * 2.0 ** -18, 448 * 7 * 2.0 ** -18]


def test_double_quant_hand_worked_group():
    pin_double_quant_hand_case()


def test_double_quant_pin_catches_planted_slips(monkeypatch):
    """The hand-worked group fails for the two slips it was chosen against (CPU)."""
    orig = nf4.double_quantize

    def make(rule):
        def dq(absmax, dq_blocksize=nf4.DQ_BLOCKSIZE):
            a = np.asarray(absmax, np.float32).reshape(-1)
            G = np.float32(a.max())
            if rule == "unrounded":   # a * 448 / G in fp64, one rounding to fp32
                scaled = (a.astype(np.float64) * 448.0 / np.float64(G)).astype(np.float32)
            else:                     # a / fp32(G / 448)
                scaled = (a / np.float32(G / np.float32(448))).astype(np.float32)
            return nf4.e4m3_encode_satfinite(scaled), np.array([G / np.float32(448)], np.float32)
        return dq
    for rule in ("unrounded", "divide"):
        monkeypatch.setattr(nf4, "double_quantize", make(rule))
        with pytest.raises(AssertionError):
            pin_double_quant_hand_case()
    monkeypatch.setattr(nf4, "double_quantize", orig)
    pin_double_quant_hand_case()


def test_double_quant_codes_use_exact_absmax():
    rng = np.random.default_rng(8)
    w = (rng.standard_normal((16, 1024)) * 0.02).astype(np.float32)
    q0 = nf4.quantize(w, double_quant=False)
    q1 = nf4.quantize(w, double_quant=True)
    assert np.array_equal(q0["codes"], q1["codes"])
    assert np.array_equal(q0["absmax"], q1["absmax"])


def test_pins_catch_planted_mistakes(monkeypatch):
    """Plausible slips planted in the oracle make a pin fail (CPU only)."""
    # nibble order swapped
    orig_pack = nf4.pack_nibbles
    monkeypatch.setattr(nf4, "pack_nibbles", lambda idx: ((np.asarray(idx, np.uint8)[1::2] << 4)
                                                         | np.asarray(idx, np.uint8)[0::2]).astype(np.uint8))
    with pytest.raises(AssertionError):
        pin_nibble_order()
    monkeypatch.setattr(nf4, "pack_nibbles", orig_pack)
    # symmetric 8+8 grid instead of the asymmetric 8+7 construction
    orig_table = nf4.nf4_code_table

    def symmetric_table():
        d = 1 - (1 / 32 + 1 / 30) / 2
        pos = sp.ndtri(np.linspace(d, 0.5, 9)[:-1])
        v = np.sort(np.concatenate([pos, -pos[:7], [0.0]])) / sp.ndtri(d)
        return v.astype(np.float32)
    monkeypatch.setattr(nf4, "nf4_code_table", symmetric_table)
    with pytest.raises(AssertionError):
        pin_table_quantiles()
    monkeypatch.setattr(nf4, "nf4_code_table", orig_table)
    # nearest-code rule with the comparison flipped to >=
    orig_ci = nf4.code_indices

    def ci_ge(w32, absmax, blocksize=nf4.BLOCKSIZE):
        flat = np.ascontiguousarray(w32, dtype=np.float32).reshape(-1)
        a = np.repeat(absmax.astype(np.float32), blocksize)[:flat.size]
        n = (flat / a).astype(np.float32)
        m = nf4.nf4_midpoints()
        return sum((n >= m[j]).astype(np.uint8) for j in range(15)).astype(np.uint8)
    monkeypatch.setattr(nf4, "code_indices", ci_ge)
    with pytest.raises(AssertionError):
        pin_bruteforce_codes(np.concatenate([MID, -MID]))
    monkeypatch.setattr(nf4, "code_indices", orig_ci)


def _bf16_rne_exact(x: float) -> int:
    """Round a float (exactly, as a rational) to bf16 with ties to even, by brute
    force over the two neighbouring bf16 values."""
    from fractions import Fraction
    v = Fraction(x)
    lo_bits = int(nf4.bf16_bits_from_f32(np.array([np.float32(x)], np.float32))[0])
    cands = {lo_bits, (lo_bits + 1) & 0xFFFF, (lo_bits - 1) & 0xFFFF}
    best = None
    for b in cands:
        f = float(nf4.f32_from_bf16_bits(np.array([b], np.uint16))[0])
        if not np.isfinite(f):
            continue
        d = abs(Fraction(f) - v)
        key = (d, b & 1)
        if best is None or key < best[0]:
            best = (key, b)
    return best[1]


def test_bf16_from_f64_rounds_once():
    """fp64 -> bf16 in one rounding: equal to the fp32 route when the value is an fp32
    number, equal to brute force on random fp64 values, and right where the fp32
    route rounds twice (a value just above a bf16 midpoint that fp32 rounds onto it)."""
    rng = np.random.default_rng(5)
    f = rng.standard_normal(20000).astype(np.float32) * np.float32(2.0) ** rng.integers(-30, 30, 20000)
    assert np.array_equal(nf4.bf16_bits_from_f64(f.astype(np.float64)), nf4.bf16_bits_from_f32(f))
    x = rng.standard_normal(3000) * 2.0 ** rng.integers(-20, 20, 3000)
    got = nf4.bf16_bits_from_f64(x)
    for xi, g in zip(x[:3000], got[:3000]):
        assert int(g) == _bf16_rne_exact(float(xi)), xi
    # 1 + 2^-8 (a bf16 midpoint) + 2^-30: rounds up in one step; via fp32 it would first
    # land exactly on the midpoint and then go to the even neighbour, 1.0
    y = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert int(nf4.bf16_bits_from_f64(np.array([y]))[0]) == 0x3F81
    assert int(nf4.bf16_bits_from_f32(np.array([np.float32(y)]))[0]) == 0x3F80
    # exact midpoints go to the even neighbour; the subnormal range and zero signs
    assert int(nf4.bf16_bits_from_f64(np.array([1.0 + 2.0 ** -8]))[0]) == 0x3F80
    assert int(nf4.bf16_bits_from_f64(np.array([1.0 + 3 * 2.0 ** -8]))[0]) == 0x3F82
    assert int(nf4.bf16_bits_from_f64(np.array([3 * 2.0 ** -134]))[0]) == 0x0002
    assert int(nf4.bf16_bits_from_f64(np.array([-0.0]))[0]) == 0x8000
