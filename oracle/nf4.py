"""NF4 blockwise quantization, double quantization and dequantization (oracle).

TEST INFRASTRUCTURE ONLY -- see ``oracle/__init__.py``.

What the pages fix ([QLoRA-blog] "1. NormalFloat", "2. Double quantization";
[AQLoRA] 3.1):
* 16 four-bit codes whose values are placed for a zero-centred normal
  distribution; each weight stores the index of one code;
* weights are split into blocks of 64, each with its own scale, so that one
  code set serves blocks of different ranges;
* for computation the codes are turned back into bf16 values before the
  matrix multiply;
* double quantization stores the first-level (per 64) scales in 8 bits with a
  higher-precision scale per group of 256 first-level scales.

Readings where the pages are silent:
* code values: asymmetric normal quantiles (construction in ``nf4_code_table``);
* absmax scaling, IEEE fp32 division, nearest code by fp32 midpoints, ties to
  the lower code;
* nibble order: element 2k in the high nibble of byte k;
* double-quant format: OCP E4M3 (max 448), RNE with saturation, per-group fp32
  factor G/448; codes are computed from the exact fp32 absmax;
* dequantized value: bf16_rne(fp32_rn(code * scale)).
"""
from __future__ import annotations

import functools
from fractions import Fraction
from typing import Optional, Tuple

import mpmath
import numpy as np

BLOCKSIZE = 64
DQ_BLOCKSIZE = 256
E4M3_MAX = 448.0
ZERO_CODE = 7  # index of the exact 0.0 in the sorted table

# --------------------------------------------------------------------------- fp32 helpers


def _f32(x: float) -> np.float32:
    return np.float32(x)


def _round_mp_to_f32(v: mpmath.mpf) -> np.float32:
    """Round a high-precision value to fp32 once (nearest, ties to even)."""
    cand = np.float32(float(v))
    best = cand
    lo = np.nextafter(cand, np.float32(-np.inf))
    hi = np.nextafter(cand, np.float32(np.inf))
    best_err = abs(mpmath.mpf(float(cand)) - v)
    for c in (lo, hi):
        err = abs(mpmath.mpf(float(c)) - v)
        if err < best_err or (err == best_err and (int(np.float32(c).view(np.uint32)) & 1) == 0):
            best, best_err = c, err
    return np.float32(best)


# --------------------------------------------------------------------------- code table


def nf4_code_table() -> np.ndarray:
    return _nf4_code_table_cached().copy()


@functools.lru_cache(maxsize=1)
def _nf4_code_table_cached() -> np.ndarray:
    """The 16 NF4 code values, sorted ascending, as fp32.

    [QLoRA-blog] "1. NormalFloat" says only that the 16 values are arranged for
    a zero-centred normal distribution. Reading (the quantile construction of
    the QLoRA paper, which is not on the pages): with
    delta = 1 - (1/32 + 1/30)/2 and Phi^-1 the standard normal quantile,
      positive codes = Phi^-1(t) for the 8 points t of linspace(delta, 1/2, 9)
                       other than 1/2;
      negative codes = -Phi^-1(t) for the 7 points t of linspace(delta, 1/2, 8)
                       other than 1/2;
      plus an exact 0; all divided by Phi^-1(delta) so the extremes are +-1.
    Evaluated with mpmath at 50 digits (Phi^-1(t) = sqrt(2) erfinv(2t - 1)),
    rounded once to fp32.

    Pinned by: invariants (16 sorted distinct values, one exact 0, +-1 ends,
    7 negative / 8 positive) and the defining quantile property checked through
    the forward normal CDF. Parity with third-party NF4 tables: parity unpinned.
    """
    with mpmath.workdps(50):
        delta = mpmath.mpf(1) - (mpmath.mpf(1) / 32 + mpmath.mpf(1) / 30) / 2
        half = mpmath.mpf(1) / 2

        def ppf(t):
            return mpmath.sqrt(2) * mpmath.erfinv(2 * t - 1)

        pos = [delta + i * (half - delta) / 8 for i in range(8)]
        neg = [delta + i * (half - delta) / 7 for i in range(7)]
        norm = ppf(delta)
        vals = [ppf(t) / norm for t in pos] + [-ppf(t) / norm for t in neg] + [mpmath.mpf(0)]
        vals.sort()
        return np.array([_round_mp_to_f32(v) for v in vals], dtype=np.float32)


def nf4_midpoints(table: Optional[np.ndarray] = None) -> np.ndarray:
    """15 fp32 decision thresholds m_j = fp32_rn((c_j + c_{j+1}) / 2).

    The sum and the halving are exact in fp64 (two fp32 operands); one rounding
    to fp32 follows. A normalised value n maps to code index #{j : n > m_j},
    i.e. the nearest code with exact ties going to the lower code.
    """
    c = nf4_code_table() if table is None else table
    c64 = c.astype(np.float64)
    return ((c64[:-1] + c64[1:]) / 2.0).astype(np.float32)


# --------------------------------------------------------------------------- bf16 / e4m3


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (NaN kept quiet)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    is_nan = np.isnan(np.asarray(x, dtype=np.float32))
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    out = rounded.astype(np.uint16)
    out = np.where(is_nan, ((u >> 16) | 0x40).astype(np.uint16), out)
    return out.astype(np.uint16)


def bf16_bits_from_f64(x: np.ndarray) -> np.ndarray:
    """fp64 -> bf16 bit patterns with one rounding (to nearest, ties to even), not
    through fp32: x = m 2^e (frexp); the bf16 quantum is 2^(e - 8), and 2^-133 below
    the normal range; rint (ties to even) on the exactly scaled value, then the
    result (a bf16 value, or an overflow to inf) is read through fp32."""
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    q = np.maximum(e.astype(np.int64) - 8, -133)
    with np.errstate(over="ignore", invalid="ignore"):
        v = np.ldexp(np.rint(np.ldexp(x, -q)), q)
        f = v.astype(np.float32)
    out = (f.view(np.uint32) >> 16).astype(np.uint16)
    return np.where(np.isnan(x), np.uint16(0x7FC0), out).astype(np.uint16)


def f32_from_bf16_bits(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def e4m3_decode(q: np.ndarray) -> np.ndarray:
    """OCP FP8 E4M3 (fn variant: no infinities, 0x7F/0xFF NaN) -> fp32."""
    q = np.asarray(q, dtype=np.uint8).astype(np.int64)
    sign = np.where(q & 0x80, -1.0, 1.0)
    e = (q >> 3) & 0xF
    m = q & 0x7
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((q & 0x7F) == 0x7F, np.nan, val)
    return (sign * val).astype(np.float32)


def e4m3_encode_satfinite(x: np.ndarray) -> np.ndarray:
    """fp32 -> OCP E4M3, round to nearest even, saturating to +-448.

    Written from the format definition: 4 exponent bits with bias 7, 3 mantissa
    bits, subnormals below 2^-6 with quantum 2^-9, largest finite 448.
    Exact: every step runs on values representable in fp64.
    """
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    if np.isnan(x).any():
        raise ValueError("NaN has no saturated E4M3 encoding")
    sign = np.signbit(x)
    a = np.abs(x)
    out = np.zeros(a.shape, dtype=np.int64)
    sat = a >= E4M3_MAX
    fin = ~sat
    af = a[fin]
    _, ex = np.frexp(af)  # af = mant * 2**ex, mant in [0.5, 1)
    e_unb = ex - 1        # floor(log2 af) for af > 0
    quantum = np.where(af >= 2.0 ** -6, np.exp2(e_unb - 3.0), 2.0 ** -9)
    quantum = np.where(af == 0, 2.0 ** -9, quantum)
    k = af / quantum                      # exact (power-of-two divisor)
    kr = np.round(k)                      # numpy rounds half to even
    q = kr * quantum
    q = np.minimum(q, E4M3_MAX)
    bits = np.zeros(af.shape, dtype=np.int64)
    nz = q > 0
    qn = q[nz]
    _, eq = np.frexp(qn)
    Eq = eq - 1
    normal = Eq >= -6
    b = np.where(normal,
                 ((Eq + 7) << 3) | np.round((qn / np.exp2(Eq) - 1.0) * 8.0).astype(np.int64),
                 np.round(qn / 2.0 ** -9).astype(np.int64))
    bits[nz] = b
    out[fin] = bits
    out[sat] = 0x7E
    out = np.where(sign, out | 0x80, out)
    return out.astype(np.uint8)


# --------------------------------------------------------------------------- quantize


def _check_finite(w32: np.ndarray) -> None:
    if not np.isfinite(w32).all():
        raise ValueError("non-finite weight: NF4 quantization of NaN/Inf is undefined")


def block_absmax(w32: np.ndarray, blocksize: int = BLOCKSIZE) -> np.ndarray:
    """Per-block absmax a_b = max |w| over each run of ``blocksize`` elements of the
    row-major flattened tensor ([QLoRA-blog] "1. NormalFloat": each block has its
    own scaling factor; [AQLoRA] 3.1: 64-element blocks). A short last block uses
    the elements present. Exact in fp32."""
    flat = np.abs(np.ascontiguousarray(w32, dtype=np.float32).reshape(-1))
    nb = -(-flat.size // blocksize)
    pad = nb * blocksize - flat.size
    if pad:
        flat = np.concatenate([flat, np.zeros(pad, np.float32)])
    return flat.reshape(nb, blocksize).max(axis=1).astype(np.float32)


def code_indices(w32: np.ndarray, absmax: np.ndarray, blocksize: int = BLOCKSIZE) -> np.ndarray:
    """Per element: n = fp32_rn(w / a_b) (IEEE division), idx = #{j : n > m_j}.

    A block with a_b = 0 maps every element to the zero code.
    """
    flat = np.ascontiguousarray(w32, dtype=np.float32).reshape(-1)
    n_el = flat.size
    a = np.repeat(absmax.astype(np.float32), blocksize)[:n_el]
    with np.errstate(divide="ignore", invalid="ignore"):
        n = np.where(a > 0, flat / np.where(a > 0, a, np.float32(1)), np.float32(0)).astype(np.float32)
    m = nf4_midpoints()
    idx = np.zeros(n_el, dtype=np.uint8)
    for j in range(15):
        idx += (n > m[j]).astype(np.uint8)
    return idx


def pack_nibbles(idx: np.ndarray) -> np.ndarray:
    """byte k = idx[2k] << 4 | idx[2k+1] (even element in the high nibble)."""
    idx = np.asarray(idx, dtype=np.uint8).reshape(-1)
    if idx.size % 2:
        raise ValueError("packed NF4 storage needs an even element count")
    return ((idx[0::2] << 4) | idx[1::2]).astype(np.uint8)


def unpack_nibbles(codes: np.ndarray, n_el: int) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8).reshape(-1)
    out = np.empty(codes.size * 2, dtype=np.uint8)
    out[0::2] = codes >> 4
    out[1::2] = codes & 0xF
    return out[:n_el]


def double_quantize(absmax: np.ndarray, dq_blocksize: int = DQ_BLOCKSIZE) -> Tuple[np.ndarray, np.ndarray]:
    """Second-level quantization of the per-block scales ([QLoRA-blog]
    "2. Double quantization": 8-bit first-level scales, a higher-precision scale
    per group of 256).

    Per group g of 256 consecutive absmax values (the last may be short):
      G = max a_b; inv = fp32_rn(448 / G); q_b = e4m3_rn_satfinite(fp32_rn(a_b * inv));
      f_g = fp32_rn(G / 448). An all-zero group gives q = 0 and f = 0.
    Returns (absmax_q uint8 [nb], absmax2 fp32 [ceil(nb/256)]).
    """
    a = np.asarray(absmax, dtype=np.float32).reshape(-1)
    nb = a.size
    ng = -(-nb // dq_blocksize)
    q = np.zeros(nb, dtype=np.uint8)
    f = np.zeros(ng, dtype=np.float32)
    for g in range(ng):
        seg = a[g * dq_blocksize:(g + 1) * dq_blocksize]
        G = np.float32(seg.max()) if seg.size else np.float32(0)
        if G == 0:
            continue
        inv = np.float32(np.float32(E4M3_MAX) / G)
        scaled = (seg * inv).astype(np.float32)
        q[g * dq_blocksize:(g + 1) * dq_blocksize] = e4m3_encode_satfinite(scaled)
        f[g] = np.float32(G / np.float32(E4M3_MAX))
    return q, f


def dq_scales(absmax_q: np.ndarray, absmax2: np.ndarray, dq_blocksize: int = DQ_BLOCKSIZE) -> np.ndarray:
    """Reconstructed first-level scales a_hat_b = fp32_rn(fp32(q_b) * f_g)."""
    q = e4m3_decode(absmax_q)
    g = np.arange(q.size) // dq_blocksize
    return (q * np.asarray(absmax2, dtype=np.float32)[g]).astype(np.float32)


def quantize(w32: np.ndarray, double_quant: bool = False, blocksize: int = BLOCKSIZE,
             dq_blocksize: int = DQ_BLOCKSIZE) -> dict:
    """NF4-quantize a weight (fp32 values; bf16 inputs are widened exactly).

    Returns dict(codes=uint8[numel/2], absmax=fp32[nb]) and, with double
    quantization, absmax_q=uint8[nb] and absmax2=fp32[ceil(nb/256)]. Codes always
    use the exact fp32 absmax (double quantization is applied to the scales
    afterwards)."""
    w32 = np.ascontiguousarray(w32, dtype=np.float32)
    _check_finite(w32)
    a = block_absmax(w32, blocksize)
    idx = code_indices(w32, a, blocksize)
    out = dict(codes=pack_nibbles(idx), absmax=a, numel=w32.size, shape=w32.shape)
    if double_quant:
        q, f = double_quantize(a, dq_blocksize)
        out["absmax_q"] = q
        out["absmax2"] = f
    return out


def scales_for(qw: dict) -> np.ndarray:
    if "absmax_q" in qw:
        return dq_scales(qw["absmax_q"], qw["absmax2"])
    return qw["absmax"]


def dequantize_f32(qw: dict, blocksize: int = BLOCKSIZE) -> np.ndarray:
    """fp32_rn(c_idx * a) per element, before the bf16 rounding."""
    n_el = qw["numel"]
    idx = unpack_nibbles(qw["codes"], n_el)
    c = nf4_code_table()
    a = np.repeat(scales_for(qw).astype(np.float32), blocksize)[:n_el]
    return (c[idx] * a).astype(np.float32).reshape(qw["shape"])


def dequantize_bf16_bits(qw: dict, blocksize: int = BLOCKSIZE) -> np.ndarray:
    """Dequantized weight as bf16 bit patterns: bf16_rne(fp32_rn(c_idx * a))
    ([QLoRA-blog] "1. NormalFloat": codes are turned back into BFloat16 before
    the matrix multiply)."""
    return bf16_bits_from_f32(dequantize_f32(qw, blocksize))


def nearest_code_bruteforce(n: float) -> int:
    """Nearest code by exact rational distance; exact ties go to the lower code.
    (Used by the tests to check ``code_indices``.)"""
    c = [Fraction(float(v)) for v in nf4_code_table()]
    x = Fraction(float(np.float32(n)))
    best, best_d = 0, abs(x - c[0])
    for j in range(1, 16):
        d = abs(x - c[j])
        if d < best_d:
            best, best_d = j, d
    return best
