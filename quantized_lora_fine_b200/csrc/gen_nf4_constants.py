"""Writes nf4_constants.cuh: the NF4 code values and decision midpoints as fp32
bit patterns for the CUDA kernels.

Construction (QLoRA paper's NormalFloat, which the QLoRA page describes only as
16 values arranged for a zero-centred normal distribution): with
delta = 1 - (1/32 + 1/30)/2, the positive codes are the standard normal
quantiles at the 8 points of linspace(delta, 1/2, 9) other than 1/2, the
negative codes the negated quantiles at the 7 points of linspace(delta, 1/2, 8)
other than 1/2, plus 0; everything divided by the quantile at delta. Quantiles
come from scipy.special.ndtri in fp64, rounded to fp32. The midpoints are
fp32_rn((c_j + c_{j+1}) / 2) with the sum formed in fp64.

Run:  python quantized_lora_fine_b200/csrc/gen_nf4_constants.py
"""
import os
import sys

import numpy as np
import scipy.special as sp


def constants():
    d = 1.0 - 0.5 * (1.0 / 32 + 1.0 / 30)
    pos = sp.ndtri(np.linspace(d, 0.5, 9)[:-1])
    neg = -sp.ndtri(np.linspace(d, 0.5, 8)[:-1])
    codes = (np.sort(np.concatenate([pos, neg, [0.0]])) / sp.ndtri(d)).astype(np.float32)
    c64 = codes.astype(np.float64)
    mids = ((c64[:-1] + c64[1:]) / 2.0).astype(np.float32)
    return codes, mids


def cell_of(n) -> int:
    """Cell of a normalised value n in [-1, 1]: bits 18..23 of fp32(n + 3) (the top
    five mantissa bits plus the low exponent bit), i.e. 32 cells of width 1/16
    and cell 32 for n = 1. Monotone in n; every cell holds at most one midpoint."""
    v = np.float32(n) + np.float32(3.0)
    return (int(np.float32(v).view(np.uint32)) >> 18) & 63


def cell_tables(mids):
    cells = [cell_of(m) for m in mids]
    assert len(set(cells)) == len(cells), "a cell holds two midpoints"
    thr = [0x7F800000] * 64          # +inf: no midpoint in the cell
    base = [15] * 64
    for c in range(64):
        base[c] = sum(1 for x in cells if x < c) if c <= 32 else 0
    for m, c in zip(mids, cells):
        thr[c] = int(np.float32(m).view(np.uint32))
    return thr, base


CELL_SHIFT = 21  # fine cells: the top 11 bits of fp32 n (sign, exponent, 2 mantissa bits)


def fine_cell_tables(codes, mids):
    """Per fine cell c (all fp32 n with bits >> 21 == c): the base index (number of
    midpoints below every value of the cell) and the low 21 bits of the cell's
    midpoint, if it holds one. Reconstructing the threshold as (bits(n) & ~0x1FFFFF)
    | low21 gives that midpoint exactly; a cell without a midpoint gets the
    largest value (positive cell) or the value closest to zero (negative cell), so
    that n > threshold never holds. Then idx = base + (n > threshold)."""
    mb = [int(v) for v in mids.view(np.uint32)]
    mf = [float(v) for v in mids]
    ncell = 1 << (32 - CELL_SHIFT)
    word, vals = [], []
    for c in range(ncell):
        neg = c >> (31 - CELL_SHIFT)
        lo_bits, hi_bits = c << CELL_SHIFT, ((c + 1) << CELL_SHIFT) - 1
        v1 = float(np.uint32(lo_bits).view(np.float32))
        v2 = float(np.uint32(hi_bits).view(np.float32))
        vmin, vmax = (v2, v1) if neg else (v1, v2)
        inside = [j for j, b in enumerate(mb) if (b >> CELL_SHIFT) == c]
        assert len(inside) <= 1, "a fine cell holds two midpoints"
        if np.isnan(vmin) or np.isnan(vmax):
            base = 15 if not neg else 0
        else:
            base = sum(1 for j, m in enumerate(mf) if j not in inside and m < vmin)
        if inside:
            low = mb[inside[0]] & ((1 << CELL_SHIFT) - 1)
        else:
            low = ((1 << CELL_SHIFT) - 1) if not neg else 0
        word.append(low | (base << 24) | (base << 28))
        c_lo = int(codes[base].view(np.uint32))
        c_hi = int(codes[min(base + 1, 15)].view(np.uint32)) if inside else c_lo
        vals.append((low, c_lo, c_hi, 0))
    return word, vals


def fine_cell_lookup(n, word):
    """Index of the nearest code for fp32 n with the fine-cell table, as the kernels do it."""
    b = int(np.float32(n).view(np.uint32))
    e = word[b >> CELL_SHIFT]
    thr = np.uint32((b & ~((1 << CELL_SHIFT) - 1) & 0xFFFFFFFF) | (e & ((1 << CELL_SHIFT) - 1))).view(np.float32)
    return ((e >> 24) & 15) + (1 if np.float32(n) > thr else 0)


def check_fine_cells(codes, mids, word, vals, rng=np.random.default_rng(0)):
    ref = lambda n: int(np.sum(np.float32(n) > mids))
    tests = [np.float32(x) for x in (0.0, -0.0, 1.0, -1.0)]
    for m in mids:
        tests += [m, np.nextafter(m, np.float32(2)), np.nextafter(m, np.float32(-2))]
    for c in range(len(word)):
        for bits in (c << CELL_SHIFT, ((c + 1) << CELL_SHIFT) - 1):
            v = np.uint32(bits).view(np.float32)
            if np.isfinite(v) and abs(v) <= 1.0:
                tests.append(v)
    tests += list(rng.uniform(-1, 1, 200000).astype(np.float32))
    tests += list((rng.uniform(-1, 1, 50000) * 2.0 ** rng.integers(-60, 0, 50000)).astype(np.float32))
    for n in tests:
        i = fine_cell_lookup(n, word)
        assert i == ref(n), (float(n), i, ref(n))
        e = vals[int(np.float32(n).view(np.uint32)) >> CELL_SHIFT]
        thr = np.uint32((int(np.float32(n).view(np.uint32)) & ~0x1FFFFF & 0xFFFFFFFF) | e[0]).view(np.float32)
        cv = e[2] if np.float32(n) > thr else e[1]
        assert cv == int(codes[ref(n)].view(np.uint32)), float(n)


def fine_float_tables(codes, mids, word):
    """Arithmetic form of the fine-cell lookup, evaluated on the FMA pipe:
    s = sat(n * 2^100 + T) is 1 iff n > the cell's midpoint (T = -m * 2^100; cells
    without a midpoint get T = -2^101 so s = 0 for every |n| <= 1), and
    idx = base + s. Per cell: {T, base} as fp32 for the quantizer, {T, code[base],
    code[base + s = 1] - code[base]} for the error pass (the difference is exact,
    checked below, so code[base] + 1 * diff rounds back to code[base + 1])."""
    mb = [int(v) for v in mids.view(np.uint32)]
    qt, et = [], []
    for c, wd in enumerate(word):
        base = (wd >> 24) & 15
        inside = [j for j, b in enumerate(mb) if (b >> CELL_SHIFT) == c]
        T = np.float32(-float(mids[inside[0]]) * 2.0 ** 100) if inside else np.float32(-(2.0 ** 101))
        qt.append((int(T.view(np.uint32)), int(np.float32(base).view(np.uint32))))
        c_lo = np.float32(codes[base])
        c_hi = np.float32(codes[min(base + 1, 15)]) if inside else c_lo
        d = np.float32(c_hi - c_lo)
        assert np.float32(c_lo + d) == c_hi and float(d) == float(c_hi) - float(c_lo), (c, c_lo, c_hi)
        et.append((int(T.view(np.uint32)), int(c_lo.view(np.uint32)), int(d.view(np.uint32)), 0))
    return qt, et


def check_float_tables(codes, mids, qt, et, rng=np.random.default_rng(1)):
    f = lambda b: np.uint32(b).view(np.float32)
    tests = [np.float32(x) for x in (0.0, -0.0, 1.0, -1.0)]
    for m in mids:
        tests += [m, np.nextafter(m, np.float32(2)), np.nextafter(m, np.float32(-2))]
    tests += list(rng.uniform(-1, 1, 200000).astype(np.float32))
    tests += list((rng.uniform(-1, 1, 50000) * 2.0 ** rng.integers(-140, 0, 50000)).astype(np.float32))
    for n in tests:
        c = int(np.float32(n).view(np.uint32)) >> CELL_SHIFT
        T, base = f(qt[c][0]), f(qt[c][1])
        # exact n * 2^100 + T, rounded once, then clamped to [0, 1]
        v = float(np.float32(float(n) * 2.0 ** 100 + float(T)))
        sat = min(max(v, 0.0), 1.0)
        assert sat in (0.0, 1.0)
        ref = int(np.sum(np.float32(n) > mids))
        assert int(base) + int(sat) == ref, (float(n), base, sat, ref)
        _, lo, d, _ = et[c]
        assert np.float32(f(lo) + np.float32(sat) * f(d)) == codes[ref]


def coarse_float_tables(codes, mids):
    """Cells of width 1/16 addressed without integer ALU work: cell(n) =
    floor(16 (n + 1)) (33 cells for n in [-1, 1]), which the kernels obtain as the
    low bits of RZ(16 n + (16 + 2^23)). Each cell holds at most one midpoint
    (midpoints are at least 0.08 apart). Per cell {T, base}: T = -m 2^100 for the
    cell's midpoint m, else -2^101; idx = base + sat(n 2^100 + T). The error
    pass's table adds {code[base], code[base + 1] - code[base]}."""
    cells = [int(np.floor(16.0 * (float(m) + 1.0))) for m in mids]
    assert len(set(cells)) == len(cells), "a coarse cell holds two midpoints"
    q, e = [], []
    for c in range(33):
        lo = c / 16.0 - 1.0
        inside = [j for j, cc in enumerate(cells) if cc == c]
        base = sum(1 for j, m in enumerate(mids) if j not in inside and float(m) < lo)
        if inside:
            T = np.float32(-float(mids[inside[0]]) * 2.0 ** 100)
        else:
            T = np.float32(-(2.0 ** 101))
        q.append((int(T.view(np.uint32)), int(np.float32(base).view(np.uint32))))
        c_lo = np.float32(codes[base])
        c_hi = np.float32(codes[min(base + 1, 15)]) if inside else c_lo
        d = np.float32(c_hi - c_lo)
        assert np.float32(c_lo + d) == c_hi and float(d) == float(c_hi) - float(c_lo)
        e.append((int(T.view(np.uint32)), int(c_lo.view(np.uint32)), int(d.view(np.uint32)), 0))
    return q, e


def coarse_cell(n):
    """floor(16 (n + 1)) the way the kernels compute it: fma(n, 16, 16 + 2^23)
    rounded toward zero, minus 2^23."""
    import fractions
    v = fractions.Fraction(float(n)) * 16 + 16 + 2 ** 23
    return int(v) - 2 ** 23  # RZ to an integer (all values are in [2^23, 2^24))


def check_coarse(codes, mids, q, e, rng=np.random.default_rng(2)):
    f = lambda b: float(np.uint32(b).view(np.float32))
    tests = [np.float32(x) for x in (0.0, -0.0, 1.0, -1.0)]
    for m in mids:
        tests += [m, np.nextafter(m, np.float32(2)), np.nextafter(m, np.float32(-2))]
    for c in range(33):
        b = np.float32(c / 16.0 - 1.0)
        tests += [b, np.nextafter(b, np.float32(2)), np.nextafter(b, np.float32(-2))]
    tests += list(rng.uniform(-1, 1, 100000).astype(np.float32))
    tests += list((rng.uniform(-1, 1, 30000) * 2.0 ** rng.integers(-140, 0, 30000)).astype(np.float32))
    for n in tests:
        if abs(float(n)) > 1.0:
            continue
        c = coarse_cell(n)
        T, base = f(q[c][0]), f(q[c][1])
        v = float(np.float32(float(n) * 2.0 ** 100 + T))
        sat = min(max(v, 0.0), 1.0)
        ref = int(np.sum(np.float32(n) > mids))
        assert sat in (0.0, 1.0) and int(base) + int(sat) == ref, (float(n), c, base, sat, ref)
        _, lo, d, _ = e[c]
        assert np.float32(np.float32(f(lo)) + np.float32(sat) * np.float32(f(d))) == codes[ref]


def coarse_code_table(codes, mids, ce):
    """{code[base], code[base + 1]} per coarse cell (both code[base] when the cell
    holds no midpoint). The error pass rebuilds the cell's midpoint from the pair:
    RN(c_lo + c_hi) = 2 m exactly (m = RN((c_lo + c_hi) / 2) by construction), so
    s = sat(RN(n 2^100 - RN(c_lo + c_hi) 2^99)) is the same test, and the code
    value is c_lo + s (c_hi - c_lo)."""
    f = lambda b: np.uint32(b).view(np.float32)
    out = []
    for (_, lo, d, _) in ce:
        c_lo = f(lo)
        c_hi = np.float32(c_lo + f(d))
        out.append((int(c_lo.view(np.uint32)), int(c_hi.view(np.uint32))))
    for j in range(15):
        assert np.float32(codes[j] + codes[j + 1]) == np.float32(2.0) * mids[j], j
    return out


def check_coarse_codes(codes, mids, cc, rng=np.random.default_rng(3)):
    f = lambda b: np.uint32(b).view(np.float32)
    tests = [np.float32(x) for x in (0.0, -0.0, 1.0, -1.0)]
    for m in mids:
        tests += [m, np.nextafter(m, np.float32(2)), np.nextafter(m, np.float32(-2))]
    tests += list(rng.uniform(-1, 1, 100000).astype(np.float32))
    tests += list((rng.uniform(-1, 1, 30000) * 2.0 ** rng.integers(-140, 0, 30000)).astype(np.float32))
    for n in tests:
        c = coarse_cell(n)
        lo, hi = f(cc[c][0]), f(cc[c][1])
        sm = np.float32(lo + hi)
        v = float(np.float32(float(n) * 2.0 ** 100 - float(sm) * 2.0 ** 99))
        sat = np.float32(min(max(v, 0.0), 1.0))
        dc = np.float32(hi - lo)
        val = np.float32(float(sat) * float(dc) + float(lo))   # one rounding, as an FMA
        assert val == codes[int(np.sum(np.float32(n) > mids))], float(n)


def render():
    codes, mids = constants()
    cq, ce = coarse_float_tables(codes, mids)
    check_coarse(codes, mids, cq, ce)
    cc = coarse_code_table(codes, mids, ce)
    check_coarse_codes(codes, mids, cc)
    thr, base = cell_tables(mids)
    word, vals = fine_cell_tables(codes, mids)
    check_fine_cells(codes, mids, word, vals)
    qt, et = fine_float_tables(codes, mids, word)
    check_float_tables(codes, mids, qt, et)
    cb = [int(v) for v in codes.view(np.uint32)]
    mb = [int(v) for v in mids.view(np.uint32)]
    lines = [
        "// Generated by gen_nf4_constants.py -- do not edit.",
        "// NF4 code values (ascending) and the 15 decision midpoints, as fp32 bits.",
        "#pragma once",
        "#include <cstdint>",
        "namespace qlb {",
        "__device__ constexpr uint32_t kNF4CodeBits[16] = {",
        "    " + ", ".join("0x%08Xu" % b for b in cb) + "};",
        "__device__ constexpr uint32_t kNF4MidBits[15] = {",
        "    " + ", ".join("0x%08Xu" % b for b in mb) + "};",
        "// values, for reading: " + ", ".join("%.9g" % v for v in codes),
        "// Index lookup: cell c = bits 18..23 of fp32(n + 3); idx = kNF4CellBase[c] + (n > kNF4CellThr[c]).",
        "__device__ constexpr uint32_t kNF4CellThrBits[64] = {",
        "    " + ", ".join("0x%08Xu" % b for b in thr) + "};",
        "__device__ constexpr uint8_t kNF4CellBase[64] = {",
        "    " + ", ".join(str(b) for b in base) + "};",
        "// Fine cells c = bits(n) >> 21 (2048 cells; each holds at most one midpoint).",
        "// kNF4Fine[c]: bits 0..20 = low 21 bits of the cell's threshold, bits 24..27 and",
        "// 28..31 = base index (twice). Threshold = (bits(n) & ~0x1FFFFF) | low21;",
        "// idx = base + (n > threshold).",
        "__device__ constexpr uint32_t kNF4Fine[2048] = {",
    ]
    for i in range(0, len(word), 8):
        lines.append("    " + ", ".join("0x%08Xu" % w for w in word[i:i + 8]) + ",")
    lines += [
        "};",
        "// kNF4FineVal[c] = {low21 threshold bits, fp32 bits of code[base], of code[base + 1]",
        "// (= code[base] without a midpoint), 0}: the code value is the third word when",
        "// n > threshold, else the second.",
        "__device__ constexpr uint32_t kNF4FineVal[2048 * 4] = {",
    ]
    for i in range(0, len(vals), 2):
        lines.append("    " + ", ".join("0x%08Xu, 0x%08Xu, 0x%08Xu, 0x%08Xu" % v for v in vals[i:i + 2]) + ",")
    lines += [
        "};",
        "// Coarse cells c = floor(16 (n + 1)), 33 of them (n in [-1, 1]), computed as the",
        "// low bits of RZ(16 n + 16 + 2^23). kNF4CoarseQ[c] = {T, base}; kNF4CoarseE[c] =",
        "// {T, code[base], code[base + 1] - code[base], 0}; s = sat(n * 2^100 + T).",
        "__device__ constexpr uint32_t kNF4CoarseQ[33 * 2] = {",
        "    " + ", ".join("0x%08Xu, 0x%08Xu" % v for v in cq) + "};",
        "__device__ constexpr uint32_t kNF4CoarseE[33 * 4] = {",
        "    " + ", ".join("0x%08Xu, 0x%08Xu, 0x%08Xu, 0x%08Xu" % v for v in ce) + "};",
        "// kNF4CoarseC[c] = {code[base], code[base + 1]} (fp32 bits; the second equals the",
        "// first without a midpoint): s = sat(n 2^100 - RN(lo + hi) 2^99), code = lo + s (hi - lo).",
        "__device__ constexpr uint32_t kNF4CoarseC[33 * 2] = {",
        "    " + ", ".join("0x%08Xu, 0x%08Xu" % v for v in cc) + "};",
        "// kNF4CoarseD[c] = {code[base], code[base + 1] - code[base]} (exact difference):",
        "// RN(2 lo + diff) = RN(lo + hi) = twice the midpoint, code = lo + s diff.",
        "__device__ constexpr uint32_t kNF4CoarseD[33 * 2] = {",
        "    " + ", ".join("0x%08Xu, 0x%08Xu" % (v[1], v[2]) for v in ce) + "};",
        "// Arithmetic lookup on the FMA pipe: s = sat(n * 2^100 + T) is 1 iff n is above",
        "// the cell's midpoint. kNF4FineQ[c] = {T, base} (fp32 bits): idx = base + s.",
        "__device__ constexpr uint32_t kNF4FineQ[2048 * 2] = {",
    ]
    for i in range(0, len(qt), 4):
        lines.append("    " + ", ".join("0x%08Xu, 0x%08Xu" % v for v in qt[i:i + 4]) + ",")
    lines += [
        "};",
        "// kNF4FineE[c] = {T, code[base], code[base + 1] - code[base] (exact), 0}: the",
        "// code value is code[base] + s * difference.",
        "__device__ constexpr uint32_t kNF4FineE[2048 * 4] = {",
    ]
    for i in range(0, len(et), 2):
        lines.append("    " + ", ".join("0x%08Xu, 0x%08Xu, 0x%08Xu, 0x%08Xu" % v for v in et[i:i + 2]) + ",")
    lines += [
        "};",
        "}  // namespace qlb",
        "",
    ]
    return "\n".join(lines)


if __name__ == "__main__":
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "nf4_constants.cuh")
    with open(out, "w") as f:
        f.write(render())
    sys.stdout.write(open(out).read())
