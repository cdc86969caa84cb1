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
import fractions
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


ZERO_CODE = 7


CELL_MUL = 15.75   # cells of width 1/15.75: 32 of them cover [-1, 1]


def lane_cell(n, sc=1.0):
    """floor(15.75 n + 16) for n in [-1, 1] (a value in [0, 31]) the way the kernels
    compute it from n_s = n / sc: the low bits of RZ(n_s (15.75 sc) + 2^23 + 16)
    (an FMA rounded toward zero; the values lie in [2^23, 2^24), where fp32 steps
    by 1). The exact product n_s 15.75 sc equals 15.75 n while n_s is normal."""
    v = fractions.Fraction(n) * fractions.Fraction(CELL_MUL) * fractions.Fraction(sc) + 16 + 2 ** 23
    return int(v) - 2 ** 23


def lane_tables(codes, mids):
    """Per lane l = cell l (32 cells of width 1/15.75; the midpoints lie at least 0.08
    apart, so a cell holds at most one), with base = the number of midpoints below
    every value of the cell: B[l] = 2^23 + base (fp32); T[l] = -m_base 2^36 if
    base < 15, else -2^38 (below every n 2^36); LO[l] = code[base]; D[l] =
    code[base + 1] - code[base] (exact in fp32), 0 if base = 15. A value n of the
    cell has code index base + s with s = [n > m_base]: m_base is the only midpoint
    that can lie in the cell (the one below it lies below the cell, the one above it
    above the cell). Its code value is LO + s D."""
    cells = [lane_cell(float(m)) for m in mids]
    assert len(set(cells)) == len(cells), "a cell holds two midpoints"
    B, T, LO, D = [], [], [], []
    for c in range(32):
        lo = fractions.Fraction(c - 16) / fractions.Fraction(CELL_MUL)   # smallest value of the cell
        base = sum(1 for m in mids if fractions.Fraction(float(m)) < lo)
        B.append(int(np.float32(base + 2 ** 23).view(np.uint32)))
        t = -float(mids[base]) * 2.0 ** 36 if base < 15 else -(2.0 ** 38)
        assert float(np.float32(t)) == t   # exact
        T.append(int(np.float32(t).view(np.uint32)))
        c_lo = np.float32(codes[base])
        d = np.float32(codes[base + 1] - c_lo) if base < 15 else np.float32(0)
        if base < 15:
            assert float(d) == float(codes[base + 1]) - float(c_lo)   # exact difference
        LO.append(int(c_lo.view(np.uint32)))
        D.append(int(d.view(np.uint32)))
    return B, T, LO, D


def check_lane_tables(codes, mids, B, T, LO, D, rng=np.random.default_rng(2)):
    """Brute force against #{j : n > m_j}, for the three block scalings the kernels
    use (sc = 1, 2^64 for tiny blocks, 2^-64 for huge ones): the kernel holds
    n_s = n / sc, reads b = B[cell], t = T[cell] (warp shuffles by lane index; only
    the low 5 bits of the lane operand count), s = sat(n_s (2^36 sc) + t), takes the
    index from the low bits of bits(b + s) and the code value as code[index] (lane
    index & 15) or LO[cell] + s D[cell] (one rounding, an FMA). Below |n| = 2^-62 the
    scaled n_s of a tiny block is subnormal and must still give the zero code."""
    f = lambda bits: float(np.uint32(bits).view(np.float32))
    tests = [np.float32(x) for x in (0.0, -0.0, 1.0, -1.0)]
    for m in mids:
        tests += [m, np.nextafter(m, np.float32(2)), np.nextafter(m, np.float32(-2))]
    for c in range(33):
        b = np.float32((c - 16) / CELL_MUL)
        tests += [b, np.nextafter(b, np.float32(2)), np.nextafter(b, np.float32(-2))]
    tests += list(rng.uniform(-1, 1, 100000).astype(np.float32))
    tests += list((rng.uniform(-1, 1, 30000) * 2.0 ** rng.integers(-149, 0, 30000)).astype(np.float32))
    for n in tests:
        if abs(float(n)) > 1.0:
            continue
        ref = int(np.sum(np.float32(n) > mids))
        for sc in (1.0, 2.0 ** 64, 2.0 ** -64):
            ns = fractions.Fraction(float(n)) / fractions.Fraction(sc)
            if ns != 0 and abs(ns) < fractions.Fraction(2) ** -126:
                assert ref == ZERO_CODE, float(n)    # the kernel's subnormal n_s: |n| < 2^-62
                ns = fractions.Fraction(0)
            v = ns * fractions.Fraction(CELL_MUL) * fractions.Fraction(sc) + 16 + 2 ** 23
            assert 0 <= int(v) - 2 ** 23 <= 31
            c = (int(v) - 2 ** 23) & 31
            b, t = f(B[c]), f(T[c])
            w = ns * fractions.Fraction(2) ** 36 * fractions.Fraction(sc) + fractions.Fraction(t)
            w = float(np.float32(float(w))) if w != 0 else 0.0      # one rounding (FMA)
            s = min(max(w, 0.0), 1.0)
            assert s in (0.0, 1.0), (float(n), sc, w)
            x = int(np.float32(b + s).view(np.uint32))
            assert x - 0x4B000000 == ref, (float(n), sc, c, x, ref)
            assert codes[x & 15] == codes[ref]
            val = np.float32(fractions.Fraction(s) * fractions.Fraction(f(D[c])) + fractions.Fraction(f(LO[c])))
            assert val == codes[ref], (float(n), sc, c)


def render():
    codes, mids = constants()
    B, T, LO, D = lane_tables(codes, mids)
    check_lane_tables(codes, mids, B, T, LO, D)
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
        "// Lane tables for the warp-shuffle code lookup: lane c = cell c = floor(15.75 n + 16)",
        "// in [0, 31] (the low bits of RZ(15.75 n + 2^23 + 16)), base_c = the number of",
        "// midpoints below the cell. kNF4LaneB[c] = 2^23 + base_c; kNF4LaneT[c] = -m_base 2^36",
        "// (-2^38 if base_c = 15). With s = sat(n 2^36 + T[c]): bits(B[c] + s) = 0x4B000000 +",
        "// code index.",
        "__device__ constexpr uint32_t kNF4LaneB[32] = {",
        "    " + ", ".join("0x%08Xu" % v for v in B) + "};",
        "__device__ constexpr uint32_t kNF4LaneT[32] = {",
        "    " + ", ".join("0x%08Xu" % v for v in T) + "};",
        "}  // namespace qlb",
        "",
    ]
    return "\n".join(lines)


if __name__ == "__main__":
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "nf4_constants.cuh")
    with open(out, "w") as f:
        f.write(render())
    sys.stdout.write(open(out).read())
