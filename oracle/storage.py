"""Storage arithmetic of the NF4 format (oracle).

TEST INFRASTRUCTURE ONLY -- see ``oracle/__init__.py``.

[QLoRA-blog] "2. Double quantization" and "A worked memory budget for 65
billion weights": a 32-bit scale per 64 weights costs 0.5 bit per weight;
8-bit scales per 64 plus a 32-bit scale per 256 scales cost about 0.127 bit
per weight.
"""
from __future__ import annotations

from fractions import Fraction

from .nf4 import BLOCKSIZE, DQ_BLOCKSIZE


def scale_bits_per_weight(double_quant: bool, blocksize: int = BLOCKSIZE,
                          dq_blocksize: int = DQ_BLOCKSIZE) -> Fraction:
    if not double_quant:
        return Fraction(32, blocksize)
    return Fraction(8, blocksize) + Fraction(32, blocksize * dq_blocksize)


def bits_per_weight(double_quant: bool) -> Fraction:
    return 4 + scale_bits_per_weight(double_quant)


def buffer_bytes(numel: int, double_quant: bool, blocksize: int = BLOCKSIZE,
                 dq_blocksize: int = DQ_BLOCKSIZE) -> dict:
    """Byte size of each stored buffer for one quantized tensor."""
    nb = -(-numel // blocksize)
    out = dict(codes=-(-numel // 2))
    if double_quant:
        out["absmax_q"] = nb
        out["absmax2"] = 4 * (-(-nb // dq_blocksize))
    else:
        out["absmax"] = 4 * nb
    out["total"] = sum(out.values())
    return out
