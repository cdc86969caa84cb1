"""The kernels' one-multiply quotient decides every bf16 pair like IEEE division.

The quantizer and the error pass form n~ = RN(w * RN(1/a)) (one fp32 multiply by
the block's reciprocal) instead of the IEEE quotient RN(w / a) that the NF4
definition uses ([QLoRA-blog] "1. NormalFloat": scale by the block absmax, take
the nearest code). The two can differ in the last bit, but for bf16 inputs never
across a code midpoint: this test enumerates every bf16 significand pair and
exponent gap with |w| <= a (the decision is invariant under scaling both by a
power of two while 1/a stays normal, which the kernels ensure by rescaling tiny
and huge blocks) and compares the code indices of the two quotients.
"""
import numpy as np

from oracle import nf4


def _indices(n: np.ndarray, mids: np.ndarray) -> np.ndarray:
    return (n[..., None] > mids).sum(axis=-1)


def test_reciprocal_quotient_picks_ieee_codes_for_all_bf16_pairs():
    mids = nf4.nf4_midpoints().astype(np.float32)
    sig = (1 + np.arange(128, dtype=np.float32) / 128).astype(np.float32)
    a = sig[:, None]
    r = (np.float32(1) / a).astype(np.float32)
    checked = 0
    for gap in range(12):                      # |w / a| < 2^-11 beyond: the zero code either way
        for sign in (np.float32(1), np.float32(-1)):
            w = (sign * sig * np.float32(2.0 ** -gap)).astype(np.float32)[None, :]
            ok = np.abs(w) <= a
            n_ieee = (w / a).astype(np.float32)
            n_recip = (w * r).astype(np.float32)
            differ = (_indices(n_ieee, mids) != _indices(n_recip, mids)) & ok
            assert not differ.any(), f"gap {gap}: {np.argwhere(differ)[:5]}"
            checked += int(ok.sum())
    assert checked == 2 * (128 * 129 // 2 + 11 * 128 * 128)


def test_reciprocal_quotient_differs_from_ieee_somewhere():
    """The shortcut is not the same number: some quotients differ in the last bit,
    which is why the statement above is about code decisions only."""
    sig = (1 + np.arange(128, dtype=np.float32) / 128).astype(np.float32)
    a = sig[:, None]
    w = sig[None, :]
    n_ieee = (w / a).astype(np.float32)
    n_recip = (w * (np.float32(1) / a).astype(np.float32)).astype(np.float32)
    assert (n_ieee != n_recip).any()
