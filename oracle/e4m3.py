"""E4M3 (the "FN" flavour: no infinities, max |x| = 448) in plain numpy.

Lesson 13, Fig. 13-1 and the answer to Q1: E4M3 has 8 bits -- 1 sign bit,
4 exponent bits, 3 mantissa bits -- and its largest magnitude is 448.  A
maximum of 448 fixes the FN variant: exponent field 15 is an ordinary binade
and only the all-ones pattern (0x7F / 0xFF) is NaN.  The exponent bias is 7.

Readings taken where the pages are silent:

* rounding is round-to-nearest, ties to the even code (mantissa LSB 0);
* magnitudes above 448 saturate to 448 ("satfinite");
* the sign is kept when a negative value rounds to zero (code 0x80);
* NaN inputs are out of scope (never produced by the quantizer's inputs).
"""

from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
EXP_BIAS = 7
NAN_CODES = (0x7F, 0xFF)


def decode_code(code: int) -> float:
    """Value of one E4M3 byte, from the bit formula (sign, 4-bit exponent,
    3-bit mantissa, bias 7; exponent field 0 is subnormal)."""
    if code in NAN_CODES:
        return float("nan")
    sign = -1.0 if (code >> 7) & 1 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0:
        mag = (m / 8.0) * 2.0 ** (1 - EXP_BIAS)
    else:
        mag = (1.0 + m / 8.0) * 2.0 ** (e - EXP_BIAS)
    return sign * mag


#: float64[256]: the exhaustive decode table (index = code byte).
DECODE = np.array([decode_code(c) for c in range(256)], dtype=np.float64)

#: the 127 finite non-negative magnitudes, in code order 0x00..0x7E, which is
#: also increasing value order.
_POS = DECODE[:0x7F].copy()


def decode(codes: np.ndarray) -> np.ndarray:
    """float64 values of an array of E4M3 bytes."""
    return DECODE[np.asarray(codes, dtype=np.uint8)]


def encode_rne(v: np.ndarray) -> np.ndarray:
    """Round float values to E4M3 codes: nearest finite code, ties to the even
    code, |v| > 448 saturating to +-448, sign kept on zero.

    ``v`` is taken exactly as given (float32 or float64); no intermediate
    rounding happens here.
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    # first magnitude >= |v|; the nearest code is it or its predecessor.
    hi = np.searchsorted(_POS, a, side="left")
    hi = np.minimum(hi, len(_POS) - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - _POS[lo]
    d_hi = _POS[hi] - a
    # exact hits: a == _POS[hi] -> d_hi == 0 -> pick hi below.
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    mag_code = np.where(pick_hi, hi, lo)
    # above the largest finite magnitude: saturate.
    mag_code = np.where(a >= _POS[-1], len(_POS) - 1, mag_code)
    sign = np.signbit(v).astype(np.uint8) << 7
    return (mag_code.astype(np.uint8) | sign).astype(np.uint8)


def encode_bruteforce(v: np.ndarray) -> np.ndarray:
    """Same rounding, by exhaustive search over all 254 finite codes.

    Slow (256 distances per value); used only to pin :func:`encode_rne`.
    """
    v = np.asarray(v, dtype=np.float64).ravel()
    finite = np.array([c for c in range(256) if c not in NAN_CODES])
    vals = DECODE[finite]
    out = np.empty(v.shape, dtype=np.uint8)
    for i, x in enumerate(v):
        xs = min(max(x, -E4M3_MAX), E4M3_MAX)  # satfinite
        d = np.abs(vals - xs)
        best = d.min()
        cands = finite[d == best]
        # candidates with equal distance: +0/-0 pair or a true tie.
        if len(cands) > 1:
            even = [c for c in cands if (c & 1) == 0]
            cands = np.array(even if even else cands)
        # prefer the candidate carrying the sign of x (matters only for zero).
        want_sign = 0x80 if np.signbit(x) else 0
        same = [c for c in cands if (c & 0x80) == want_sign]
        out[i] = same[0] if same else cands[0]
    return out
