"""UE8M0 scale factors and the packed scale layout.

Lesson 13, Fig. 13-1 text: newer versions of the library accept UE8M0 scales
in place of FP32 ones -- an unsigned 8-bit exponent e standing for 2^(e - 127),
with no sign and no mantissa.  Deep dive, section 3 (interface conventions):
on sm_100 the LHS scales are handed over as four UE8M0 values packed into one
32-bit integer, in the transposed (MN-major), TMA-aligned layout.

Readings taken where the pages give no more:

* the four values in one integer are four consecutive K groups of one row;
  group 4p + t sits in bits 8t .. 8t + 7 (the byte order of a little-endian
  [.., 4] byte array), so a [M, K/128] scale matrix packs into int32
  [ceil(K/512)][ld] with ld >= M;
* groups past K/128 (K/128 not a multiple of 4) contribute a zero byte;
* a scale of +0 (an all-zero group, whose codes are all 0x00) is encoded as
  0; -0 is rejected like any signed value;
* every other scale must be a positive power of two in the float32 normal
  range, as the power-of-two quantizer produces; anything else is rejected.

This module works from the values (``numpy.frexp``), not from float32 bit
fields.
"""

from __future__ import annotations

import numpy as np

GROUPS_PER_WORD = 4


def encode(sf: np.ndarray) -> np.ndarray:
    """UE8M0 bytes (uint8, same shape) of float32 power-of-two scales."""
    x = np.asarray(sf, np.float32).astype(np.float64)
    if not np.all(np.isfinite(x)) or np.any(np.signbit(x)):
        raise ValueError("UE8M0 scales must be finite and carry no sign (-0 included)")
    out = np.zeros(x.shape, np.uint8)
    nz = x != 0
    mant, exp = np.frexp(x[nz])          # x = mant * 2^exp, mant in [0.5, 1)
    if np.any(mant != 0.5):
        raise ValueError("a UE8M0 scale must be a power of two")
    e = exp.astype(np.int64) - 1         # x = 2^e
    if np.any(e < -126) or np.any(e > 127):
        raise ValueError("a UE8M0 scale must lie in the float32 normal range")
    out[nz] = (e + 127).astype(np.uint8)
    return out


def decode(codes: np.ndarray) -> np.ndarray:
    """float64 values 2^(e - 127) of UE8M0 bytes e."""
    return np.ldexp(1.0, np.asarray(codes, np.int64) - 127)


def pack_1x128(alpha: np.ndarray) -> np.ndarray:
    """Packed layout of 1x128 scales.

    alpha float32 [M, K/128] (row i, group g) -> int32 [ceil(K/512), M]: word
    (p, i) holds groups 4p .. 4p + 3 of row i, group 4p + t in bits
    8t .. 8t + 7, missing groups as zero bytes.
    """
    codes = encode(alpha)
    m, kg = codes.shape
    words = -(-kg // GROUPS_PER_WORD)
    out = np.zeros((words, m), np.int64)
    for p in range(words):
        for t in range(GROUPS_PER_WORD):
            g = GROUPS_PER_WORD * p + t
            if g < kg:
                out[p] += codes[:, g].astype(np.int64) * (256 ** t)
    return out.astype(np.uint32).view(np.int32)


def unpack_1x128(packed: np.ndarray, m: int, kg: int) -> np.ndarray:
    """float64 scales [m, kg] (row i, group g) of the packed layout: the
    inverse of ``pack_1x128`` on the first m rows of each word row (the
    columns past m of a TMA-aligned ld are ignored)."""
    words = np.asarray(packed).view(np.uint32).astype(np.int64)
    if words.ndim != 2 or words.shape[0] != -(-kg // GROUPS_PER_WORD) or words.shape[1] < m:
        raise ValueError("packed scales must be [ceil(kg/4), ld >= m]")
    codes = np.zeros((m, kg), np.int64)
    for g in range(kg):
        p, t = divmod(g, GROUPS_PER_WORD)
        codes[:, g] = (words[p, :m] >> (8 * t)) & 0xFF
    out = decode(codes)
    out[codes == 0] = 0.0   # code 0 stands for an all-zero group (scale +0)
    return out
