"""Round float64 values to bfloat16, round-to-nearest-even, in one step.

Lesson 13, Fig. 13-1 and section 2: the epilogue only converts the FP32
accumulator to BF16 and writes it back.  The rounding mode is not stated; the
reading taken is round-to-nearest-even (the IEEE default).

The oracle rounds the exact (float64) result directly to bfloat16, with no
float32 step in between, so that it is the correctly rounded BF16 value of the
formula.  bfloat16 has 8 significant bits (7 stored) and float32's exponent
range (normal min 2**-126, subnormal spacing 2**-133).
"""

from __future__ import annotations

import numpy as np


def round_f64(x: np.ndarray) -> np.ndarray:
    """float64 array of the nearest bfloat16 values (ties to even)."""
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = (x != 0) & np.isfinite(x)
    xm = x[nz]
    _, e = np.frexp(xm)  # |xm| = m * 2**e, m in [0.5, 1)
    # spacing of bfloat16 values in the binade of xm: 2**(e-8), floored at
    # the subnormal spacing 2**-133.
    q_exp = np.maximum(e - 8, -133)
    scaled = np.ldexp(xm, -q_exp)  # exact: a power-of-two rescale
    r = np.rint(scaled)  # numpy rint is round-half-to-even
    out[nz] = np.ldexp(r, q_exp)
    out[~np.isfinite(x)] = x[~np.isfinite(x)]
    # keep the sign of zero results
    out = np.copysign(out, x)
    big = np.abs(out) > float.fromhex("0x1.fep127")
    out[big] = np.copysign(np.inf, x[big])
    return out


def to_bits(x: np.ndarray) -> np.ndarray:
    """uint16 bfloat16 bit patterns of float64 values, rounded as above."""
    r = round_f64(x).astype(np.float32)  # exact: r is a bfloat16 value
    return (r.view(np.uint32) >> 16).astype(np.uint16)


def from_bits(bits: np.ndarray) -> np.ndarray:
    """float64 values of uint16 bfloat16 bit patterns."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)
