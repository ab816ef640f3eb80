"""Fine-grained FP8 quantization: 1x128 activation groups, 128x128 weight blocks.

Lesson 13, Fig. 13-1 ("activation A: 1 x 128 groups", "weight B: 128 x 128
blocks") and the answer to Q1:

* activation A [M, K]: one scale per row per 128-wide group along K,
  alpha = max|A_group| / 448, so an outlier only affects its own 128 values;
* weight B [N, K]: one FP32 scale beta per 128 x 128 block, quantized offline;
* scales are FP32; newer versions also allow UE8M0 (power-of-two) scales.

Readings taken where the pages are silent:

* the code of an element is E4M3_RNE(fl32(x / alpha)): the float32 quotient,
  correctly rounded, then rounded to E4M3 (ties to even, satfinite);
* alpha = fl32(amax / 448), the correctly rounded float32 quotient;
* a group whose amax is 0 gets alpha = 0 and every code 0x00;
* power-of-two mode rounds alpha *up* to the next power of two
  (2**ceil(log2 alpha), from alpha's float32 bits) before dividing;
* a partial 128x128 block (N not a multiple of 128) takes its amax over the
  rows that exist.

float32 quotients are computed in float64 and rounded once to float32.  For a
quotient of two float32 values this equals the correctly rounded float32
quotient (double rounding is innocuous for division because 53 >= 2*24 + 2).
"""

from __future__ import annotations

import numpy as np

from . import e4m3

GROUP = 128  # Lesson 13, Fig. 13-1: 1 x 128 groups, 128 x 128 blocks


def f32_div(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Correctly rounded float32 quotient a / b of float32 operands."""
    return (np.asarray(a, np.float32).astype(np.float64)
            / np.asarray(b, np.float32).astype(np.float64)).astype(np.float32)


def pow2_round_up(alpha: np.ndarray) -> np.ndarray:
    """Smallest power of two >= alpha, for float32 alpha >= 0 (0 stays 0).

    Read from the float32 bits: a normal value with an all-zero mantissa is
    already a power of two; otherwise the exponent goes up by one and the
    mantissa is cleared.  A subnormal mantissa field m becomes the smallest
    power of two >= m (which may carry into the smallest normal exponent).
    """
    a = np.ascontiguousarray(alpha, dtype=np.float32)
    bits = a.view(np.uint32).copy()
    exp = (bits >> 23) & 0xFF
    man = bits & 0x7FFFFF
    out = bits.copy()
    normal = (exp > 0) & (man != 0)
    out[normal] = (exp[normal] + 1) << 23
    sub = (exp == 0) & (man != 0)
    if np.any(sub):
        m = man[sub].astype(np.uint64)
        p = np.ones_like(m)
        while np.any(p < m):
            p = np.where(p < m, p << 1, p)
        out[sub] = p.astype(np.uint32)
    return out.view(np.float32).reshape(a.shape)


def _scale_and_codes(x_groups: np.ndarray, amax: np.ndarray, pow2: bool):
    """Shared tail of both quantizers.

    ``x_groups``: float32 values; ``amax``: float32 amax broadcastable against
    ``x_groups``.  Returns (codes uint8 shaped like x_groups, alpha float32
    shaped like amax).
    """
    alpha = f32_div(amax, np.float32(e4m3.E4M3_MAX))
    if pow2:
        alpha = pow2_round_up(alpha)
    safe = np.where(alpha == 0, np.float32(1), alpha)
    quotient = f32_div(x_groups, safe)
    codes = e4m3.encode_rne(quotient)
    codes = np.where(alpha == 0, np.uint8(0), codes).astype(np.uint8)
    return codes, alpha


def quantize_1x128(x: np.ndarray, pow2: bool = False):
    """Quantize activations x [M, K] (K % 128 == 0) per 1 x 128 group.

    Returns (q uint8 [M, K], alpha float32 [M, K/128]) with the logical
    (row-major, [M, K/128]) scale layout of the Lesson 13 exercise.  The
    library stores alpha transposed (MN-major, [K/128, ld]); tests transpose.
    """
    x = np.asarray(x, dtype=np.float32)
    M, K = x.shape
    if K % GROUP:
        raise ValueError("K must be a multiple of 128")
    g = x.reshape(M, K // GROUP, GROUP)
    amax = np.abs(g).max(axis=2, keepdims=True)  # exact in float32
    codes, alpha = _scale_and_codes(g, amax, pow2)
    return codes.reshape(M, K), alpha[:, :, 0]


def quantize_128x128(w: np.ndarray, pow2: bool = False):
    """Quantize weights w [N, K] (K % 128 == 0) per 128 x 128 block.

    Returns (q uint8 [N, K], beta float32 [ceil(N/128), K/128]).  The last
    block along N holds N % 128 rows when N is not a multiple of 128.
    """
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    if K % GROUP:
        raise ValueError("K must be a multiple of 128")
    nb, kg = -(-N // GROUP), K // GROUP
    q = np.empty((N, K), dtype=np.uint8)
    beta = np.empty((nb, kg), dtype=np.float32)
    for b in range(nb):
        rows = w[b * GROUP:(b + 1) * GROUP]  # [r, K], r <= 128
        blk = rows.reshape(rows.shape[0], kg, GROUP)
        amax = np.abs(blk).max(axis=(0, 2), keepdims=True)  # [1, kg, 1]
        codes, s = _scale_and_codes(blk, amax, pow2)
        q[b * GROUP:(b + 1) * GROUP] = codes.reshape(rows.shape[0], K)
        beta[b] = s[0, :, 0]
    return q, beta


def quantize_128x128_grouped(w: np.ndarray, pow2: bool = False):
    """Per-expert 128 x 128 quantization of w [G, N, K]."""
    w = np.asarray(w, dtype=np.float32)
    qs, bs = zip(*(quantize_128x128(w[e], pow2) for e in range(w.shape[0])))
    return np.stack(qs), np.stack(bs)


def dequantize_1x128(q: np.ndarray, alpha: np.ndarray) -> np.ndarray:
    """float64 values q * alpha for 1 x 128 groups (alpha [M, K/128])."""
    v = e4m3.decode(q)
    return v * np.repeat(np.asarray(alpha, np.float64), GROUP, axis=1)


def dequantize_128x128(q: np.ndarray, beta: np.ndarray) -> np.ndarray:
    """float64 values q * beta for 128 x 128 blocks (beta [ceil(N/128), K/128])."""
    v = e4m3.decode(q)
    N, K = v.shape
    full = np.repeat(np.repeat(np.asarray(beta, np.float64), GROUP, axis=0),
                     GROUP, axis=1)
    return v * full[:N, :K]
