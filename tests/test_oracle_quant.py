"""Pins for the oracle's 1x128 / 128x128 quantizers and BF16 rounding (CPU).

Pinned against: an exact rational-arithmetic restatement on tiny inputs, the
invariants Fig. 13-1 and Q1 of Lesson 13 imply (amax maps to +-448; a group's
scale depends only on its own 128 values), torch's bfloat16 conversion, and a
frexp-based definition of the power-of-two round-up.
"""

import math
from fractions import Fraction

import numpy as np
import torch

from oracle import bf16, e4m3, quant
from moe_grouped_gemm_act_b200 import inputs


# ---------------------------------------------------------------- exact helpers
def f32_round(q: Fraction) -> float:
    """Round an exact rational to the nearest float32 (ties to even), in exact
    integer arithmetic -- independent of numpy's float64 -> float32 path."""
    if q == 0:
        return 0.0
    s = -1 if q < 0 else 1
    a = abs(q)
    e = math.floor(math.log2(a.numerator) - math.log2(a.denominator))
    # fix e so that 2**e <= a < 2**(e+1)
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -126)                         # subnormal range: fixed quantum
    quantum = Fraction(2) ** (e - 23)
    r = a / quantum
    n = r.numerator // r.denominator
    rem = r - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return s * float(n * quantum)


def e4m3_nearest(x: float) -> int:
    return int(e4m3.encode_bruteforce(np.array([x], np.float64))[0])


def quantize_group_exact(vals, pow2=False):
    """One group, step by step in exact arithmetic."""
    amax = max(abs(Fraction(float(v))) for v in vals)
    alpha = f32_round(amax / 448)
    if pow2 and alpha > 0:
        m, e = math.frexp(alpha)
        alpha = alpha if m == 0.5 else math.ldexp(1.0, e)
    if alpha == 0:
        return [0] * len(vals), alpha
    codes = []
    for v in vals:
        qv = f32_round(Fraction(float(v)) / Fraction(alpha))
        if qv == 0 and math.copysign(1.0, float(v)) < 0:
            qv = -0.0
        codes.append(e4m3_nearest(qv))
    return codes, alpha


# ---------------------------------------------------------------- 1x128
def test_1x128_matches_exact_restatement():
    x = inputs.activations(3, 256, seed=11, outliers=True)
    x[1, 128:256] *= np.float32(1e-3)
    x[2, 0:128] = 0.0                     # all-zero group
    x[2, 5] = -0.0
    q, alpha = quant.quantize_1x128(x)
    for i in range(3):
        for g in range(2):
            codes, a = quantize_group_exact(x[i, g * 128:(g + 1) * 128])
            assert np.float32(a) == alpha[i, g]
            assert list(q[i, g * 128:(g + 1) * 128]) == codes


def test_1x128_pow2_matches_exact_restatement():
    x = inputs.activations(2, 256, seed=12, outliers=True)
    q, alpha = quant.quantize_1x128(x, pow2=True)
    for i in range(2):
        for g in range(2):
            codes, a = quantize_group_exact(x[i, g * 128:(g + 1) * 128], pow2=True)
            assert np.float32(a) == alpha[i, g]
            assert list(q[i, g * 128:(g + 1) * 128]) == codes


def test_amax_maps_to_448():
    x = inputs.activations(64, 1024, seed=13, outliers=True)
    q, alpha = quant.quantize_1x128(x)
    g = x.reshape(64, 8, 128)
    arg = np.abs(g).argmax(axis=2)
    codes = q.reshape(64, 8, 128)
    top = np.take_along_axis(codes, arg[..., None], axis=2)[..., 0]
    sign = np.signbit(np.take_along_axis(g, arg[..., None], axis=2)[..., 0])
    assert np.all(top == np.where(sign, 0xFE, 0x7E))
    assert np.all(np.abs(e4m3.decode(q)) <= 448)


def test_pow2_scale_properties():
    x = inputs.activations(64, 1024, seed=14, outliers=True)
    q, alpha = quant.quantize_1x128(x, pow2=True)
    m, _ = np.frexp(alpha.astype(np.float64))
    assert np.all(m == 0.5)                                 # powers of two
    plain = (np.abs(x).reshape(64, 8, 128).max(axis=2).astype(np.float64) / 448)
    assert np.all(alpha >= plain.astype(np.float32))
    assert np.all(alpha / 2 < plain * (1 + 2 ** -23))
    top = np.abs(e4m3.decode(q)).reshape(64, 8, 128).max(axis=2)
    assert np.all((top >= 224) & (top <= 448))


def test_pow2_round_up_vs_frexp():
    g = np.random.default_rng(5)
    a = np.concatenate([
        (g.random(5000) * 10).astype(np.float32),
        np.float32(2.0) ** np.arange(-149, 127, dtype=np.float32),
        np.array([1.5e-45, 3e-45, 1e-40, 1.1754942e-38, 1.17549435e-38], np.float32),
    ])
    got = quant.pow2_round_up(a)
    for v, p in zip(a.tolist(), got.tolist()):
        m, e = math.frexp(v)
        want = v if m == 0.5 else math.ldexp(1.0, e)
        assert p == want, (v, p, want)


def test_dequant_error_bound():
    x = inputs.activations(32, 512, seed=15, outliers=True)
    q, alpha = quant.quantize_1x128(x)
    deq = quant.dequantize_1x128(q, alpha)
    a = np.repeat(alpha.astype(np.float64), 128, axis=1)
    t = x.astype(np.float64) / a
    # half a code spacing at |t|, plus the float32 rounding of the quotient
    _, ex = np.frexp(np.maximum(np.abs(t), 2.0 ** -6))
    half_ulp = np.ldexp(1.0, ex - 1 - 3 - 1)
    assert np.all(np.abs(deq - x) <= (half_ulp * (1 + 2 ** -20) + 0) * a)


def test_group_locality_of_outliers():
    # Q1 of Lesson 13: an outlier only affects the 128 values of its group.
    x = inputs.activations(4, 512, seed=16)
    q0, a0 = quant.quantize_1x128(x)
    y = x.copy()
    y[2, 300] = np.float32(1000.0)
    q1, a1 = quant.quantize_1x128(y)
    changed = np.argwhere(q0 != q1)
    assert len(changed) > 0
    assert np.all(changed[:, 0] == 2) and np.all(changed[:, 1] // 128 == 2)
    assert np.array_equal(np.argwhere(a0 != a1), [[2, 2]])


# ---------------------------------------------------------------- 128x128
def test_128x128_matches_exact_restatement_partial_block():
    w = inputs.weights((130, 256), seed=17)       # last block holds 2 rows
    q, beta = quant.quantize_128x128(w)
    assert beta.shape == (2, 2)
    for b in range(2):
        for g in range(2):
            blk = w[b * 128:(b + 1) * 128, g * 128:(g + 1) * 128]
            codes, s = quantize_group_exact(blk.ravel())
            assert np.float32(s) == beta[b, g]
            assert np.array_equal(q[b * 128:(b + 1) * 128, g * 128:(g + 1) * 128].ravel(),
                                  np.array(codes, np.uint8))


def test_128x128_is_1x128_of_the_block_amax():
    # a 128x128 block quantized alone equals a 1x128 quantization of a row
    # layout with the same amax (both are "amax / 448 then divide").
    w = inputs.weights((128, 128), seed=18)
    q, beta = quant.quantize_128x128(w)
    flat = w.reshape(1, -1)
    q2, a2 = quant.quantize_1x128(flat.reshape(128, 128))
    amax = np.abs(w).max()
    assert beta[0, 0] == np.float32(np.float64(amax) / 448)
    assert np.all(np.abs(e4m3.decode(q)) <= 448)
    assert (q == 0x7E).sum() + (q == 0xFE).sum() >= 1


# ---------------------------------------------------------------- bf16
def test_bf16_matches_torch_for_float32_inputs():
    g = np.random.default_rng(3)
    v = np.concatenate([
        g.standard_normal(100000).astype(np.float32) * 1000,
        np.float32(2.0) ** np.arange(-140, 120, dtype=np.float32),
    ])
    # include exact ties: bf16 value + half spacing
    base = torch.from_numpy(v).to(torch.bfloat16).to(torch.float32).numpy()
    ties = base + np.abs(base) * np.float32(2 ** -9)
    v = np.concatenate([v, ties.astype(np.float32), -v])
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = bf16.to_bits(v.astype(np.float64))
    assert np.array_equal(got, ref)


def test_bf16_rounds_float64_directly():
    # 1 + 2**-8 + 2**-40: just above a bf16 tie -> must round up, whereas
    # rounding to float32 first would create an exact tie and round to even (1).
    x = 1 + 2.0 ** -8 + 2.0 ** -40
    assert bf16.round_f64(np.array([x]))[0] == 1 + 2.0 ** -7
    assert bf16.round_f64(np.array([1 + 2.0 ** -8]))[0] == 1.0
    assert bf16.round_f64(np.array([1 + 3 * 2.0 ** -8]))[0] == 1 + 2.0 ** -6
