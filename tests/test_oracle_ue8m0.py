"""Pins for the oracle's UE8M0 encoding and packed scale layout (CPU only).

UE8M0 (Lesson 13, Fig. 13-1 text) is an 8-bit biased exponent; the packed
layout (Deep dive, section 3) puts four of them in one 32-bit integer,
MN-major.  Pinned against:
* the float32 exponent field read from the IEEE bit pattern (the oracle
  itself works from numpy.frexp), for every normal power of two;
* a worked example with the expected words written out as hex literals;
* the byte view of the packed words (little-endian groups in K order);
* round trips through decode and through the power-of-two quantizer;
* rejection of everything that is not +0 or a normal power of two.
"""

import numpy as np
import pytest

from oracle import e4m3, gemm, quant, ue8m0
from moe_grouped_gemm_act_b200 import inputs


def test_encode_matches_the_float32_exponent_field_for_every_power_of_two():
    e = np.arange(-126, 128)
    x = np.ldexp(1.0, e).astype(np.float32)
    field = (x.view(np.uint32) >> 23) & 0xFF
    assert np.array_equal(ue8m0.encode(x), field.astype(np.uint8))
    assert np.array_equal(ue8m0.encode(x).astype(np.int64), e + 127)
    assert np.array_equal(ue8m0.decode(ue8m0.encode(x)), x.astype(np.float64))


def test_zero_encodes_as_zero():
    assert ue8m0.encode(np.zeros(3, np.float32)).tolist() == [0, 0, 0]


def test_worked_example_words():
    # row 0: scales 1, 2, 0.5, 4 | 2^-10  ->  bytes 127, 128, 126, 129 | 117
    # row 1: 0, 2^127, 2^-126, 1 | 0      ->  bytes 0, 254, 1, 127 | 0
    alpha = np.array([[1.0, 2.0, 0.5, 4.0, 2.0 ** -10],
                      [0.0, 2.0 ** 127, 2.0 ** -126, 1.0, 0.0]], np.float32)
    got = ue8m0.pack_1x128(alpha).view(np.uint32)
    want = np.array([[0x817E807F, 0x7F01FE00],
                     [0x00000075, 0x00000000]], np.uint32)
    assert got.shape == (2, 2)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("m,kg", [(1, 1), (37, 5), (64, 8), (5, 131)])
def test_packed_bytes_are_the_groups_in_k_order(m, kg):
    rng = inputs.rng(60 + kg)
    e = rng.integers(-126, 128, size=(m, kg))
    alpha = np.ldexp(1.0, e).astype(np.float32)
    alpha[rng.random((m, kg)) < 0.1] = 0.0
    words = ue8m0.pack_1x128(alpha)
    nw = -(-kg // 4)
    assert words.shape == (nw, m) and words.dtype == np.int32
    as_bytes = words.view(np.uint8).reshape(nw, m, 4)       # little-endian
    codes = ue8m0.encode(alpha)
    padded = np.zeros((m, nw * 4), np.uint8)
    padded[:, :kg] = codes
    assert np.array_equal(as_bytes.transpose(1, 0, 2).reshape(m, nw * 4), padded)


def test_power_of_two_quantizer_scales_round_trip():
    x = inputs.activations(48, 1024, seed=61, outliers=True)
    x[3, 128:256] = 0.0                                       # a zero group
    _, alpha = quant.quantize_1x128(x, pow2=True)
    codes = ue8m0.encode(alpha)
    assert codes[3, 1] == 0
    nz = alpha != 0
    assert np.array_equal(ue8m0.decode(codes[nz]), alpha[nz].astype(np.float64))


@pytest.mark.parametrize("bad", [3.0, 0.75, -2.0, -0.0, np.inf, np.nan, 2.0 ** -130, 1e-45])
def test_rejects_values_that_are_not_a_normal_power_of_two(bad):
    with pytest.raises(ValueError):
        ue8m0.encode(np.array([1.0, bad], np.float32))


def test_fp32_scales_are_rejected():
    x = inputs.activations(8, 512, seed=62)
    _, alpha = quant.quantize_1x128(x)            # amax / 448: not powers of two
    with pytest.raises(ValueError):
        ue8m0.pack_1x128(alpha)


def mutant_big_endian(alpha):
    w = ue8m0.pack_1x128(alpha).view(np.uint32)
    return w.byteswap().view(np.int32)


def mutant_row_major(alpha):
    return np.ascontiguousarray(ue8m0.pack_1x128(alpha).T)


@pytest.mark.parametrize("mutant", [mutant_big_endian, mutant_row_major])
def test_planted_layout_mistakes_are_caught(mutant):
    alpha = np.array([[1.0, 2.0, 0.5, 4.0, 2.0 ** -10],
                      [0.0, 2.0 ** 127, 2.0 ** -126, 1.0, 0.0]], np.float32)
    want = np.array([[0x817E807F, 0x7F01FE00],
                     [0x00000075, 0x00000000]], np.uint32)
    got = mutant(alpha).view(np.uint32)
    assert got.shape != want.shape or not np.array_equal(got, want)


# ------------------------------------------------ unpacking and the UE8M0 GEMM
def test_unpack_inverts_pack_including_zero_groups():
    rng = np.random.default_rng(11)
    for m, kg in [(5, 1), (130, 7), (64, 16)]:
        sf = np.ldexp(1.0, rng.integers(-20, 21, size=(m, kg))).astype(np.float32)
        sf[rng.random((m, kg)) < 0.1] = 0.0
        packed = ue8m0.pack_1x128(sf)
        wide = np.zeros((packed.shape[0], m + 3), np.int32)   # a TMA-aligned ld
        wide[:, :m] = packed
        assert np.array_equal(ue8m0.unpack_1x128(wide, m, kg), sf.astype(np.float64))


def _pow2_case(m, n, k, seed):
    x = inputs.activations(m, k, seed=seed, outliers=True)
    w = inputs.weights((n, k), seed=seed + 1)
    qa, alpha = quant.quantize_1x128(x, pow2=True)
    qb, beta = quant.quantize_128x128(w, pow2=True)
    return qa, alpha, qb, beta


def test_ue8m0_gemm_with_block_scales_is_the_dense_oracle():
    # B's 128 x 128 block scales written out per row (each row of a block
    # carries its block's codes): the packed-code GEMM must reproduce the
    # pinned Fig. 13-1 oracle exactly (same float64 operations)
    qa, alpha, qb, beta = _pow2_case(150, 264, 640, seed=3)
    beta_rows = beta[np.arange(264) // 128]
    got = gemm.fp8_gemm_nt_ue8m0_f64(qa, ue8m0.pack_1x128(alpha), qb,
                                     ue8m0.pack_1x128(beta_rows))
    assert np.array_equal(got, gemm.fp8_gemm_nt_f64(qa, alpha, qb, beta))


def test_rowscaled_gemm_matches_an_elementwise_restatement():
    # distinct scales on every row of B (not block-constant), brute force
    rng = np.random.default_rng(5)
    m, n, k = 3, 5, 256
    qa = e4m3.encode_rne(rng.integers(-6, 7, size=(m, k)).astype(np.float32))
    qb = e4m3.encode_rne(rng.integers(-6, 7, size=(n, k)).astype(np.float32))
    alpha = np.ldexp(1.0, rng.integers(-3, 4, size=(m, 2)))
    beta = np.ldexp(1.0, rng.integers(-3, 4, size=(n, 2)))
    a, b = e4m3.decode(qa), e4m3.decode(qb)
    want = np.zeros((m, n))
    for i in range(m):
        for j in range(n):
            for kk in range(k):
                want[i, j] += alpha[i, kk // 128] * beta[j, kk // 128] * a[i, kk] * b[j, kk]
    got = gemm.fp8_gemm_nt_rowscaled_f64(qa, alpha, qb, beta)
    assert np.allclose(got, want, rtol=1e-12, atol=0)
    # a mistake in the byte order of the packed words is caught
    packed = ue8m0.pack_1x128(beta.astype(np.float32))
    swapped = packed.view(np.uint8).reshape(packed.shape + (4,))[..., ::-1].copy().view(np.int32)
    swapped = swapped.reshape(packed.shape)
    bad = gemm.fp8_gemm_nt_ue8m0_f64(qa, ue8m0.pack_1x128(alpha.astype(np.float32)), qb, swapped)
    assert not np.allclose(bad, want)
