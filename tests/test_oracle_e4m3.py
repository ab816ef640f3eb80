"""Pins for the oracle's E4M3 table and encoder (CPU only).

Pinned against: the page's stated format facts (Lesson 13, Fig. 13-1 / Q1),
torch's independent float8_e4m3fn conversions, and exhaustive brute force.
"""

import json
import os

import numpy as np
import pytest
import torch

from oracle import e4m3

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_page_facts():
    facts = json.load(open(os.path.join(GOLDEN, "e4m3_facts.json")))["facts"]
    finite = e4m3.DECODE[np.isfinite(e4m3.DECODE)]
    assert np.max(np.abs(finite)) == facts["max_abs"]
    # 1 sign + 4 exponent + 3 mantissa bits: 2 * 2**4 * 2**3 = 256 codes
    assert 1 + facts["exponent_bits"] + facts["mantissa_bits"] == facts["total_bits"]
    assert len(e4m3.DECODE) == 2 ** facts["total_bits"]
    # exactly the two all-ones patterns are NaN (FN flavour, no infinities)
    assert [c for c in range(256) if np.isnan(e4m3.DECODE[c])] == [0x7F, 0xFF]
    assert not np.any(np.isinf(e4m3.DECODE))


def test_decode_matches_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = e4m3.DECODE
    both_nan = np.isnan(ref) & np.isnan(ours)
    assert np.all(both_nan | (ref == ours))
    # signed zero
    assert np.signbit(ours[0x80]) and not np.signbit(ours[0x00])


def test_positive_codes_increasing():
    pos = e4m3.DECODE[:0x7F]
    assert np.all(np.diff(pos) > 0)
    assert e4m3.DECODE[0x01] == 2.0 ** -9 and e4m3.DECODE[0x08] == 2.0 ** -6


def _boundary_values():
    """All codes, all midpoints between neighbours, and float32 neighbours of
    each, on both signs, plus values beyond the range."""
    pos = e4m3.DECODE[:0x7F]
    mids = (pos[:-1] + pos[1:]) / 2
    base = np.concatenate([pos, mids, [448.0, 456.0, 464.0, 479.0, 480.0,
                                       500.0, 1e4, 3e38, 1e-30, 1e-45]])
    base = base.astype(np.float32)
    up = np.nextafter(base, np.float32(np.inf))
    dn = np.nextafter(base, np.float32(0))
    vals = np.concatenate([base, up, dn])
    return np.concatenate([vals, -vals]).astype(np.float32)


def test_encode_matches_bruteforce_on_boundaries():
    v = _boundary_values()
    assert np.array_equal(e4m3.encode_rne(v), e4m3.encode_bruteforce(v))


def test_encode_matches_bruteforce_random():
    g = np.random.default_rng(123)
    v = np.concatenate([
        g.standard_normal(3000).astype(np.float32) * 100,
        (g.random(2000).astype(np.float32) - 0.5) * np.float32(0.05),
        g.standard_normal(1000).astype(np.float32) * 1e-3,
    ])
    assert np.array_equal(e4m3.encode_rne(v), e4m3.encode_bruteforce(v))


def test_encode_matches_torch_in_range():
    # torch's float -> float8_e4m3fn rounds to nearest even; it maps overflow
    # to NaN instead of saturating, so compare where |v| <= 448.
    v = _boundary_values()
    g = np.random.default_rng(7)
    v = np.concatenate([v, (g.standard_normal(200000) * 60).astype(np.float32)])
    v = v[np.abs(v) <= 448]
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(e4m3.encode_rne(v), ref)


def test_encode_special_cases():
    enc = lambda x: int(e4m3.encode_rne(np.array([x], np.float32))[0])
    assert enc(448.0) == 0x7E and enc(-448.0) == 0xFE
    assert enc(1e30) == 0x7E and enc(-1e30) == 0xFE          # satfinite
    assert enc(0.0) == 0x00 and enc(-0.0) == 0x80
    assert enc(-1e-9) == 0x80                                 # sign kept
    assert enc(2.0 ** -10) == 0x00                            # tie -> even (0)
    assert enc(3 * 2.0 ** -10) == 0x02                        # tie 1|2 -> 2
    assert enc(7.5 * 2.0 ** -9) == 0x08                       # subnormal->normal tie
    assert enc(1.0) == 0x38 and enc(-2.0) == 0xC0
    for n in range(-16, 17):                                  # small integers exact
        assert e4m3.DECODE[enc(float(n))] == n


@pytest.mark.parametrize("c", range(0, 0x7F))
def test_roundtrip_every_finite_code(c):
    for code in (c, c | 0x80):
        v = np.array([e4m3.DECODE[code]], np.float32)
        assert int(e4m3.encode_rne(v)[0]) == code
