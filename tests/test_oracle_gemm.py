"""Pins for the oracle's block-scaled GEMM and its grouped forms (CPU only).

Pinned against:
* the worked exercise of Lesson 13 (its inputs regenerated from the stated seed
  and draws, its reference -- dequantize each block, then multiply -- and its
  tolerance, atol 1e-5);
* an element-by-element restatement of Fig. 13-1 in plain Python on tiny
  shapes (partial 128-column block included);
* closed forms (constant codes, integer results);
* the grouped layouts' definitions (Fig. 13-3, Q3): per-expert dense results,
  untouched padding / masked rows.
Planted-mistake tests check that each pin actually catches the mistakes it is
meant to catch.
"""

import json
import os

import numpy as np
import pytest

from oracle import bf16, e4m3, gemm, quant
from moe_grouped_gemm_act_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def exercise_inputs():
    spec = json.load(open(os.path.join(GOLDEN, "lesson13_exercise.json")))
    np.random.seed(spec["seed"])
    M, N, K, bk, bn = spec["M"], spec["N"], spec["K"], spec["block_k"], spec["block_n"]
    dims = {"M": M, "N": N, "K": K, "K/block_k": K // bk, "N/block_n": N // bn}
    out = {}
    for d in spec["draws"]:
        shape = tuple(dims[s] for s in d["shape"])
        if d["kind"] == "randint":
            v = np.random.randint(d["low"], d["high"], size=shape)
        else:
            v = np.random.uniform(d["low"], d["high"], size=shape)
        out[d["name"]] = v.astype(np.float32)
    return spec, out


def page_reference(A, B, SA, SB):
    """The exercise's own reference: dequantize each K block of A and B with
    its scales, multiply, sum the blocks (float64)."""
    M, K = A.shape
    N = B.shape[0]
    ref = np.zeros((M, N))
    for b in range(K // 128):
        ks = slice(b * 128, (b + 1) * 128)
        a_sub = A[:, ks].astype(np.float64) * SA[:, b:b + 1]
        b_sub = B[:, ks].astype(np.float64) * SB[np.arange(N) // 128, b][:, None]
        ref += a_sub @ b_sub.T
    return ref


def oracle_on_exercise(fn=gemm.fp8_gemm_nt_f64):
    spec, d = exercise_inputs()
    qa = e4m3.encode_rne(d["A_sim"])       # integers in [-10, 10): exact codes
    qb = e4m3.encode_rne(d["B_sim"])
    assert np.array_equal(e4m3.decode(qa), d["A_sim"])
    return spec, d, fn(qa, d["S_A"], qb, d["S_B"])


def test_lesson13_exercise():
    spec, d, out = oracle_on_exercise()
    ref = page_reference(d["A_sim"], d["B_sim"], d["S_A"], d["S_B"])
    assert np.allclose(out, ref, atol=spec["check"]["atol"], rtol=0)


def elementwise(qa, alpha, qb, beta):
    """Fig. 13-1 element by element, plain Python floats."""
    M, K = qa.shape
    N = qb.shape[0]
    av, bv = e4m3.decode(qa).tolist(), e4m3.decode(qb).tolist()
    out = np.zeros((M, N))
    for i in range(M):
        for j in range(N):
            s = 0.0
            for g in range(K // 128):
                part = 0.0
                for k in range(128):
                    part += av[i][128 * g + k] * bv[j][128 * g + k]
                s += float(alpha[i, g]) * float(beta[j // 128, g]) * part
            out[i, j] = s
    return out


def small_case(m=3, n=136, k=256, seed=21):
    x = inputs.activations(m, k, seed=seed, outliers=True)
    w = inputs.weights((n, k), seed=seed + 1)
    qa, alpha = quant.quantize_1x128(x)
    qb, beta = quant.quantize_128x128(w)
    return qa, alpha, qb, beta


def test_elementwise_restatement_partial_block():
    qa, alpha, qb, beta = small_case()
    got = gemm.fp8_gemm_nt_f64(qa, alpha, qb, beta)
    ref = elementwise(qa, alpha, qb, beta)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-300)


def test_dequantized_matmul_equals_formula():
    qa, alpha, qb, beta = small_case(m=40, n=272, k=640, seed=31)
    got = gemm.fp8_gemm_nt_f64(qa, alpha, qb, beta)
    ref = quant.dequantize_1x128(qa, alpha) @ quant.dequantize_128x128(qb, beta).T
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_closed_form_constant_codes():
    M, N, K = 4, 256, 512
    qa = np.full((M, K), 0x38, np.uint8)             # 1.0
    qb = np.full((N, K), 0x40, np.uint8)             # 2.0
    alpha = np.tile(np.arange(1, 5, dtype=np.float32), (M, 1))   # alpha[i,g]=g+1
    beta = np.array([[1, 1, 1, 1], [0.5, 0.5, 0.5, 0.5]], np.float32)
    d = gemm.fp8_gemm_nt_f64(qa, alpha, qb, beta)
    # sum_g (g+1) * beta_jb * 128 * 2
    want0 = 256 * (1 + 2 + 3 + 4)
    assert np.all(d[:, :128] == want0) and np.all(d[:, 128:] == want0 / 2)
    assert np.all(bf16.to_bits(d[:, :128]) == bf16.to_bits(np.array([2560.0]))[0])


def test_closed_form_integer_exact():
    # integer codes in [-4, 4] with unit scales: D is an exact integer
    g = np.random.default_rng(9)
    M, N, K = 8, 64, 1024
    a = g.integers(-4, 5, size=(M, K)).astype(np.float32)
    b = g.integers(-4, 5, size=(N, K)).astype(np.float32)
    qa, qb = e4m3.encode_rne(a), e4m3.encode_rne(b)
    d = gemm.fp8_gemm_nt_f64(qa, np.ones((M, 8), np.float32), qb,
                             np.ones((1, 8), np.float32))
    assert np.array_equal(d, a.astype(np.int64) @ b.astype(np.int64).T)


# ------------------------------------------------------------- planted mistakes
def mutant_col_index(qa, alpha, qb, beta):
    """Fig. 13-1 with j % 128 instead of floor(j / 128) for beta's column."""
    a, b = e4m3.decode(qa), e4m3.decode(qb)
    N = qb.shape[0]
    d = np.zeros((qa.shape[0], N))
    for g in range(qa.shape[1] // 128):
        ks = slice(g * 128, (g + 1) * 128)
        idx = (np.arange(N) % 128) % beta.shape[0]
        d += (a[:, ks] @ b[:, ks].T) * alpha[:, g][:, None] * beta[idx, g][None, :]
    return d


def mutant_dropped_alpha(qa, alpha, qb, beta):
    return gemm.fp8_gemm_nt_f64(qa, np.ones_like(alpha), qb, beta)


def mutant_last_group_only(qa, alpha, qb, beta):
    """Scales of the last group applied to every group."""
    a2 = np.repeat(alpha[:, -1:], alpha.shape[1], axis=1)
    b2 = np.repeat(beta[:, -1:], beta.shape[1], axis=1)
    return gemm.fp8_gemm_nt_f64(qa, a2, qb, b2)


@pytest.mark.parametrize("mutant", [mutant_col_index, mutant_dropped_alpha,
                                    mutant_last_group_only])
def test_planted_mistakes_are_caught(mutant):
    spec, d, out = oracle_on_exercise(mutant)
    ref = page_reference(d["A_sim"], d["B_sim"], d["S_A"], d["S_B"])
    assert not np.allclose(out, ref, atol=spec["check"]["atol"], rtol=0)


# ------------------------------------------------------------- grouped forms
def test_contiguous_matches_per_expert_dense_and_keeps_padding():
    lay = inputs.contiguous_layout(500, 4, seed=40)
    K, N, G = 256, 144, 4
    x = inputs.activations(lay.m_total, K, seed=41)
    w = inputs.weights((G, N, K), seed=42)
    qa, alpha = quant.quantize_1x128(x)
    qb, beta = quant.quantize_128x128_grouped(w)
    sentinel = np.full((lay.m_total, N), 0x7FC1, np.uint16)
    out = gemm.m_grouped_contiguous(qa, alpha, qb, beta, lay.m_indices, sentinel)
    assert lay.m_total % 128 == 0
    for i in range(lay.m_total):
        e = lay.m_indices[i]
        if e < 0:
            assert np.all(out[i] == 0x7FC1)
        else:
            want = bf16.to_bits(elementwise(qa[i:i + 1], alpha[i:i + 1], qb[e], beta[e]))
            assert np.array_equal(out[i], want[0])


def test_masked_matches_per_expert_dense_and_keeps_rows():
    G, m_max, N, K = 3, 130, 128, 256
    masked = np.array([0, 130, 57], np.int32)
    x = inputs.activations(G * m_max, K, seed=50).reshape(G, m_max, K)
    w = inputs.weights((G, N, K), seed=51)
    qa, alpha = zip(*(quant.quantize_1x128(x[e]) for e in range(G)))
    qa, alpha = np.stack(qa), np.stack(alpha)
    qb, beta = quant.quantize_128x128_grouped(w)
    sentinel = np.full((G, m_max, N), 0xFFFF, np.uint16)
    out = gemm.m_grouped_masked(qa, alpha, qb, beta, masked, sentinel)
    for e in range(G):
        m = masked[e]
        assert np.all(out[e, m:] == 0xFFFF)
        if m:
            want = bf16.to_bits(quant.dequantize_1x128(qa[e, :m], alpha[e, :m])
                                @ quant.dequantize_128x128(qb[e], beta[e]).T)
            assert np.array_equal(out[e, :m], want)


def test_masked_clamps_out_of_range_counts():
    G, m_max, N, K = 2, 8, 16, 128
    qa = np.full((G, m_max, K), 0x38, np.uint8)
    alpha = np.ones((G, m_max, 1), np.float32)
    qb = np.full((G, N, K), 0x38, np.uint8)
    beta = np.ones((G, 1, 1), np.float32)
    out = gemm.m_grouped_masked(qa, alpha, qb, beta, np.array([-5, 99]),
                                np.zeros((G, m_max, N), np.uint16))
    assert np.all(out[0] == 0)
    assert np.all(bf16.from_bits(out[1]) == 128.0)


# ------------------------------------------------------------- D = C + A B^T
def test_accumulate_with_zero_c_is_the_plain_gemm():
    qa, alpha, qb, beta = small_case(m=24, n=200, k=384, seed=41)
    c = np.zeros((24, 200), np.float32)
    assert np.array_equal(gemm.fp8_gemm_nt_accumulate(qa, alpha, qb, beta, c),
                          gemm.fp8_gemm_nt(qa, alpha, qb, beta))


def test_accumulate_with_zero_product_rounds_c_like_torch():
    import torch
    g = np.random.default_rng(42)
    c = (g.standard_normal((16, 136)) * 7).astype(np.float32)
    qa = np.zeros((16, 256), np.uint8)                      # all +0.0
    qb = e4m3.encode_rne(g.standard_normal((136, 256)).astype(np.float32))
    got = gemm.fp8_gemm_nt_accumulate(qa, np.ones((16, 2), np.float32), qb,
                                      np.ones((2, 2), np.float32), c)
    want = torch.from_numpy(c).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)


def test_accumulate_integer_exact():
    g = np.random.default_rng(43)
    M, N, K = 8, 64, 512
    a = g.integers(-4, 5, size=(M, K)).astype(np.float32)
    b = g.integers(-4, 5, size=(N, K)).astype(np.float32)
    c = g.integers(-100, 101, size=(M, N)).astype(np.float32)
    d = gemm.fp8_gemm_nt_accumulate_f64(e4m3.encode_rne(a), np.ones((M, 4), np.float32),
                                        e4m3.encode_rne(b), np.ones((1, 4), np.float32), c)
    assert np.array_equal(d, a.astype(np.int64) @ b.astype(np.int64).T + c.astype(np.int64))


def test_accumulate_rounds_once_after_adding_c():
    # A.B = 1 + 2^-8 (a tie between two BF16 values, rounding to 1.0) and
    # C = 2^-8: rounding once gives BF16(1 + 2^-7) = 0x3F81; rounding the
    # product first and then adding C would give 0x3F80
    qa = np.zeros((1, 128), np.uint8)
    qb = np.zeros((1, 128), np.uint8)
    a = np.zeros((1, 128), np.float32)
    a[0, 0], a[0, 1] = 1.0, 2.0 ** -8
    qa[:] = e4m3.encode_rne(a)
    qb[0, 0], qb[0, 1] = e4m3.encode_rne(np.array([1.0, 1.0], np.float32))
    one = np.ones((1, 1), np.float32)
    assert gemm.fp8_gemm_nt_f64(qa, one, qb, one)[0, 0] == 1.0 + 2.0 ** -8
    c = np.array([[2.0 ** -8]], np.float32)
    assert gemm.fp8_gemm_nt_accumulate(qa, one, qb, one, c)[0, 0] == 0x3F81
    twice = bf16.to_bits(bf16.round_f64(gemm.fp8_gemm_nt_f64(qa, one, qb, one)) + c)
    assert twice[0, 0] == 0x3F80


# ------------------------------------------------------------- operand layouts
@pytest.mark.parametrize("layout,spec", [("nt", "mk,nk->mn"), ("nn", "mk,kn->mn"),
                                         ("tn", "km,kn->mn"), ("tt", "km,nk->mn")])
def test_layouts_match_an_einsum_over_the_stored_operands(layout, spec):
    # the stored operands are contracted as they lie (no transposes), with
    # each element's scale looked up by its logical (row, K) position
    m, n, k = 24, 200, 384
    qa, alpha, qb, beta = small_case(m=m, n=n, k=k, seed=120)
    a_st = qa if layout[0] == "n" else np.ascontiguousarray(qa.T)
    b_st = qb if layout[1] == "t" else np.ascontiguousarray(qb.T)
    av = e4m3.decode(a_st)
    bv = e4m3.decode(b_st)
    ka = np.arange(k) // 128
    sa = alpha[:, ka] if layout[0] == "n" else alpha[:, ka].T          # like a_st
    sb_nk = beta[np.arange(n) // 128][:, ka]                            # [N, K]
    sb = sb_nk if layout[1] == "t" else sb_nk.T                         # like b_st
    want = np.einsum(spec, av * sa, bv * sb)
    got = gemm.fp8_gemm_f64(layout, a_st, alpha, b_st, beta)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_layout_names_are_checked():
    qa, alpha, qb, beta = small_case(m=8, n=16, k=128, seed=121)
    with pytest.raises(ValueError):
        gemm.fp8_gemm_f64("tx", qa, alpha, qb, beta)


def test_a_layout_mix_up_is_caught():
    # reading an "nn" B as if it were stored [N, K] fails the einsum pin
    m, n, k = 16, 128, 128
    qa, alpha, qb, beta = small_case(m=m, n=n, k=k, seed=122)
    b_kn = np.ascontiguousarray(qb.T)
    right = gemm.fp8_gemm_f64("nn", qa, alpha, b_kn, beta)
    wrong = gemm.fp8_gemm_nt_f64(qa, alpha, np.ascontiguousarray(b_kn[:n, :k]), beta)
    assert not np.allclose(right, wrong)
