"""Pins for the oracle's k-grouped contiguous GEMM (CPU only).

The group axis is K: group g's D[g] = C[g] + A_g B_g^T over its own K segment,
with 1x128 scales on both operands (Deep dive, section 3, the grouped GEMM
table; Lesson 13, Fig. 13-1 for the per-block scaling).

Pinned against:
* a per-element restatement in plain Python loops on a tiny case (an empty
  group and a segment of several blocks included);
* dequantize-then-multiply per segment (numpy matmul of the dequantized
  operands), on ragged M and N;
* the already pinned dense oracle, where B's row scales are constant over
  each 128-row block (the dense 128x128 case);
* closed forms: integer codes with unit scales give exact integer products;
  empty groups return C; the sum over groups is the product over all of K.
Planted-mistake tests check that the pins catch the plausible slips.
"""

import numpy as np
import pytest

from oracle import e4m3, gemm, quant
from moe_grouped_gemm_act_b200 import inputs


def case(m, n, k_sizes, seed, c=False):
    k_total = int(sum(k_sizes))
    a = inputs.activations(m, k_total, seed=seed, outliers=True)
    b = inputs.activations(n, k_total, seed=seed + 1)
    qa, alpha = quant.quantize_1x128(a)
    qb, beta = quant.quantize_1x128(b)
    cc = inputs.rng(seed + 2).standard_normal((len(k_sizes), m, n)) if c else None
    return qa, alpha, qb, beta, np.asarray(k_sizes), cc


def per_segment_dequantized(qa, alpha, qb, beta, k_sizes, c):
    a = quant.dequantize_1x128(qa, alpha)
    b = quant.dequantize_1x128(qb, beta)
    out, k0 = [], 0
    for g, size in enumerate(k_sizes):
        seg = slice(k0, k0 + int(size))
        d = a[:, seg] @ b[:, seg].T
        out.append(d + (c[g] if c is not None else 0.0))
        k0 += int(size)
    return np.stack(out)


def close(got, want):
    scale = max(np.abs(want).max(), 1e-300)
    return np.allclose(got, want, rtol=1e-12, atol=1e-12 * scale)


def test_elementwise_restatement_with_empty_group():
    k_sizes = [128, 0, 256]
    qa, alpha, qb, beta, ks, c = case(3, 5, k_sizes, seed=40, c=True)
    got = gemm.k_grouped_contiguous_f64(qa, alpha, qb, beta, ks, c)
    av, bv = e4m3.decode(qa), e4m3.decode(qb)
    want = np.array(c, dtype=np.float64, copy=True)
    starts = np.concatenate([[0], np.cumsum(k_sizes)])
    for g in range(len(k_sizes)):
        for i in range(3):
            for j in range(5):
                acc = 0.0
                for k in range(int(starts[g]), int(starts[g + 1])):
                    acc += float(alpha[i, k // 128]) * float(beta[j, k // 128]) * av[i, k] * bv[j, k]
                want[g, i, j] += acc
    assert close(got, want)
    assert np.array_equal(got[1], c[1])


@pytest.mark.parametrize("m,n,k_sizes", [(40, 72, [384, 128, 0, 640]), (129, 8, [128] * 5)])
def test_matches_dequantized_matmul_per_segment(m, n, k_sizes):
    qa, alpha, qb, beta, ks, c = case(m, n, k_sizes, seed=41, c=True)
    got = gemm.k_grouped_contiguous_f64(qa, alpha, qb, beta, ks, c)
    assert close(got, per_segment_dequantized(qa, alpha, qb, beta, ks, c))


def test_block_constant_row_scales_equal_the_dense_gemm():
    # B's 1x128 scales repeated over each 128-row block make the dense
    # 128x128-scaled GEMM of every segment
    m, n, k_sizes = 24, 200, [256, 384]
    qa, alpha, _, _, ks, _ = case(m, n, k_sizes, seed=42)
    w = inputs.weights((n, sum(k_sizes)), seed=43)
    qb, beta_blk = quant.quantize_128x128(w)
    beta_rows = beta_blk[np.arange(n) // 128]
    got = gemm.k_grouped_contiguous_f64(qa, alpha, qb, beta_rows, ks)
    k0 = 0
    for g, size in enumerate(k_sizes):
        seg, blk = slice(k0, k0 + size), slice(k0 // 128, (k0 + size) // 128)
        want = gemm.fp8_gemm_nt_f64(qa[:, seg], alpha[:, blk], qb[:, seg], beta_blk[:, blk])
        assert close(got[g], want)
        k0 += size


def test_integer_codes_give_exact_products():
    rng = np.random.default_rng(44)
    k_sizes = [512, 128, 1024]
    m, n, k = 6, 10, sum(k_sizes)
    a = rng.integers(-4, 5, size=(m, k)).astype(np.float32)
    b = rng.integers(-4, 5, size=(n, k)).astype(np.float32)
    ones_a = np.ones((m, k // 128), np.float32)
    ones_b = np.ones((n, k // 128), np.float32)
    got = gemm.k_grouped_contiguous_f64(e4m3.encode_rne(a), ones_a, e4m3.encode_rne(b),
                                        ones_b, k_sizes)
    k0 = 0
    for g, size in enumerate(k_sizes):
        ai, bi = a[:, k0:k0 + size].astype(np.int64), b[:, k0:k0 + size].astype(np.int64)
        assert np.array_equal(got[g], ai @ bi.T)
        k0 += size


def test_empty_groups_return_c_and_zero_without_c():
    qa, alpha, qb, beta, _, _ = case(8, 16, [256], seed=45)
    c = inputs.rng(46).standard_normal((3, 8, 16))
    got = gemm.k_grouped_contiguous_f64(qa, alpha, qb, beta, [0, 256, 0], c)
    assert np.array_equal(got[0], c[0]) and np.array_equal(got[2], c[2])
    got0 = gemm.k_grouped_contiguous_f64(qa, alpha, qb, beta, [0, 256, 0])
    assert not got0[0].any() and not got0[2].any()
    assert close(got[1] - c[1], got0[1])


def test_sum_over_groups_is_the_product_over_all_of_k():
    lay = inputs.k_grouped_layout(700, 4, seed=47)
    qa, alpha, qb, beta, ks, _ = case(16, 24, list(lay.k_sizes), seed=48)
    got = gemm.k_grouped_contiguous_f64(qa, alpha, qb, beta, ks)
    whole = quant.dequantize_1x128(qa, alpha) @ quant.dequantize_1x128(qb, beta).T
    assert close(got.sum(axis=0), whole)


@pytest.mark.parametrize("k_sizes", [[128, 100, 156], [256, 128], [-128, 640]])
def test_rejects_segments_off_the_128_grid_or_not_summing_to_k(k_sizes):
    qa, alpha, qb, beta, _, _ = case(4, 8, [512], seed=49)
    with pytest.raises(ValueError):
        gemm.k_grouped_contiguous_f64(qa, alpha, qb, beta, k_sizes)


def test_layout_generator_pads_each_segment():
    lay = inputs.k_grouped_layout(1000, 8, seed=50)
    assert lay.counts.sum() == 1000
    assert np.all(lay.k_sizes % 128 == 0)
    assert np.all(lay.k_sizes >= lay.counts) and np.all(lay.k_sizes - lay.counts < 128)
    assert lay.k_total == lay.k_sizes.sum()


# ------------------------------------------------------------- planted mistakes
def mutant_segment_local_scales(qa, alpha, qb, beta, k_sizes, c):
    """Each segment reads the scales of the first blocks (segment-local block
    index instead of the global one)."""
    G, k0 = len(k_sizes), 0
    out = np.array(c, np.float64, copy=True)
    av, bv = e4m3.decode(qa), e4m3.decode(qb)
    for g in range(G):
        for lb in range(int(k_sizes[g]) // 128):
            ks = slice(k0 + lb * 128, k0 + (lb + 1) * 128)
            out[g] += (av[:, ks] @ bv[:, ks].T) * (alpha[:, lb][:, None] * beta[:, lb][None, :])
        k0 += int(k_sizes[g])
    return out


def mutant_dropped_c(qa, alpha, qb, beta, k_sizes, c):
    return gemm.k_grouped_contiguous_f64(qa, alpha, qb, beta, k_sizes)


def mutant_b_scale_by_block(qa, alpha, qb, beta, k_sizes, c):
    """B's scale taken per 128-row block (the dense 128x128 reading)."""
    rows = (np.arange(qb.shape[0]) // 128) * 128
    return gemm.k_grouped_contiguous_f64(qa, alpha, qb, beta[rows], k_sizes, c)


def mutant_one_segment_everywhere(qa, alpha, qb, beta, k_sizes, c):
    """Every group gets the whole-K product."""
    whole = gemm.k_grouped_contiguous_f64(qa, alpha, qb, beta, [int(sum(k_sizes))])[0]
    return np.array(c, np.float64) + whole[None]


@pytest.mark.parametrize("mutant", [mutant_segment_local_scales, mutant_dropped_c,
                                    mutant_b_scale_by_block, mutant_one_segment_everywhere])
def test_planted_mistakes_are_caught(mutant):
    qa, alpha, qb, beta, ks, c = case(40, 72, [384, 128, 0, 640], seed=51, c=True)
    want = per_segment_dequantized(qa, alpha, qb, beta, ks, c)
    assert close(gemm.k_grouped_contiguous_f64(qa, alpha, qb, beta, ks, c), want)
    assert not close(mutant(qa, alpha, qb, beta, ks, c), want)
