"""GPU parity of the NN, TN and TT dense GEMMs and of the TN k-grouped GEMM
(operands stored with K outermost, loaded as MN-major tiles) against the
oracle's layout forms, through the C ABI: ragged shapes over several tiles
for both tile widths, exact integers bit for bit, the split-K paths (cluster
and workspace reductions, the tail split), and the host's alignment checks.

Inputs are quantized by the oracle in their logical [M, K] / [N, K] views and
then stored transposed where the layout says so; the scales keep their
logical layouts."""

import numpy as np
import pytest
import torch

import moe_grouped_gemm_act_b200 as dg
from moe_grouped_gemm_act_b200 import inputs
from oracle import bf16, e4m3, gemm, quant

from _helpers import bits_of, check_f32, check_gemm, dev, env, sfa_to_device

pytestmark = pytest.mark.gpu

CALLS = {"nn": dg.dg_fp8_gemm_nn, "tn": dg.dg_fp8_gemm_tn, "tt": dg.dg_fp8_gemm_tt,
         "nt": dg.dg_fp8_gemm_nt}


def stored(layout, qa, qb):
    """The operands as the layout stores them."""
    a = qa.T if layout[0] == "t" else qa
    b = qb if layout[1] == "t" else qb.T
    return np.ascontiguousarray(a), np.ascontiguousarray(b)


def run(layout, qa, alpha, qb, beta, workspace=False):
    m, n = qa.shape[0], qb.shape[0]
    a_s, b_s = stored(layout, qa, qb)
    d = torch.zeros((m, n), dtype=torch.bfloat16, device="cuda")
    ws = None
    if workspace:
        nbytes = max(dg.dg_fp8_gemm_nt_workspace_size(m, n, qa.shape[1]),
                     -(-m // 128) * (n + 256) * 8 * 128 * 4 + (1 << 16))
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    CALLS[layout](dev(a_s), sfa_to_device(alpha), dev(b_s), dev(beta), d, workspace=ws)
    torch.cuda.synchronize()
    assert dg.dg_get_device_status() == 0
    return bits_of(d), a_s, b_s


def case(m, n, k, seed):
    x = inputs.activations(m, k, seed=seed, outliers=True)
    w = inputs.weights((n, k), seed=seed + 1)
    qa, alpha = quant.quantize_1x128(x)
    qb, beta = quant.quantize_128x128(w)
    return qa, alpha, qb, beta


@pytest.mark.parametrize("layout", ["nn", "tn", "tt"])
@pytest.mark.parametrize("m,n,k,bn", [(304, 400, 1024, 256), (304, 400, 1024, 128),
                                      (16, 144, 256, 128), (1024, 2112, 1536, 256),
                                      (528, 1040, 2048, 128)])
def test_layout_parity(layout, m, n, k, bn):
    qa, alpha, qb, beta = case(m, n, k, seed=m + n + k)
    with env(DG_BLOCK_N=bn):
        got, a_s, b_s = run(layout, qa, alpha, qb, beta)
    # the oracle's layout form, on the operands exactly as stored
    want = gemm.fp8_gemm_f64(layout, a_s, alpha, b_s, beta)
    check_gemm(got, want, f"{layout} {m}x{n}x{k} BN={bn}")


@pytest.mark.parametrize("layout", ["nn", "tn", "tt"])
def test_layout_exact_integers_bit_exact(layout):
    g = np.random.default_rng(7)
    m, n, k = 256, 384, 2048
    a = g.integers(-4, 5, size=(m, k)).astype(np.float32)
    b = g.integers(-4, 5, size=(n, k)).astype(np.float32)
    got, _, _ = run(layout, e4m3.encode_rne(a), np.ones((m, k // 128), np.float32),
                    e4m3.encode_rne(b), np.ones((3, k // 128), np.float32))
    exact = a.astype(np.int64) @ b.astype(np.int64).T
    assert np.array_equal(got, bf16.to_bits(exact.astype(np.float64)))


@pytest.mark.parametrize("layout", ["nn", "tn", "tt"])
@pytest.mark.parametrize("cluster", [0, 1])
def test_layout_split_k(layout, cluster):
    # decode-sized shape, every tile split 4 ways, both reductions; they sum
    # the splits in the same order, so agree bit for bit
    qa, alpha, qb, beta = case(64, 528, 2048, seed=40)
    with env(DG_BLOCK_N=128, DG_SPLITS=4, DG_CLUSTER_SPLIT=cluster):
        got, a_s, b_s = run(layout, qa, alpha, qb, beta, workspace=True)
    check_gemm(got, gemm.fp8_gemm_f64(layout, a_s, alpha, b_s, beta), f"{layout} split")


@pytest.mark.parametrize("layout", ["nn", "tn", "tt"])
def test_layout_tail_split(layout):
    qa, alpha, qb, beta = case(1008, 1040, 1024, seed=41)
    dg.dg_set_num_sms(12)
    try:
        with env(DG_BLOCK_N=256, DG_TAIL_SPLITS=3):
            got, a_s, b_s = run(layout, qa, alpha, qb, beta, workspace=True)
    finally:
        dg.dg_set_num_sms(0)
    check_gemm(got, gemm.fp8_gemm_f64(layout, a_s, alpha, b_s, beta), f"{layout} tail split")


def test_layouts_reject_unaligned_mn_major_operands():
    lib = dg.load_library()
    a = torch.zeros((256, 136), dtype=torch.uint8, device="cuda")
    b = torch.zeros((256, 136), dtype=torch.uint8, device="cuda")
    sfa = torch.ones((2, 136), dtype=torch.float32, device="cuda")
    sfb = torch.ones((2, 2), dtype=torch.float32, device="cuda")
    d = torch.empty((136, 136), dtype=torch.bfloat16, device="cuda")
    P = lambda t: t.data_ptr()
    # M = 136 is not a multiple of 16 for a [K][M] A; N = 136 for a [K][N] B
    for name in ("dg_fp8_gemm_tn", "dg_fp8_gemm_tt", "dg_fp8_gemm_nn"):
        rc = getattr(lib, name)(P(a), P(sfa), 136, P(b), P(sfb), P(d), 136, 136, 256, None, 0,
                                None)
        assert rc == dg.DG_ERR_ALIGNMENT, name


def test_k_grouped_tn_matches_the_oracle():
    # the weight-gradient layout: tokens (K) outermost for both operands,
    # ragged groups including empty ones, with C
    k_sizes = [0, 384, 128, 0, 640]
    m, n = 208, 272
    k_total = int(sum(k_sizes))
    a = inputs.activations(m, k_total, seed=90, outliers=True)
    b = inputs.activations(n, k_total, seed=91)
    qa, alpha = quant.quantize_1x128(a)
    qb, beta = quant.quantize_1x128(b)
    c = (inputs.rng(92).standard_normal((len(k_sizes), m, n)) * 4).astype(np.float32)
    ks = np.asarray(k_sizes, np.int32)
    want = gemm.k_grouped_contiguous_f64(qa, alpha, qb, beta, ks, c)
    for bn in (256, 128):
        d = torch.full((len(k_sizes), m, n), float("nan"), dtype=torch.float32, device="cuda")
        with env(DG_BLOCK_N=bn):
            dg.dg_k_grouped_fp8_gemm_tn_contiguous(
                dev(np.ascontiguousarray(qa.T)), sfa_to_device(alpha),
                dev(np.ascontiguousarray(qb.T)), sfa_to_device(beta), d, dev(ks), c=dev(c))
            torch.cuda.synchronize()
        assert dg.dg_get_device_status() == 0
        got = d.cpu().numpy()
        for g, size in enumerate(k_sizes):
            if size == 0:
                assert np.array_equal(got[g], c[g])
            else:
                check_f32(got[g], want[g], f"k-grouped TN BN={bn} group {g}")
