"""GPU parity of the three GEMM entry points against the oracle (through the
C ABI): shapes spanning several tiles with ragged tails, every N-tile instance,
split K, the exact-integer special case, untouched padding / masked rows,
determinism and CUDA-graph replay of the masked call."""

import numpy as np
import pytest
import torch

import moe_grouped_gemm_act_b200 as dg
from moe_grouped_gemm_act_b200 import inputs
from oracle import bf16, e4m3, gemm, quant

from _helpers import bits_of, check_gemm, dev, env, sfa_batched_to_device, sfa_to_device

pytestmark = pytest.mark.gpu

SENTINEL = 0x7FC1  # a NaN bit pattern no GEMM result can produce


def dense_case(m, n, k, seed, outliers=True):
    x = inputs.activations(m, k, seed=seed, outliers=outliers)
    w = inputs.weights((n, k), seed=seed + 1)
    qa, alpha = quant.quantize_1x128(x)
    qb, beta = quant.quantize_128x128(w)
    return qa, alpha, qb, beta


def run_dense(qa, alpha, qb, beta, workspace=False):
    m, n = qa.shape[0], qb.shape[0]
    d = torch.full((m, n), 0, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    ws = None
    if workspace:
        # room for any forced split (tiles x splits x 128 x BN FP32 + tickets)
        nbytes = max(dg.dg_fp8_gemm_nt_workspace_size(m, n, qa.shape[1]),
                     -(-m // 128) * (n + 256) * 8 * 128 * 4 + (1 << 16))
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    dg.dg_fp8_gemm_nt(dev(qa), sfa_to_device(alpha), dev(qb), dev(beta), d, workspace=ws)
    torch.cuda.synchronize()
    assert dg.dg_get_device_status() == 0
    return bits_of(d)


# ------------------------------------------------------------------ dense
def test_dense_parity_config():
    c = inputs.DENSE_PARITY
    x = inputs.activations(c["m"], c["k"], seed=c["seed_a"])
    w = inputs.weights((c["n"], c["k"]), seed=c["seed_b"])
    qa, alpha = quant.quantize_1x128(x)
    qb, beta = quant.quantize_128x128(w)
    got = run_dense(qa, alpha, qb, beta)
    check_gemm(got, gemm.fp8_gemm_nt_f64(qa, alpha, qb, beta), "128x256x512")


@pytest.mark.parametrize("bn", [16, 32, 64, 128])
@pytest.mark.parametrize("m,n,k", [(300, 392, 1024), (1, 136, 256), (129, 2112, 384)])
def test_dense_ragged_every_block_n(bn, m, n, k):
    qa, alpha, qb, beta = dense_case(m, n, k, seed=m + n + k)
    with env(DG_BLOCK_N=bn):
        got = run_dense(qa, alpha, qb, beta)
    check_gemm(got, gemm.fp8_gemm_nt_f64(qa, alpha, qb, beta), f"{m}x{n}x{k} BN={bn}")


@pytest.mark.parametrize("bn,pair", [(256, 0), (128, 0), (256, 1)])
@pytest.mark.parametrize("m,n", [(200, 400), (130, 136), (1, 520), (64, 7168), (385, 2112)])
def test_dense_stores_stay_inside_d(m, n, bn, pair):
    # D sits inside a larger buffer of sentinels: the epilogue's TMA stores
    # (boxes of 128 rows x 64 columns, clipped at D's last row and column)
    # must leave every element around it as it was, and D must be right
    k = 512
    qa, alpha, qb, beta = dense_case(m, n, k, seed=3 * m + n)
    pad = 4096  # elements on each side (keeps D 16-byte aligned)
    buf = torch.full((pad + m * n + pad,), SENTINEL, dtype=torch.int16, device="cuda")
    d = buf[pad:pad + m * n].view(m, n).view(torch.bfloat16)
    with env(DG_BLOCK_N=bn, DG_PAIR=pair, DG_SPLITS=1):
        dg.dg_fp8_gemm_nt(dev(qa), sfa_to_device(alpha), dev(qb), dev(beta), d)
        torch.cuda.synchronize()
    assert dg.dg_get_device_status() == 0
    host = buf.cpu().numpy()
    assert np.all(host[:pad] == SENTINEL) and np.all(host[pad + m * n:] == SENTINEL)
    got = host[pad:pad + m * n].reshape(m, n).view(np.uint16)
    check_gemm(got, gemm.fp8_gemm_nt_f64(qa, alpha, qb, beta), f"{m}x{n} BN={bn} pair={pair}")


@pytest.mark.parametrize("pair", [0, 1])
@pytest.mark.parametrize("m,n,k", [(300, 392, 1024), (1000, 2112, 384), (513, 256, 256),
                                   (256, 4096, 2048), (2048, 7168, 1536)])
def test_dense_pair_and_single_cta_forms(pair, m, n, k):
    # the 2-CTA form (cta_group::2, 256 x 256 tiles, each CTA loading half of
    # B) and the single-CTA form
    qa, alpha, qb, beta = dense_case(m, n, k, seed=m + 7 * n + k)
    with env(DG_PAIR=pair):
        got = run_dense(qa, alpha, qb, beta)
    check_gemm(got, gemm.fp8_gemm_nt_f64(qa, alpha, qb, beta), f"{m}x{n}x{k} pair={pair}")


def test_dense_pair_exact_integers_bit_exact_and_deterministic():
    g = np.random.default_rng(2)
    m, n, k = 640, 768, 4096
    a = g.integers(-4, 5, size=(m, k)).astype(np.float32)
    b = g.integers(-4, 5, size=(n, k)).astype(np.float32)
    qa, qb = e4m3.encode_rne(a), e4m3.encode_rne(b)
    ones_a, ones_b = np.ones((m, k // 128), np.float32), np.ones((n // 128, k // 128), np.float32)
    with env(DG_PAIR=1):
        got = run_dense(qa, ones_a, qb, ones_b)
        again = run_dense(qa, ones_a, qb, ones_b)
    exact = a.astype(np.int64) @ b.astype(np.int64).T
    assert np.array_equal(got, bf16.to_bits(exact.astype(np.float64)))
    assert np.array_equal(got, again)


def test_dense_pair_starved_wait_runs_out_and_the_next_call_is_clean():
    # the abort path of the 2-CTA form: rank 0 of the first pair leaves out
    # one stage; its MMA warp's wait runs out, rank 1's producer then runs
    # out waiting for the stage to be freed, both CTAs wait for their own
    # copies and leave; the next call is correct
    qa, alpha, qb, beta = dense_case(512, 512, 2048, seed=12)
    d = torch.zeros((512, 512), dtype=torch.bfloat16, device="cuda")
    dg.dg_get_device_status()
    with env(DG_PAIR=1, DG_TEST_STARVE_LOAD=2, DG_TEST_WAIT_LIMIT_US=20000):
        dg.dg_fp8_gemm_nt(dev(qa), sfa_to_device(alpha), dev(qb), dev(beta), d)
        torch.cuda.synchronize()
    assert dg.dg_get_device_status() == dg.DG_ERR_TIMEOUT
    with env(DG_PAIR=1):
        got = run_dense(qa, alpha, qb, beta)
    check_gemm(got, gemm.fp8_gemm_nt_f64(qa, alpha, qb, beta), "pair, after the timeout")


@pytest.mark.parametrize("splits", [2, 3, 8])
@pytest.mark.parametrize("bn", [32, 128, 256])
def test_dense_split_k(splits, bn):
    # both reductions: the splits of a tile as one cluster (distributed shared
    # memory) and through the workspace; both sum the splits in order, so
    # they must agree bit for bit
    qa, alpha, qb, beta = dense_case(64, 528, 2048, seed=splits)
    want = gemm.fp8_gemm_nt_f64(qa, alpha, qb, beta)
    with env(DG_BLOCK_N=bn, DG_SPLITS=splits, DG_CLUSTER_SPLIT=1):
        a = run_dense(qa, alpha, qb, beta, workspace=True)
        b = run_dense(qa, alpha, qb, beta, workspace=True)
    with env(DG_BLOCK_N=bn, DG_SPLITS=splits, DG_CLUSTER_SPLIT=0):
        c = run_dense(qa, alpha, qb, beta, workspace=True)
    check_gemm(a, want, f"split {splits}")
    assert np.array_equal(a, b), "split-K result not deterministic"
    assert np.array_equal(a, c), "cluster and workspace reductions differ"


@pytest.mark.parametrize("bn", [224, 192, 160, 96])
@pytest.mark.parametrize("m,n,k,splits", [(64, 2112, 2048, 4), (128, 1000, 1536, 3),
                                          (1, 736, 1024, 2), (200, 2048, 2048, 2)])
def test_cluster_split_non_power_of_two_widths(bn, m, n, k, splits):
    # tiles whose width is not a power of two (the cluster split of decode
    # shapes): a promotion thread's columns may span two 128-column blocks of
    # B's scales, each with its own beta; ragged N and M, every split summed
    # in order (deterministic)
    qa, alpha, qb, beta = dense_case(m, n, k, seed=bn + m + n)
    with env(DG_BLOCK_N=bn, DG_SPLITS=splits, DG_CLUSTER_SPLIT=1):
        a = run_dense(qa, alpha, qb, beta, workspace=True)
        b = run_dense(qa, alpha, qb, beta, workspace=True)
    check_gemm(a, gemm.fp8_gemm_nt_f64(qa, alpha, qb, beta), f"{m}x{n}x{k} BN={bn} S={splits}")
    assert np.array_equal(a, b), "cluster split not deterministic"


def test_dense_split_k_cluster_ragged_rows():
    # M = 200: two M blocks, the second with 72 valid rows; N ragged
    qa, alpha, qb, beta = dense_case(200, 776, 3072, seed=31)
    want = gemm.fp8_gemm_nt_f64(qa, alpha, qb, beta)
    with env(DG_BLOCK_N=128, DG_SPLITS=4, DG_CLUSTER_SPLIT=1):
        got = run_dense(qa, alpha, qb, beta, workspace=True)
    check_gemm(got, want, "cluster split, ragged")


@pytest.mark.parametrize("splits", [2, 3])
def test_dense_tail_split(splits):
    # 8 x 5 = 40 tiles of 128 x 256 (ragged M and N) on 12 CTAs: three whole
    # waves, then the last 4 tiles split along K over the CTAs
    qa, alpha, qb, beta = dense_case(1000, 1032, 1024, seed=20 + splits)
    want = gemm.fp8_gemm_nt_f64(qa, alpha, qb, beta)
    dg.dg_set_num_sms(12)
    try:
        with env(DG_BLOCK_N=256, DG_TAIL_SPLITS=splits):
            a = run_dense(qa, alpha, qb, beta, workspace=True)
            b = run_dense(qa, alpha, qb, beta, workspace=True)
    finally:
        dg.dg_set_num_sms(0)
    check_gemm(a, want, f"tail split {splits}")
    assert np.array_equal(a, b), "tail-split result not deterministic"


@pytest.mark.parametrize("bn", [256, 64])
def test_starved_wait_runs_out_and_the_next_call_is_clean(bn):
    # CTA 0's producer leaves out the loads of its third K block (a test hook
    # of the library): nothing completes that stage, so the MMA warp's bounded
    # wait runs out (20 ms here), the CTA aborts -- after the copies it still
    # has in flight have landed and its TMEM is freed -- and the call reports
    # DG_ERR_TIMEOUT.  The GPU stays usable: a normal call right after it is
    # correct and reports nothing.
    qa, alpha, qb, beta = dense_case(256, 512, 2048, seed=11)
    d = torch.zeros((256, 512), dtype=torch.bfloat16, device="cuda")
    dg.dg_get_device_status()
    with env(DG_TEST_STARVE_LOAD=2, DG_TEST_WAIT_LIMIT_US=20000, DG_BLOCK_N=bn):
        dg.dg_fp8_gemm_nt(dev(qa), sfa_to_device(alpha), dev(qb), dev(beta), d)
        torch.cuda.synchronize()
    assert dg.dg_get_device_status() == dg.DG_ERR_TIMEOUT
    assert dg.dg_get_device_status() == 0   # read clears
    with env(DG_BLOCK_N=bn):
        got = run_dense(qa, alpha, qb, beta)
    check_gemm(got, gemm.fp8_gemm_nt_f64(qa, alpha, qb, beta), f"after the timeout, BN={bn}")


def test_dense_exact_integers_bit_exact():
    # integer codes in [-4, 4] with unit scales: every 128-K partial and the
    # FP32 running sum are exact, so D must equal BF16(exact) bit for bit
    g = np.random.default_rng(1)
    m, n, k = 256, 384, 7168
    a = g.integers(-4, 5, size=(m, k)).astype(np.float32)
    b = g.integers(-4, 5, size=(n, k)).astype(np.float32)
    qa, qb = e4m3.encode_rne(a), e4m3.encode_rne(b)
    alpha = np.ones((m, k // 128), np.float32)
    beta = np.ones((-(-n // 128), k // 128), np.float32)
    got = run_dense(qa, alpha, qb, beta)
    exact = a.astype(np.int64) @ b.astype(np.int64).T
    assert np.array_equal(got, bf16.to_bits(exact.astype(np.float64)))


def test_dense_deterministic():
    qa, alpha, qb, beta = dense_case(512, 1024, 2048, seed=3)
    assert np.array_equal(run_dense(qa, alpha, qb, beta), run_dense(qa, alpha, qb, beta))


def test_dense_lesson13_exercise_inputs():
    # the worked exercise of Lesson 13 (integers in [-10, 10) are exact E4M3)
    np.random.seed(42)
    A = np.random.randint(-10, 10, size=(128, 256)).astype(np.float32)
    B = np.random.randint(-10, 10, size=(256, 256)).astype(np.float32)
    SA = np.random.uniform(0.01, 0.05, size=(128, 2)).astype(np.float32)
    SB = np.random.uniform(0.01, 0.05, size=(2, 2)).astype(np.float32)
    qa, qb = e4m3.encode_rne(A), e4m3.encode_rne(B)
    got = run_dense(qa, SA, qb, SB)
    check_gemm(got, gemm.fp8_gemm_nt_f64(qa, SA, qb, SB), "exercise")


@pytest.mark.parametrize("n,k", inputs.PREFILL_NK)
def test_dense_prefill_full_size_sampled_rows(n, k):
    # full bench shape, launch configuration of the bench; all columns of a
    # sampled row set (first/last row of every M tile + 2 random rows per tile)
    m = inputs.PREFILL_M
    x = inputs.activations(m, k, seed=inputs.PREFILL_SEEDS["seed_a"], outliers=True)
    w = inputs.weights((n, k), seed=inputs.PREFILL_SEEDS["seed_b"])
    qa_d, sfa_d = dg.dg_quantize_1x128(torch.from_numpy(x).cuda())
    qb_d, sfb_d = dg.dg_quantize_128x128(torch.from_numpy(w).cuda())
    d = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    # with the workspace the library asks for, as the bench runs it
    nbytes = dg.dg_fp8_gemm_nt_workspace_size(m, n, k)
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device="cuda")
    dg.dg_fp8_gemm_nt(qa_d, sfa_d, qb_d, sfb_d, d, workspace=ws)
    torch.cuda.synchronize()
    assert dg.dg_get_device_status() == 0
    g = np.random.default_rng(n + k)
    rows = []
    for t in range(m // 128):
        rows += [128 * t, 128 * t + 127, *(128 * t + g.integers(1, 127, size=2))]
    rows = np.array(sorted(set(rows)))
    qa, alpha = quant.quantize_1x128(x[rows])
    qb, beta = quant.quantize_128x128(w)
    # the device quantizers are bit-exact; check that on the sampled rows too
    assert np.array_equal(qa_d.cpu().numpy()[rows], qa)
    want = gemm.fp8_gemm_nt_f64(qa, alpha, qb, beta)
    check_gemm(bits_of(d)[rows], want, f"prefill {n}x{k}")


@pytest.mark.parametrize("m", inputs.DECODE_M)
@pytest.mark.parametrize("n,k", inputs.PREFILL_NK)
def test_dense_decode_full_size(m, n, k):
    x = inputs.activations(m, k, seed=inputs.DECODE_SEEDS["seed_a"], outliers=True)
    w = inputs.weights((n, k), seed=inputs.DECODE_SEEDS["seed_b"])
    qb_d, sfb_d = dg.dg_quantize_128x128(torch.from_numpy(w).cuda())
    qa, alpha = quant.quantize_1x128(x)
    d = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    nbytes = dg.dg_fp8_gemm_nt_workspace_size(m, n, k)
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device="cuda")
    dg.dg_fp8_gemm_nt(dev(qa), sfa_to_device(alpha), qb_d, sfb_d, d, workspace=ws)
    torch.cuda.synchronize()
    assert dg.dg_get_device_status() == 0
    qb, beta = quant.quantize_128x128(w)
    check_gemm(bits_of(d), gemm.fp8_gemm_nt_f64(qa, alpha, qb, beta), f"decode {m}x{n}x{k}")


# ------------------------------------------------------------ D = C + A B^T
def run_dense_acc(qa, alpha, qb, beta, c, workspace=False):
    m, n = qa.shape[0], qb.shape[0]
    d = torch.full((m, n), 0, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    ws = None
    if workspace:
        nbytes = max(dg.dg_fp8_gemm_nt_workspace_size(m, n, qa.shape[1]),
                     -(-m // 128) * (n + 256) * 8 * 128 * 4 + (1 << 16))
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    dg.dg_fp8_gemm_nt_accumulate(dev(qa), sfa_to_device(alpha), dev(qb), dev(beta),
                                 torch.from_numpy(c).cuda(), d, workspace=ws)
    torch.cuda.synchronize()
    assert dg.dg_get_device_status() == 0
    return bits_of(d)


def acc_c(m, n, seed):
    return (np.random.default_rng(seed).standard_normal((m, n)) * 4).astype(np.float32)


@pytest.mark.parametrize("bn", [16, 32, 64, 128, 256])
@pytest.mark.parametrize("m,n,k", [(300, 520, 1024), (1, 136, 256), (129, 2112, 384)])
def test_dense_accumulate_ragged_every_block_n(bn, m, n, k):
    qa, alpha, qb, beta = dense_case(m, n, k, seed=3 * m + n + k)
    c = acc_c(m, n, seed=m + n)
    with env(DG_BLOCK_N=bn):
        got = run_dense_acc(qa, alpha, qb, beta, c)
    want = gemm.fp8_gemm_nt_accumulate_f64(qa, alpha, qb, beta, c)
    check_gemm(got, want, f"C + AB^T {m}x{n}x{k} BN={bn}")


@pytest.mark.parametrize("mode", ["split", "tail"])
def test_dense_accumulate_split_paths(mode):
    # C is added once, by the split that stores the reduced tile
    if mode == "split":
        m, n, k, knobs = 64, 528, 2048, dict(DG_BLOCK_N=128, DG_SPLITS=4)
    else:
        m, n, k, knobs = 1000, 1032, 1024, dict(DG_BLOCK_N=256, DG_TAIL_SPLITS=3)
    qa, alpha, qb, beta = dense_case(m, n, k, seed=77)
    c = acc_c(m, n, seed=78)
    if mode == "tail":
        dg.dg_set_num_sms(12)
    try:
        with env(**knobs):
            a = run_dense_acc(qa, alpha, qb, beta, c, workspace=True)
            b = run_dense_acc(qa, alpha, qb, beta, c, workspace=True)
    finally:
        dg.dg_set_num_sms(0)
    check_gemm(a, gemm.fp8_gemm_nt_accumulate_f64(qa, alpha, qb, beta, c), f"C + AB^T {mode}")
    assert np.array_equal(a, b), "not deterministic"


def test_dense_accumulate_integers_bit_exact():
    # integer codes in [-4, 4], unit scales, integer C: D = BF16(exact)
    g = np.random.default_rng(5)
    m, n, k = 256, 384, 2048
    a = g.integers(-4, 5, size=(m, k)).astype(np.float32)
    b = g.integers(-4, 5, size=(n, k)).astype(np.float32)
    c = g.integers(-300, 301, size=(m, n)).astype(np.float32)
    got = run_dense_acc(e4m3.encode_rne(a), np.ones((m, k // 128), np.float32),
                        e4m3.encode_rne(b), np.ones((3, k // 128), np.float32), c)
    exact = a.astype(np.int64) @ b.astype(np.int64).T + c.astype(np.int64)
    assert np.array_equal(got, bf16.to_bits(exact.astype(np.float64)))


def test_dense_accumulate_zero_c_matches_plain_gemm():
    qa, alpha, qb, beta = dense_case(384, 1024, 1536, seed=9)
    plain = run_dense(qa, alpha, qb, beta)
    acc = run_dense_acc(qa, alpha, qb, beta, np.zeros((384, 1024), np.float32))
    assert np.array_equal(plain, acc)


def test_dense_accumulate_requires_c():
    qa, alpha, qb, beta = dense_case(128, 128, 128, seed=1)
    lib = dg.load_library()
    d = torch.empty((128, 128), dtype=torch.bfloat16, device="cuda")
    a_d, s_d, b_d, t_d = dev(qa), sfa_to_device(alpha), dev(qb), dev(beta)
    rc = lib.dg_fp8_gemm_nt_accumulate(a_d.data_ptr(), s_d.data_ptr(), s_d.shape[-1],
                                       b_d.data_ptr(), t_d.data_ptr(), None, d.data_ptr(),
                                       128, 128, 128, None, 0, None)
    assert rc == dg.DG_ERR_INVALID_ARG


def test_dense_m_zero_is_noop():
    d = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    a = torch.empty((0, 128), dtype=torch.uint8, device="cuda")
    sfa = torch.empty((1, 4), dtype=torch.float32, device="cuda")
    b = torch.zeros((128, 128), dtype=torch.uint8, device="cuda")
    sfb = torch.zeros((1, 1), dtype=torch.float32, device="cuda")
    dg.dg_fp8_gemm_nt(a, sfa, b, sfb, d)


def test_dense_rejects_bad_shapes():
    a = torch.zeros((128, 200), dtype=torch.uint8, device="cuda")
    sfa = torch.zeros((2, 128), dtype=torch.float32, device="cuda")
    b = torch.zeros((128, 200), dtype=torch.uint8, device="cuda")
    sfb = torch.zeros((1, 2), dtype=torch.float32, device="cuda")
    d = torch.empty((128, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(dg.DGError):
        dg.dg_fp8_gemm_nt(a, sfa, b, sfb, d)   # K % 128 != 0


def test_binding_refuses_wrong_extents_before_the_call():
    # the C ABI cannot see extents: a short D or beta, or a D of the wrong
    # dtype, is refused by the binding and nothing is launched
    a = torch.zeros((128, 256), dtype=torch.uint8, device="cuda")
    sfa = torch.ones((2, 128), dtype=torch.float32, device="cuda")
    b = torch.zeros((384, 256), dtype=torch.uint8, device="cuda")
    sfb = torch.ones((3, 2), dtype=torch.float32, device="cuda")
    for d in (torch.empty((128, 256), dtype=torch.bfloat16, device="cuda"),
              torch.empty((128, 384), dtype=torch.float32, device="cuda")):
        with pytest.raises(ValueError):
            dg.dg_fp8_gemm_nt(a, sfa, b, sfb, d)
    d = torch.empty((128, 384), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        dg.dg_fp8_gemm_nt(a, sfa, b, sfb[:2], d)
    dg.dg_fp8_gemm_nt(a, sfa, b, sfb, d)   # the right extents go through
    torch.cuda.synchronize()
    assert dg.dg_get_device_status() == 0


# ------------------------------------------------------------------ contiguous
def contiguous_case(tokens, groups, n, k, seed):
    lay = inputs.contiguous_layout(tokens, groups, seed=seed)
    x = inputs.activations(lay.m_total, k, seed=seed + 1, outliers=True)
    w = inputs.weights((groups, n, k), seed=seed + 2)
    qa, alpha = quant.quantize_1x128(x)
    qb, beta = quant.quantize_128x128_grouped(w)
    pad = lay.m_indices < 0
    qa[pad] = 0x7F            # NaN codes on padding rows: must not leak
    alpha[pad] = np.nan
    return lay, qa, alpha, qb, beta


def run_contiguous(lay, qa, alpha, qb, beta):
    m_total, n = qa.shape[0], qb.shape[1]
    d = torch.full((m_total, n), SENTINEL, dtype=torch.int16, device="cuda")
    dg.dg_m_grouped_fp8_gemm_nt_contiguous(
        dev(qa), sfa_to_device(alpha), dev(qb), dev(beta), d.view(torch.bfloat16),
        dev(lay.m_indices))
    torch.cuda.synchronize()
    assert dg.dg_get_device_status() == 0
    return bits_of(d.view(torch.bfloat16))


@pytest.mark.parametrize("bn", [16, 64, 128])
def test_contiguous_parity_and_padding_untouched(bn):
    lay, qa, alpha, qb, beta = contiguous_case(1000, 5, 264, 512, seed=60)
    with env(DG_BLOCK_N=bn):
        got = run_contiguous(lay, qa, alpha, qb, beta)
    pad = lay.m_indices < 0
    assert np.all(got[pad] == SENTINEL)
    want = gemm.m_grouped_contiguous_f64(qa, alpha, qb, beta, lay.m_indices,
                                         np.zeros(got.shape))
    check_gemm(got[~pad], want[~pad], f"contiguous BN={bn}")


def test_contiguous_empty_expert_and_padding_only_blocks():
    # expert 1 has no tokens; an extra all-padding 128-row block at the end
    lay, qa, alpha, qb, beta = contiguous_case(300, 3, 128, 256, seed=61)
    lay.m_indices[lay.m_indices == 1] = -1
    idx = np.concatenate([lay.m_indices, np.full(128, -1, np.int32)])
    qa = np.concatenate([qa, np.full((128, qa.shape[1]), 0x7F, np.uint8)])
    alpha = np.concatenate([alpha, np.full((128, alpha.shape[1]), np.nan, np.float32)])
    lay2 = inputs.ContiguousLayout(lay.counts, idx, len(idx))
    got = run_contiguous(lay2, qa, alpha, qb, beta)
    pad = idx < 0
    assert np.all(got[pad] == SENTINEL)
    want = gemm.m_grouped_contiguous_f64(qa, alpha, qb, beta, idx, np.zeros(got.shape))
    check_gemm(got[~pad], want[~pad], "contiguous sparse")


def test_contiguous_bad_index_reports_status():
    lay, qa, alpha, qb, beta = contiguous_case(256, 2, 128, 256, seed=62)
    idx = lay.m_indices.copy()
    idx[0] = 7                       # >= G
    d = torch.full((qa.shape[0], 128), SENTINEL, dtype=torch.int16, device="cuda")
    dg.dg_m_grouped_fp8_gemm_nt_contiguous(
        dev(qa), sfa_to_device(alpha), dev(qb), dev(beta), d.view(torch.bfloat16), dev(idx))
    assert dg.dg_get_device_status() == dg.DG_ERR_DEVICE_DATA
    assert dg.dg_get_device_status() == 0   # read clears


def test_contiguous_full_size_sampled_rows():
    c = inputs.CONTIGUOUS
    lay = inputs.contiguous_layout(c["tokens"], c["groups"], seed=c["seed"])
    k, n, G = c["k"], c["n"], c["groups"]
    x = inputs.activations(lay.m_total, k, seed=c["seed"] + 1, outliers=True)
    w = inputs.weights((G, n, k), seed=c["seed"] + 2)
    qa_d, sfa_d = dg.dg_quantize_1x128(torch.from_numpy(x).cuda())
    qb_d, sfb_d = dg.dg_quantize_128x128(torch.from_numpy(w).cuda())
    d = torch.full((lay.m_total, n), SENTINEL, dtype=torch.int16, device="cuda")
    dg.dg_m_grouped_fp8_gemm_nt_contiguous(qa_d, sfa_d, qb_d, sfb_d,
                                           d.view(torch.bfloat16), dev(lay.m_indices))
    torch.cuda.synchronize()
    assert dg.dg_get_device_status() == 0
    got = bits_of(d.view(torch.bfloat16))
    pad = lay.m_indices < 0
    assert np.all(got[pad] == SENTINEL)
    # every 128-row tile holding tokens: its first and last valid row and two
    # random valid rows (all columns of each)
    g = np.random.default_rng(5)
    rows = []
    for t in range(lay.m_total // 128):
        valid = np.nonzero(~pad[128 * t:128 * (t + 1)])[0] + 128 * t
        if len(valid):
            rows += [valid[0], valid[-1], *g.choice(valid, size=min(2, len(valid)),
                                                    replace=False)]
    rows = np.array(sorted(set(int(r) for r in rows)))
    assert len(rows) >= 2 * (lay.m_total // 128 - len(lay.counts))
    qa, alpha = quant.quantize_1x128(x[rows])
    for e in range(G):
        sel = rows[lay.m_indices[rows] == e]
        if len(sel) == 0:
            continue
        qb, beta = quant.quantize_128x128(w[e])
        i = np.searchsorted(rows, sel)
        want = gemm.fp8_gemm_nt_f64(qa[i], alpha[i], qb, beta)
        check_gemm(got[sel], want, f"contiguous expert {e}")


# ------------------------------------------------------------------ masked
def masked_case(G, m_max, n, k, seed, pow2=False):
    x = inputs.activations(G * m_max, k, seed=seed, outliers=True).reshape(G, m_max, k)
    w = inputs.weights((G, n, k), seed=seed + 1)
    qa, alpha = zip(*(quant.quantize_1x128(x[e], pow2=pow2) for e in range(G)))
    qa, alpha = np.stack(qa), np.stack(alpha)
    qb, beta = quant.quantize_128x128_grouped(w, pow2=pow2)
    return qa, alpha, qb, beta


def run_masked(qa, alpha, qb, beta, masked_m):
    G, m_max, _ = qa.shape
    n = qb.shape[1]
    d = torch.full((G, m_max, n), SENTINEL, dtype=torch.int16, device="cuda")
    dg.dg_m_grouped_fp8_gemm_nt_masked(dev(qa), sfa_batched_to_device(alpha), dev(qb),
                                       dev(beta), d.view(torch.bfloat16),
                                       dev(np.asarray(masked_m, np.int32)))
    torch.cuda.synchronize()
    return bits_of(d.view(torch.bfloat16))


def check_masked(got, qa, alpha, qb, beta, masked_m, what):
    for e in range(qa.shape[0]):
        m = int(min(max(masked_m[e], 0), qa.shape[1]))
        assert np.all(got[e, m:] == SENTINEL), f"{what}: rows >= masked_m written"
        if m:
            check_gemm(got[e, :m], gemm.fp8_gemm_nt_f64(qa[e, :m], alpha[e, :m], qb[e], beta[e]),
                       f"{what} expert {e}")


@pytest.mark.parametrize("bn", [16, 128])
def test_masked_parity_and_rows_untouched(bn):
    qa, alpha, qb, beta = masked_case(5, 300, 264, 512, seed=70)
    masked_m = [0, 300, 129, 1, 128]
    with env(DG_BLOCK_N=bn):
        got = run_masked(qa, alpha, qb, beta, masked_m)
    assert dg.dg_get_device_status() == 0
    check_masked(got, qa, alpha, qb, beta, masked_m, f"masked BN={bn}")


def test_masked_pow2_scales():
    qa, alpha, qb, beta = masked_case(4, 256, 512, 1024, seed=71, pow2=True)
    masked_m = [256, 17, 0, 200]
    got = run_masked(qa, alpha, qb, beta, masked_m)
    check_masked(got, qa, alpha, qb, beta, masked_m, "masked pow2")


def test_masked_out_of_range_counts_clamped_and_reported():
    qa, alpha, qb, beta = masked_case(3, 128, 128, 256, seed=72)
    masked_m = [-3, 500, 64]
    got = run_masked(qa, alpha, qb, beta, masked_m)
    assert dg.dg_get_device_status() == dg.DG_ERR_DEVICE_DATA
    check_masked(got, qa, alpha, qb, beta, masked_m, "masked clamp")


def test_masked_cuda_graph_replay():
    G, m_max, n, k = 6, 256, 384, 1024
    qa, alpha, qb, beta = masked_case(G, m_max, n, k, seed=73)
    a, sfa, b, sfb = dev(qa), sfa_batched_to_device(alpha), dev(qb), dev(beta)
    mm = torch.zeros(G, dtype=torch.int32, device="cuda")
    d = torch.full((G, m_max, n), SENTINEL, dtype=torch.int16, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        dg.dg_m_grouped_fp8_gemm_nt_masked(a, sfa, b, sfb, d.view(torch.bfloat16), mm)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        dg.dg_m_grouped_fp8_gemm_nt_masked(a, sfa, b, sfb, d.view(torch.bfloat16), mm)
    rng = np.random.default_rng(3)
    for _ in range(3):
        counts = rng.integers(0, m_max + 1, size=G).astype(np.int32)
        mm.copy_(torch.from_numpy(counts))
        d.fill_(SENTINEL)
        graph.replay()
        torch.cuda.synchronize()
        got = bits_of(d.view(torch.bfloat16))
        check_masked(got, qa, alpha, qb, beta, counts, "graph replay")
    assert dg.dg_get_device_status() == 0


@pytest.mark.parametrize("pow2", [False, True])
def test_masked_full_size(pow2):
    # the full masked workload (32 experts, M_max 256, N 7168, K 2048) in the
    # bench's launch configuration, every expert's valid rows against the
    # oracle; pow2: every scale rounded up to a power of two (the
    # UE8M0-representable variant of the workload)
    c = inputs.MASKED
    G, m_max, n, k = c["groups"], c["m_max"], c["n"], c["k"]
    masked_m = inputs.masked_counts(G, m_max, seed=c["seed"])
    x = inputs.activations(G * m_max, k, seed=c["seed"] + 1, outliers=True).reshape(G, m_max, k)
    w = inputs.weights((G, n, k), seed=c["seed"] + 2)
    qa_d, sfa_d = dg.dg_quantize_1x128(torch.from_numpy(x).cuda(), pow2=pow2)
    qb_d, sfb_d = dg.dg_quantize_128x128(torch.from_numpy(w).cuda(), pow2=pow2)
    d = torch.full((G, m_max, n), SENTINEL, dtype=torch.int16, device="cuda")
    dg.dg_m_grouped_fp8_gemm_nt_masked(qa_d, sfa_d, qb_d, sfb_d, d.view(torch.bfloat16),
                                       dev(masked_m))
    torch.cuda.synchronize()
    assert dg.dg_get_device_status() == 0
    got = bits_of(d.view(torch.bfloat16))
    qb_all = qb_d.cpu().numpy()
    for e in range(G):
        assert np.all(got[e, masked_m[e]:] == SENTINEL)
        m = int(masked_m[e])
        if not m:
            continue
        qa, alpha = quant.quantize_1x128(x[e, :m], pow2=pow2)
        qb, beta = quant.quantize_128x128(w[e], pow2=pow2)
        # the device quantizers agree with the oracle's bit for bit
        assert np.array_equal(qa_d[e, :m].cpu().numpy(), qa)
        assert np.array_equal(qb_all[e], qb)
        check_gemm(got[e, :m], gemm.fp8_gemm_nt_f64(qa, alpha, qb, beta),
                   f"masked{' pow2' if pow2 else ''} e{e}")
