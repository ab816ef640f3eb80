"""GPU parity of the UE8M0 GEMMs (power-of-two scales as packed UE8M0 words,
applied by the tensor cores' block-scaled MMA) against the oracle, through
the C ABI: exact integers bit for bit (also with non-unit power-of-two
scales), power-of-two-quantized inputs on ragged shapes, agreement with the
FP32-scale promotion path, the masked layout (rows >= masked_m untouched, the
full-size workload), determinism, the B-scale packer bit for bit, the
starved-wait abort path and the host argument checks."""

import numpy as np
import pytest
import torch

import moe_grouped_gemm_act_b200 as dg
from moe_grouped_gemm_act_b200 import inputs
from oracle import bf16, e4m3, gemm, quant, ue8m0

from _helpers import bits_of, check_gemm, dev, env, sfa_to_device

pytestmark = pytest.mark.gpu

SENTINEL = 0x7FC1


def packed(sf_rows: np.ndarray, ld: int | None = None) -> torch.Tensor:
    """Oracle packing of per-row scales [R, Kg] to a device tensor
    [ceil(Kg/4), ld]."""
    words = ue8m0.pack_1x128(sf_rows.astype(np.float32))
    ld = ld or -(-words.shape[1] // 4) * 4
    out = np.zeros((words.shape[0], ld), np.int32)
    out[:, :words.shape[1]] = words
    return dev(out)


def block_rows(beta: np.ndarray, n: int) -> np.ndarray:
    """128 x 128 block scales written out per row of B."""
    return beta[np.arange(n) // 128]


def run_ue(qa, sfa_words, qb, sfb_words):
    m, n = qa.shape[0], qb.shape[0]
    d = torch.full((m, n), SENTINEL, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    dg.dg_fp8_gemm_nt_ue8m0(dev(qa), sfa_words, dev(qb), sfb_words, d)
    torch.cuda.synchronize()
    assert dg.dg_get_device_status() == 0
    return bits_of(d)


def test_exact_integers_bit_exact_unit_scales():
    # integer codes in [-4, 4] with scale 1 (code 127): every product, every
    # 32-wide slice and the FP32 sum over K = 7168 are exact
    g = np.random.default_rng(1)
    m, n, k = 256, 384, 7168
    a = g.integers(-4, 5, size=(m, k)).astype(np.float32)
    b = g.integers(-4, 5, size=(n, k)).astype(np.float32)
    got = run_ue(e4m3.encode_rne(a), packed(np.ones((m, k // 128))), e4m3.encode_rne(b),
                 packed(np.ones((n, k // 128))))
    exact = a.astype(np.int64) @ b.astype(np.int64).T
    assert np.array_equal(got, bf16.to_bits(exact.astype(np.float64)))


def test_exact_integers_bit_exact_power_of_two_scales():
    # per-row and per-group powers of two on both operands, still exact:
    # checks that each K group's scale bytes reach the right rows and slices
    g = np.random.default_rng(2)
    m, n, k = 200, 264, 1024
    kg = k // 128
    a = g.integers(-4, 5, size=(m, k)).astype(np.float32)
    b = g.integers(-4, 5, size=(n, k)).astype(np.float32)
    # scales in {1/2, 1, 2}: every running sum stays a multiple of 1/4 far
    # below 2^12, exact in any accumulator of 14 or more bits
    alpha = np.ldexp(1.0, g.integers(-1, 2, size=(m, kg)))
    beta = np.ldexp(1.0, g.integers(-1, 2, size=(n, kg)))   # distinct per row of B
    got = run_ue(e4m3.encode_rne(a), packed(alpha), e4m3.encode_rne(b), packed(beta))
    want = gemm.fp8_gemm_nt_rowscaled_f64(e4m3.encode_rne(a), alpha, e4m3.encode_rne(b), beta)
    assert np.array_equal(got, bf16.to_bits(want))


@pytest.mark.parametrize("m,n,k", [(300, 392, 1024), (129, 2112, 384), (1, 136, 256),
                                   (512, 1024, 2048)])
def test_pow2_quantized_inputs_match_the_oracle(m, n, k):
    x = inputs.activations(m, k, seed=m + n, outliers=True)
    w = inputs.weights((n, k), seed=m + n + 1)
    qa, alpha = quant.quantize_1x128(x, pow2=True)
    qb, beta = quant.quantize_128x128(w, pow2=True)
    sfa_w = ue8m0.pack_1x128(alpha)
    sfb_w = ue8m0.pack_1x128(block_rows(beta, n))
    # the device quantizers and packers give the oracle's bits
    qa_d, sfa_d = dg.dg_quantize_1x128(torch.from_numpy(x).cuda(), pow2=True)
    qb_d, sfb_d = dg.dg_quantize_128x128(torch.from_numpy(w).cuda(), pow2=True)
    pa = dg.dg_pack_ue8m0(sfa_d, m)
    pb = dg.dg_pack_ue8m0_128x128(sfb_d, n)
    torch.cuda.synchronize()
    assert dg.dg_get_device_status() == 0
    assert np.array_equal(pa.cpu().numpy()[:, :m], sfa_w)
    assert np.array_equal(pb.cpu().numpy()[:, :n], sfb_w)
    assert np.array_equal(qa_d.cpu().numpy(), qa)
    d = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    dg.dg_fp8_gemm_nt_ue8m0(qa_d, pa, qb_d, pb, d)
    torch.cuda.synchronize()
    assert dg.dg_get_device_status() == 0
    want = gemm.fp8_gemm_nt_ue8m0_f64(qa, sfa_w, qb, sfb_w)
    check_gemm(bits_of(d), want, f"UE8M0 {m}x{n}x{k}")
    # the FP32-scale promotion path on the same power-of-two scales
    d2 = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    dg.dg_fp8_gemm_nt(qa_d, sfa_d, qb_d, sfb_d, d2)
    torch.cuda.synchronize()
    check_gemm(bits_of(d2), want, f"promotion on the pow2 scales {m}x{n}x{k}")
    # and the same call again gives the same bits
    d3 = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    dg.dg_fp8_gemm_nt_ue8m0(qa_d, pa, qb_d, pb, d3)
    torch.cuda.synchronize()
    assert torch.equal(d.view(torch.int16), d3.view(torch.int16))


@pytest.mark.parametrize("m,n", [(200, 392), (1, 520), (130, 2112)])
def test_stores_stay_inside_d(m, n):
    # D sits inside a buffer of sentinels: the epilogue's TMA stores (boxes of
    # 128 rows x 64 columns, one per 64-column phase, clipped at D's last row
    # and column) leave every element around it as it was
    k = 512
    x = inputs.activations(m, k, seed=5 * m + n, outliers=True)
    w = inputs.weights((n, k), seed=5 * m + n + 1)
    qa_d, sfa_d = dg.dg_quantize_1x128(torch.from_numpy(x).cuda(), pow2=True)
    qb_d, sfb_d = dg.dg_quantize_128x128(torch.from_numpy(w).cuda(), pow2=True)
    pa = dg.dg_pack_ue8m0(sfa_d, m)
    pb = dg.dg_pack_ue8m0_128x128(sfb_d, n)
    pad = 4096  # elements on each side (keeps D 16-byte aligned)
    buf = torch.full((pad + m * n + pad,), SENTINEL, dtype=torch.int16, device="cuda")
    d = buf[pad:pad + m * n].view(m, n).view(torch.bfloat16)
    dg.dg_fp8_gemm_nt_ue8m0(qa_d, pa, qb_d, pb, d)
    torch.cuda.synchronize()
    assert dg.dg_get_device_status() == 0
    host = buf.cpu().numpy()
    assert np.all(host[:pad] == SENTINEL) and np.all(host[pad + m * n:] == SENTINEL)
    qa, alpha = quant.quantize_1x128(x, pow2=True)
    qb, beta = quant.quantize_128x128(w, pow2=True)
    want = gemm.fp8_gemm_nt_ue8m0_f64(qa, ue8m0.pack_1x128(alpha), qb,
                                      ue8m0.pack_1x128(block_rows(beta, n)))
    check_gemm(host[pad:pad + m * n].reshape(m, n).view(np.uint16), want, f"UE8M0 {m}x{n}")


def test_pack_128x128_grouped_bit_exact_and_rejects_non_powers_of_two():
    rng = np.random.default_rng(4)
    G, n, kg = 3, 300, 9
    beta = np.ldexp(1.0, rng.integers(-30, 30, size=(G, -(-n // 128), kg))).astype(np.float32)
    beta[0, 1, 2] = 0.0
    got = dg.dg_pack_ue8m0_128x128(dev(beta), n)
    torch.cuda.synchronize()
    assert dg.dg_get_device_status() == 0
    for g in range(G):
        want = ue8m0.pack_1x128(block_rows(beta[g], n))
        assert np.array_equal(got[g].cpu().numpy()[:, :n], want)
    bad = beta.copy()
    bad[1, 0, 0] = 3.0
    dg.dg_pack_ue8m0_128x128(dev(bad), n)
    assert dg.dg_get_device_status() == dg.DG_ERR_DEVICE_DATA


def masked_ue_case(G, m_max, n, k, seed):
    x = inputs.activations(G * m_max, k, seed=seed, outliers=True).reshape(G, m_max, k)
    w = inputs.weights((G, n, k), seed=seed + 1)
    return x, w


def run_masked_ue(x, w, masked_m):
    G, m_max, k = x.shape
    n = w.shape[1]
    qa_d, sfa_d = dg.dg_quantize_1x128(torch.from_numpy(x).cuda(), pow2=True)
    qb_d, sfb_d = dg.dg_quantize_128x128(torch.from_numpy(w).cuda(), pow2=True)
    pa = dg.dg_pack_ue8m0(sfa_d, m_max)
    pb = dg.dg_pack_ue8m0_128x128(sfb_d, n)
    d = torch.full((G, m_max, n), SENTINEL, dtype=torch.int16, device="cuda")
    dg.dg_m_grouped_fp8_gemm_nt_masked_ue8m0(qa_d, pa, qb_d, pb, d.view(torch.bfloat16),
                                             dev(np.asarray(masked_m, np.int32)))
    torch.cuda.synchronize()
    return bits_of(d.view(torch.bfloat16))


def check_masked_ue(got, x, w, masked_m, what):
    G, m_max, _ = x.shape
    n = w.shape[1]
    for e in range(G):
        m = int(min(max(int(masked_m[e]), 0), m_max))
        assert np.all(got[e, m:] == SENTINEL), f"{what}: rows >= masked_m written"
        if m:
            qa, alpha = quant.quantize_1x128(x[e, :m], pow2=True)
            qb, beta = quant.quantize_128x128(w[e], pow2=True)
            want = gemm.fp8_gemm_nt_ue8m0_f64(qa, ue8m0.pack_1x128(alpha), qb,
                                              ue8m0.pack_1x128(block_rows(beta, n)))
            check_gemm(got[e, :m], want, f"{what} expert {e}")


def test_masked_ue8m0_ragged_and_rows_untouched():
    x, w = masked_ue_case(5, 300, 264, 512, seed=80)
    masked_m = [0, 300, 129, 1, 128]
    got = run_masked_ue(x, w, masked_m)
    assert dg.dg_get_device_status() == 0
    check_masked_ue(got, x, w, masked_m, "masked UE8M0")


def test_masked_ue8m0_out_of_range_counts_clamped_and_reported():
    x, w = masked_ue_case(3, 128, 128, 256, seed=81)
    masked_m = [-3, 500, 64]
    got = run_masked_ue(x, w, masked_m)
    assert dg.dg_get_device_status() == dg.DG_ERR_DEVICE_DATA
    check_masked_ue(got, x, w, masked_m, "masked UE8M0 clamp")


def test_masked_ue8m0_full_size():
    # the masked workload's power-of-two variant at full size (32 experts,
    # M_max 256, N 7168, K 2048), every expert against the oracle
    c = inputs.MASKED
    G, m_max, n, k = c["groups"], c["m_max"], c["n"], c["k"]
    masked_m = inputs.masked_counts(G, m_max, seed=c["seed"])
    x = inputs.activations(G * m_max, k, seed=c["seed"] + 1, outliers=True).reshape(G, m_max, k)
    w = inputs.weights((G, n, k), seed=c["seed"] + 2)
    got = run_masked_ue(x, w, masked_m)
    assert dg.dg_get_device_status() == 0
    check_masked_ue(got, x, w, masked_m, "masked UE8M0 full size")


def test_starved_wait_runs_out_on_the_ue8m0_path():
    # the abort path with the scale-factor copies in the stages: CTA 0's
    # producer leaves out one stage (operands and scale words); the wait runs
    # out, the call reports DG_ERR_TIMEOUT and the next call is correct
    g = np.random.default_rng(3)
    m, n, k = 256, 512, 2048
    a = g.integers(-4, 5, size=(m, k)).astype(np.float32)
    b = g.integers(-4, 5, size=(n, k)).astype(np.float32)
    qa, qb = e4m3.encode_rne(a), e4m3.encode_rne(b)
    pa, pb = packed(np.ones((m, k // 128))), packed(np.ones((n, k // 128)))
    d = torch.zeros((m, n), dtype=torch.bfloat16, device="cuda")
    dg.dg_get_device_status()
    with env(DG_TEST_STARVE_LOAD=2, DG_TEST_WAIT_LIMIT_US=20000):
        dg.dg_fp8_gemm_nt_ue8m0(dev(qa), pa, dev(qb), pb, d)
        torch.cuda.synchronize()
    assert dg.dg_get_device_status() == dg.DG_ERR_TIMEOUT
    got = run_ue(qa, pa, qb, pb)
    exact = a.astype(np.int64) @ b.astype(np.int64).T
    assert np.array_equal(got, bf16.to_bits(exact.astype(np.float64)))


def test_host_argument_checks():
    lib = dg.load_library()
    a = torch.zeros((128, 256), dtype=torch.uint8, device="cuda")
    b = torch.zeros((128, 256), dtype=torch.uint8, device="cuda")
    sf = torch.zeros((1, 128), dtype=torch.int32, device="cuda")
    d = torch.empty((128, 128), dtype=torch.bfloat16, device="cuda")
    P = lambda t: t.data_ptr()
    # ld of the scale words below M / N, not a multiple of 4, K off the grid
    assert lib.dg_fp8_gemm_nt_ue8m0(P(a), P(sf), 64, P(b), P(sf), 128, P(d), 128, 128, 256,
                                    None) == dg.DG_ERR_INVALID_ARG
    assert lib.dg_fp8_gemm_nt_ue8m0(P(a), P(sf), 130, P(b), P(sf), 128, P(d), 128, 128, 256,
                                    None) == dg.DG_ERR_ALIGNMENT
    assert lib.dg_fp8_gemm_nt_ue8m0(P(a), P(sf), 128, P(b), P(sf), 128, P(d), 128, 128, 200,
                                    None) == dg.DG_ERR_INVALID_ARG
    with pytest.raises(ValueError):   # the binding sees the short word rows
        dg.dg_fp8_gemm_nt_ue8m0(a, sf[:, :64], b, sf, d)
