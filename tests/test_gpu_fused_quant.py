"""GPU parity of dg_fp8_gemm_nt_quantize, the GEMM whose epilogue quantizes
its output 1 x 128 (the FP8 cast fused into the producing kernel), through
the C ABI:

* exact integers: D is exact, so its BF16 rounding is the oracle's, and the
  codes and scales must equal the oracle quantizer applied to the oracle's
  BF16 result, bit for bit (FP32 and power-of-two scales);
* random inputs: bit for bit equal to the unfused composition -- the BF16
  GEMM in the same tile form, then dg_quantize_1x128 on its output -- and,
  dequantized, within the E4M3 rounding bound of the oracle's D;
* host checks."""

import numpy as np
import pytest
import torch

import moe_grouped_gemm_act_b200 as dg
from moe_grouped_gemm_act_b200 import inputs
from oracle import bf16, e4m3, gemm, quant

from _helpers import check_gemm, dev, env, sfa_to_device

pytestmark = pytest.mark.gpu


def run_fused(qa, alpha, qb, beta, pow2):
    dq, sfd = dg.dg_fp8_gemm_nt_quantize(dev(qa), sfa_to_device(alpha), dev(qb), dev(beta),
                                         pow2=pow2)
    torch.cuda.synchronize()
    assert dg.dg_get_device_status() == 0
    m = qa.shape[0]
    return dq.cpu().numpy(), sfd.cpu().numpy()[:, :m].T   # codes [M, N], scales [M, N/128]


@pytest.mark.parametrize("pow2", [False, True])
def test_exact_integers_match_the_oracle_bit_for_bit(pow2):
    g = np.random.default_rng(3)
    m, n, k = 200, 512, 2048
    a = g.integers(-4, 5, size=(m, k)).astype(np.float32)
    b = g.integers(-4, 5, size=(n, k)).astype(np.float32)
    qa, qb = e4m3.encode_rne(a), e4m3.encode_rne(b)
    codes, scales = run_fused(qa, np.ones((m, k // 128), np.float32), qb,
                              np.ones((n // 128, k // 128), np.float32), pow2)
    exact = (a.astype(np.int64) @ b.astype(np.int64).T).astype(np.float64)
    d32 = bf16.from_bits(bf16.to_bits(exact)).astype(np.float32)   # the BF16 result
    want_q, want_s = quant.quantize_1x128(d32, pow2=pow2)
    assert np.array_equal(codes, want_q)
    assert np.array_equal(scales, want_s)


@pytest.mark.parametrize("pow2", [False, True])
@pytest.mark.parametrize("m,n,k", [(300, 384, 1024), (129, 2176, 384), (1, 256, 256),
                                   (1024, 4096, 2048)])
def test_matches_the_unfused_composition_and_the_oracle(m, n, k, pow2):
    x = inputs.activations(m, k, seed=m + n, outliers=True)
    w = inputs.weights((n, k), seed=m + n + 1)
    qa, alpha = quant.quantize_1x128(x)
    qb, beta = quant.quantize_128x128(w)
    codes, scales = run_fused(qa, alpha, qb, beta, pow2)
    # the composition in the same tile form (256 wide, K not split)
    d = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    with env(DG_BLOCK_N=256, DG_SPLITS=1):
        dg.dg_fp8_gemm_nt(dev(qa), sfa_to_device(alpha), dev(qb), dev(beta), d)
    q2, s2 = dg.dg_quantize_1x128(d, pow2=pow2)
    torch.cuda.synchronize()
    assert np.array_equal(codes, q2.cpu().numpy())
    assert np.array_equal(scales, s2.cpu().numpy()[:, :m].T)
    # dequantized against the oracle's D: BF16 and E4M3 rounding (relative
    # 2^-9 and 2^-4), the GEMM's own bound, and half an E4M3 subnormal step
    # of each group's scale
    want = gemm.fp8_gemm_nt_f64(qa, alpha, qb, beta)
    deq = e4m3.decode(codes) * np.repeat(scales.astype(np.float64), 128, axis=1)
    rms = np.sqrt(np.mean(want ** 2))
    bound = (2.0 ** -4 + 2.0 ** -9 + 8e-3) * np.abs(want) + 2e-3 * rms + \
        np.repeat(scales.astype(np.float64), 128, axis=1) * 2.0 ** -10
    assert np.all(np.abs(deq - want) <= bound)
    # the BF16 part of the composition is itself within the GEMM bound
    check_gemm(d.view(torch.int16).cpu().numpy().view(np.uint16), want, f"{m}x{n}x{k}")


def test_host_argument_checks():
    lib = dg.load_library()
    a = torch.zeros((128, 256), dtype=torch.uint8, device="cuda")
    b = torch.zeros((200, 256), dtype=torch.uint8, device="cuda")
    sfa = torch.ones((2, 128), dtype=torch.float32, device="cuda")
    sfb = torch.ones((2, 2), dtype=torch.float32, device="cuda")
    dq = torch.empty((128, 256), dtype=torch.uint8, device="cuda")
    sfd = torch.empty((2, 128), dtype=torch.float32, device="cuda")
    P = lambda t: t.data_ptr()
    # N = 200 is not a whole number of 128-column groups
    assert lib.dg_fp8_gemm_nt_quantize(P(a), P(sfa), 128, P(b), P(sfb), P(dq), P(sfd), 128,
                                       128, 200, 256, 0, None) == dg.DG_ERR_INVALID_ARG
    # unknown flag, scale rows too short
    assert lib.dg_fp8_gemm_nt_quantize(P(a), P(sfa), 128, P(b), P(sfb), P(dq), P(sfd), 128,
                                       128, 128, 256, 4, None) == dg.DG_ERR_INVALID_ARG
    assert lib.dg_fp8_gemm_nt_quantize(P(a), P(sfa), 128, P(b), P(sfb), P(dq), P(sfd), 64,
                                       128, 128, 256, 0, None) == dg.DG_ERR_INVALID_ARG
    with pytest.raises(ValueError):
        dg.dg_fp8_gemm_nt_quantize(a, sfa, b, sfb)
