"""GPU parity of the quantizer kernels against the oracle: bit-exact codes and
bit-exact scales (FP32 and power-of-two modes), through the C ABI."""

import numpy as np
import pytest
import torch

import moe_grouped_gemm_act_b200 as dg
from moe_grouped_gemm_act_b200 import inputs
from oracle import quant

pytestmark = pytest.mark.gpu


def run_1x128(x_np, pow2=False, dtype=torch.float32):
    x = torch.from_numpy(x_np).to(dtype).cuda()
    q, sf = dg.dg_quantize_1x128(x, pow2=pow2)
    torch.cuda.synchronize()
    m = x_np.shape[-2]
    return q.cpu().numpy(), sf.cpu().numpy()[..., :m]


def edge_case_rows(k=512):
    """Rows exercising the corner cases of the rounding."""
    from oracle import e4m3
    rows = []
    rows.append(np.zeros(k, np.float32))                          # all zero
    r = np.zeros(k, np.float32); r[3] = -0.0; r[200] = 5.0; rows.append(r)
    r = np.full(k, 1e-3, np.float32); r[::7] = -1e-9; r[1] = 448.0; rows.append(r)  # -0 codes
    # exact E4M3 midpoints after scaling by alpha = 1 (amax 448)
    pos = e4m3.DECODE[:0x7F]
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    r = np.zeros(k, np.float32); r[:len(mids)] = mids[:k]; r[k - 1] = 448.0; rows.append(r)
    r = -r; rows.append(r)
    r = np.full(k, 3e-39, np.float32); r[0] = 1e-38; rows.append(r)  # subnormal scales
    r = np.ones(k, np.float32) * 7.0; r[5] = 3.0e38; rows.append(r)   # huge outlier
    g = np.random.default_rng(0)
    rows.append((g.standard_normal(k) * 1e-30).astype(np.float32))
    return np.stack(rows)


@pytest.mark.parametrize("pow2", [False, True])
def test_1x128_edge_cases_bit_exact(pow2):
    x = edge_case_rows()
    q, sf = run_1x128(x, pow2)
    q0, a0 = quant.quantize_1x128(x, pow2=pow2)
    assert np.array_equal(q, q0)
    assert np.array_equal(sf.T.view(np.uint32), a0.view(np.uint32))


def near_midpoint_rows(rows=64, k=1024, seed=0):
    """Groups whose quotients x / alpha sit within a few float32 ulps of E4M3
    rounding midpoints, for scales that are not powers of two: these decide
    whether the device quotient is the correctly rounded one."""
    from oracle import e4m3
    g = np.random.default_rng(seed)
    pos = e4m3.DECODE[:0x7F]
    mids = ((pos[:-1] + pos[1:]) / 2)
    out = np.zeros((rows, k), np.float32)
    for r in range(rows):
        for grp in range(k // 128):
            amax = np.float32(g.uniform(0.5, 2.0) * 10.0 ** g.integers(-20, 20))
            s = amax / np.float32(448.0)                    # float32 division, RN
            m = g.choice(mids, size=127) * g.choice([-1, 1], size=127)
            x = (m * np.float64(s)).astype(np.float32)       # near m * s
            x = np.nextafter(x, np.float32(np.inf) * np.sign(x),
                             dtype=np.float32) if r % 3 == 1 else x
            x = np.nextafter(x, np.float32(0), dtype=np.float32) if r % 3 == 2 else x
            x = np.clip(x, -amax, amax)
            out[r, grp * 128] = amax
            out[r, grp * 128 + 1:(grp + 1) * 128] = x
    return out


@pytest.mark.parametrize("pow2", [False, True])
def test_1x128_near_midpoints_bit_exact(pow2):
    x = near_midpoint_rows()
    q, sf = run_1x128(x, pow2)
    q0, a0 = quant.quantize_1x128(x, pow2=pow2)
    assert np.array_equal(sf.T.view(np.uint32), a0.view(np.uint32))
    assert np.array_equal(q, q0)


def test_1x128_wide_dynamic_range_bit_exact():
    x = inputs.activations(512, 1024, seed=21, outliers=True)
    g = np.random.default_rng(4)
    x *= (10.0 ** g.uniform(-38, 36, size=(512, 1))).astype(np.float32)
    x[5, :128] *= np.float32(1e-10)              # subnormal inputs and scales
    q, sf = run_1x128(x)
    q0, a0 = quant.quantize_1x128(x)
    assert np.array_equal(sf.T.view(np.uint32), a0.view(np.uint32))
    assert np.array_equal(q, q0)


@pytest.mark.parametrize("m,k", [(1, 128), (3, 384), (128, 512), (300, 1024), (1000, 7168)])
@pytest.mark.parametrize("pow2", [False, True])
def test_1x128_random_bit_exact(m, k, pow2):
    x = inputs.activations(m, k, seed=100 + m, outliers=True)
    q, sf = run_1x128(x, pow2)
    q0, a0 = quant.quantize_1x128(x, pow2=pow2)
    assert np.array_equal(q, q0)
    assert np.array_equal(sf.T.view(np.uint32), a0.view(np.uint32))


def test_1x128_bf16_input_bit_exact():
    x = inputs.activations(257, 1024, seed=5, outliers=True)
    xb = torch.from_numpy(x).to(torch.bfloat16)
    q, sf = run_1x128(x, dtype=torch.bfloat16)
    q0, a0 = quant.quantize_1x128(xb.float().numpy())
    assert np.array_equal(q, q0)
    assert np.array_equal(sf.T.view(np.uint32), a0.view(np.uint32))


def test_1x128_batched_layout():
    G, M, K = 3, 70, 256
    x = inputs.activations(G * M, K, seed=9, outliers=True).reshape(G, M, K)
    q, sf = run_1x128(x)
    for g in range(G):
        q0, a0 = quant.quantize_1x128(x[g])
        assert np.array_equal(q[g], q0)
        assert np.array_equal(sf[g].T, a0)


def test_1x128_full_prefill_rows_sampled():
    # the bench's activation shape, M=4096 K=16384; every row checked on a
    # deterministic sample of 64 rows spread over the matrix
    M, K = 4096, 16384
    x = inputs.activations(M, K, seed=2, outliers=True)
    q, sf = run_1x128(x)
    rows = np.linspace(0, M - 1, 64).astype(int)
    q0, a0 = quant.quantize_1x128(x[rows])
    assert np.array_equal(q[rows], q0)
    assert np.array_equal(sf[:, rows].T, a0)


@pytest.mark.parametrize("n,k,pow2", [(256, 512, False), (130, 384, False),
                                      (2112, 1024, True), (7, 128, False)])
def test_128x128_bit_exact(n, k, pow2):
    w = inputs.weights((n, k), seed=n + k)
    q, sf = dg.dg_quantize_128x128(torch.from_numpy(w).cuda(), pow2=pow2)
    q0, b0 = quant.quantize_128x128(w, pow2=pow2)
    assert np.array_equal(q.cpu().numpy(), q0)
    assert np.array_equal(sf.cpu().numpy().view(np.uint32), b0.view(np.uint32))


def test_128x128_grouped_bit_exact():
    w = inputs.weights((3, 200, 256), seed=77)
    w[1, :, :] = 0.0
    q, sf = dg.dg_quantize_128x128(torch.from_numpy(w).cuda())
    q0, b0 = quant.quantize_128x128_grouped(w)
    assert np.array_equal(q.cpu().numpy(), q0)
    assert np.array_equal(sf.cpu().numpy(), b0)


def test_quantize_rejects_bad_args():
    x = torch.zeros(4, 100, device="cuda")
    with pytest.raises(dg.DGError):
        dg.dg_quantize_1x128(x)          # K % 128 != 0


# ------------------------------------------------ operands stored K outermost
@pytest.mark.parametrize("pow2", [False, True])
@pytest.mark.parametrize("k,m,dtype", [(256, 300, torch.float32), (1024, 64, torch.float32),
                                       (384, 136, torch.bfloat16)])
def test_128x1_is_the_1x128_quantizer_of_the_transpose(k, m, dtype, pow2):
    # groups of 128 consecutive K elements of each column of x [K][M] -- the
    # oracle's 1x128 quantizer on the logical [M][K] operand, bit for bit
    x = inputs.activations(m, k, seed=k + m, outliers=True)
    x[3, :128] = 0.0                       # an all-zero group
    xd = torch.from_numpy(np.ascontiguousarray(x.T)).cuda().to(dtype)
    xs = xd.float().cpu().numpy().T       # the values the device sees, [M][K]
    q, sf = dg.dg_quantize_128x1(xd, pow2=pow2)
    torch.cuda.synchronize()
    q0, a0 = quant.quantize_1x128(np.ascontiguousarray(xs), pow2=pow2)
    assert np.array_equal(q.cpu().numpy(), q0.T)
    assert np.array_equal(sf.cpu().numpy()[:, :m], a0.T)
