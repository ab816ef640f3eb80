"""GPU test of dg_fp8_gemm_nt_noalloc, the dense GEMM entry point for callers
that cannot allocate device memory (runtimes that reserve all memory up front,
plugins whose host framework owns every buffer, loops that cannot afford
cudaMalloc's synchronisation).  Its split-K scratch is the library's own fixed
device array instead of a caller workspace.

What is checked, on two calls in a row:
* the result is bit-identical to dg_fp8_gemm_nt given the workspace size the
  library reports (both pick the same tile form and split), and within the
  GEMM tolerance of the oracle;
* shapes whose split goes through the scratch array -- a decode shape with
  the cluster reduction switched off, and the largest prefill shape, whose
  last partial wave of tiles is split along K -- so that the second call runs
  on an array holding the first call's partial sums and arrival counters;
* shapes that need no scratch (cluster reduction, no split);
* the bound that makes the array's size refusal unreachable on B200.

This file is named so that pytest collects it last."""

import numpy as np
import pytest
import torch

import moe_grouped_gemm_act_b200 as dg
from moe_grouped_gemm_act_b200 import inputs
from oracle import bf16, gemm, quant

from _helpers import bits_of, check_gemm, env

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 32 << 20


def device_case(m, n, k, seed):
    """Host inputs and their device quantization (bit-exact with the oracle's,
    which the quantizer tests check)."""
    x = inputs.activations(m, k, seed=seed, outliers=True)
    w = inputs.weights((n, k), seed=seed + 1)
    qa_d, sfa_d = dg.dg_quantize_1x128(torch.from_numpy(x).cuda())
    qb_d, sfb_d = dg.dg_quantize_128x128(torch.from_numpy(w).cuda())
    return x, w, (qa_d, sfa_d, qb_d, sfb_d)


def sampled_rows(m, seed):
    """First and last row of every 128-row tile plus two random rows."""
    g = np.random.default_rng(seed)
    rows = []
    for t in range(-(-m // 128)):
        lo, hi = 128 * t, min(128 * t + 127, m - 1)
        rows += [lo, hi]
        if hi > lo + 1:
            rows += list(g.integers(lo + 1, hi, size=2))
    return np.array(sorted(set(rows)))


def run_both(m, n, k, seed, **knobs):
    """dg_fp8_gemm_nt with the reported workspace, then two noalloc calls;
    returns (host inputs, reference bits, [bits of each noalloc call])."""
    x, w, (a, sfa, b, sfb) = device_case(m, n, k, seed)
    with env(**knobs):
        need = dg.dg_fp8_gemm_nt_workspace_size(m, n, k)
        assert need <= SCRATCH_BYTES
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
        ref = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
        dg.dg_fp8_gemm_nt(a, sfa, b, sfb, ref, workspace=ws)
        torch.cuda.synchronize()
        got = []
        for _ in range(2):
            d = torch.full((m, n), 0x7FC1, dtype=torch.int16, device="cuda").view(torch.bfloat16)
            dg.dg_fp8_gemm_nt_noalloc(a, sfa, b, sfb, d)
            torch.cuda.synchronize()
            got.append(bits_of(d))
    assert dg.dg_get_device_status() == 0
    return (x, w), bits_of(ref), got, need


def check_against_oracle(x, w, bits, rows, what):
    qa, alpha = quant.quantize_1x128(x[rows])
    qb, beta = quant.quantize_128x128(w)
    check_gemm(bits[rows], gemm.fp8_gemm_nt_f64(qa, alpha, qb, beta), what)


@pytest.mark.parametrize("m,n,k,knobs,uses_scratch", [
    # decode shape split along K, partials through the scratch array (the
    # cluster reduction, which needs none, switched off)
    (64, 7168, 16384, dict(DG_CLUSTER_SPLIT=0), True),
    # the largest prefill shape: 896 tiles of 128 x 256 on 148 SMs, the last
    # partial wave's tiles split along K through the scratch array
    (4096, 7168, 16384, {}, True),
    # decode shape reduced through distributed shared memory (no scratch)
    (128, 2112, 7168, {}, False),
    # no split at all
    (300, 392, 1024, {}, False),
])
def test_noalloc_matches_workspace_entry_point(m, n, k, knobs, uses_scratch):
    (x, w), ref, got, need = run_both(m, n, k, seed=m + n, **knobs)
    if uses_scratch:
        assert need > 0, "this shape was meant to split K through the scratch"
    for call, bits in enumerate(got):
        # same tile form and split as the workspace entry point: same bits
        assert np.array_equal(bits, ref), f"noalloc call {call + 1} differs from dg_fp8_gemm_nt"
        check_gemm(bits, bf16.from_bits(ref), f"noalloc call {call + 1} {m}x{n}x{k}")
    check_against_oracle(x, w, got[1], sampled_rows(m, seed=n + k), f"noalloc {m}x{n}x{k}")


def test_noalloc_scratch_need_is_bounded_by_the_sm_count():
    # Every split keeps split tiles x splits <= the SM count, so no shape
    # needs more than SMs x 128 x 256 x 4 bytes (+ counters) -- below the
    # 32 MiB array on B200, where the DG_ERR_WORKSPACE refusal is unreachable.
    sms = dg.dg_get_num_sms()
    assert sms > 0
    bound = sms * 128 * 256 * 4 + 4 * sms
    assert bound <= SCRATCH_BYTES
    worst = 0
    for m in (1, 64, 128, 129, 256, 300, 1000, 4096, 8192):
        for n in (8, 136, 392, 2112, 4096, 7168, 24576):
            for k in (128, 1024, 1536, 7168, 16384):
                need = dg.dg_fp8_gemm_nt_workspace_size(m, n, k)
                assert need <= ((bound + 255) // 256) * 256, (m, n, k, need)
                worst = max(worst, need)
    assert worst > 0, "no listed shape splits K"
