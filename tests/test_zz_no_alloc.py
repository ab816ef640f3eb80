"""GPU test of dg_fp8_gemm_nt_noalloc, the dense GEMM entry point for callers
that cannot allocate device memory (runtimes that reserve all memory up front,
plugins whose host framework owns every buffer, loops that cannot afford
cudaMalloc's synchronisation).  It must give the same results as
dg_fp8_gemm_nt with a caller-allocated workspace, on two calls in a row (the
second call finds the first call's partial sums still in the library's fixed
scratch array).

This file is named so that pytest collects it last."""

import numpy as np
import pytest
import torch

import moe_grouped_gemm_act_b200 as dg
from moe_grouped_gemm_act_b200 import inputs
from oracle import bf16, quant

from _helpers import bits_of, check_gemm, dev, sfa_to_device

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 32 << 20


def case(m, n, k, seed):
    x = inputs.activations(m, k, seed=seed, outliers=True)
    w = inputs.weights((n, k), seed=seed + 1)
    qa, alpha = quant.quantize_1x128(x)
    qb, beta = quant.quantize_128x128(w)
    return dev(qa), sfa_to_device(alpha), dev(qb), dev(beta)


@pytest.mark.parametrize("m,n,k", [(64, 7168, 16384), (128, 2112, 7168),
                                   (64, 24576, 1536), (300, 392, 1024)])
def test_noalloc_matches_workspace_entry_point(m, n, k):
    a, sfa, b, sfb = case(m, n, k, seed=m + n)
    need = dg.dg_fp8_gemm_nt_workspace_size(m, n, k)
    assert need <= SCRATCH_BYTES
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    ref = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    dg.dg_fp8_gemm_nt(a, sfa, b, sfb, ref, workspace=ws)
    torch.cuda.synchronize()
    want = bf16.from_bits(bits_of(ref))
    for call in range(2):
        d = torch.full((m, n), 0x7FC1, dtype=torch.int16, device="cuda").view(torch.bfloat16)
        dg.dg_fp8_gemm_nt_noalloc(a, sfa, b, sfb, d)
        torch.cuda.synchronize()
        check_gemm(bits_of(d), want, f"noalloc call {call + 1} {m}x{n}x{k}")
    assert dg.dg_get_device_status() == 0


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # a shape whose preferred K split needs more than the array is refused
    # before anything is launched (buffers are full-size all the same)
    for m, n, k in [(256, 24576, 7168), (192, 24576, 16384), (256, 24576, 16384)]:
        if dg.dg_fp8_gemm_nt_workspace_size(m, n, k) > SCRATCH_BYTES:
            a = torch.zeros((m, k), dtype=torch.uint8, device="cuda")
            sfa = torch.zeros((k // 128, m), dtype=torch.float32, device="cuda")
            b = torch.zeros((n, k), dtype=torch.uint8, device="cuda")
            sfb = torch.zeros((-(-n // 128), k // 128), dtype=torch.float32, device="cuda")
            d = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
            with pytest.raises(dg.DGError) as e:
                dg.dg_fp8_gemm_nt_noalloc(a, sfa, b, sfb, d)
            assert e.value.status == -5   # DG_ERR_WORKSPACE
            return
    pytest.skip("no listed shape needs more than the scratch array on this device")
