"""GPU parity of the UE8M0 scale packing against the oracle, through the C
ABI: bit-exact words for power-of-two scales straight from the device
quantizer, ragged row counts and group counts, batches, the full-size scale
grid of a 4096 x 16384 activation; untouched padding; invalid scales
reported through the device status word."""

import numpy as np
import pytest
import torch

import moe_grouped_gemm_act_b200 as dg
from moe_grouped_gemm_act_b200 import inputs
from oracle import quant, ue8m0

pytestmark = pytest.mark.gpu

SENTINEL = 0x5A5A5A5A


def pow2_scales(m, kg, seed, batch=1):
    """Random +0 / normal power-of-two scales, float32 [batch, m, kg]."""
    g = inputs.rng(seed)
    a = np.ldexp(1.0, g.integers(-126, 128, size=(batch, m, kg))).astype(np.float32)
    a[g.random((batch, m, kg)) < 0.05] = 0.0
    return a


def to_device_mn_major(alpha):
    """[batch, m, kg] -> device float32 [batch, kg, ld], ld = 4-aligned m."""
    b, m, kg = alpha.shape
    ld = dg.dg_get_tma_aligned_size(m, 4)
    sf = np.zeros((b, kg, ld), np.float32)
    sf[:, :, :m] = alpha.transpose(0, 2, 1)
    return torch.from_numpy(sf).cuda()


def packed_like(b, m, kg):
    ld = dg.dg_get_tma_aligned_size(m, 4)
    return torch.full((b, -(-kg // 4), ld), SENTINEL, dtype=torch.int32, device="cuda")


@pytest.mark.parametrize("m,k", [(1, 128), (37, 640), (128, 512), (300, 896)])
def test_pack_of_device_quantizer_scales_bit_exact(cuda_device, m, k):
    x = inputs.activations(m, k, seed=70 + m, outliers=True)
    x[0, :128] = 0.0                                   # a +0 scale
    _, sf = dg.dg_quantize_1x128(torch.from_numpy(x).cuda(), pow2=True)
    dg.dg_get_device_status()                          # read and clear
    packed = dg.dg_pack_ue8m0(sf, m)
    torch.cuda.synchronize()
    assert dg.dg_get_device_status() == dg.DG_OK
    _, alpha = quant.quantize_1x128(x, pow2=True)
    want = ue8m0.pack_1x128(alpha)
    got = packed.cpu().numpy()[:, :m]
    assert got.shape == want.shape
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


@pytest.mark.parametrize("batch,m,kg", [(1, 4096, 128), (3, 50, 5), (32, 256, 16), (2, 7, 131)])
def test_pack_matches_oracle_and_leaves_padding(cuda_device, batch, m, kg):
    alpha = pow2_scales(m, kg, seed=80 + kg, batch=batch)
    sf = to_device_mn_major(alpha)
    out = packed_like(batch, m, kg)
    dg.dg_get_device_status()
    dg.dg_pack_ue8m0(sf, m, packed=out)
    torch.cuda.synchronize()
    assert dg.dg_get_device_status() == dg.DG_OK
    got = out.cpu().numpy()
    for b in range(batch):
        want = ue8m0.pack_1x128(alpha[b])
        assert np.array_equal(got[b, :, :m].view(np.uint32), want.view(np.uint32))
    assert np.all(got[:, :, m:] == SENTINEL)


def test_fp32_scales_are_reported(cuda_device):
    x = inputs.activations(64, 512, seed=90)
    _, sf = dg.dg_quantize_1x128(torch.from_numpy(x).cuda())   # amax/448, not powers of two
    dg.dg_get_device_status()
    dg.dg_pack_ue8m0(sf, 64)
    torch.cuda.synchronize()
    assert dg.dg_get_device_status() == dg.DG_ERR_DEVICE_DATA
    assert dg.dg_get_device_status() == dg.DG_OK                # cleared by the read


@pytest.mark.parametrize("bad", [-2.0, -0.0, 3.0, float("inf"), float("nan"), 2.0 ** -130])
def test_each_invalid_scale_is_reported(cuda_device, bad):
    alpha = pow2_scales(8, 4, seed=91)
    alpha[0, 5, 2] = bad
    sf = to_device_mn_major(alpha)
    dg.dg_get_device_status()
    dg.dg_pack_ue8m0(sf, 8)
    torch.cuda.synchronize()
    assert dg.dg_get_device_status() == dg.DG_ERR_DEVICE_DATA
    with pytest.raises(ValueError):
        ue8m0.encode(alpha[0])


def test_empty_rows_and_bad_arguments(cuda_device):
    sf = to_device_mn_major(pow2_scales(6, 3, seed=92))
    out = packed_like(1, 6, 3)
    dg.dg_pack_ue8m0(sf, 0, packed=out)                 # M == 0: nothing written
    torch.cuda.synchronize()
    assert torch.all(out == SENTINEL)
    lib = dg.load_library()
    stream = torch.cuda.current_stream().cuda_stream
    # ld not a multiple of 4
    assert lib.dg_pack_ue8m0(sf.data_ptr(), 1, 6, 3, 6, out.data_ptr(), 8, stream) == \
        dg.DG_ERR_ALIGNMENT
    # ld below M, no groups, no batch
    assert lib.dg_pack_ue8m0(sf.data_ptr(), 1, 6, 3, 4, out.data_ptr(), 8, stream) == \
        dg.DG_ERR_INVALID_ARG
    assert lib.dg_pack_ue8m0(sf.data_ptr(), 1, 6, 0, 8, out.data_ptr(), 8, stream) == \
        dg.DG_ERR_INVALID_ARG
    assert lib.dg_pack_ue8m0(sf.data_ptr(), 0, 6, 3, 8, out.data_ptr(), 8, stream) == \
        dg.DG_ERR_INVALID_ARG
    assert lib.dg_pack_ue8m0(None, 1, 6, 3, 8, out.data_ptr(), 8, stream) == \
        dg.DG_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert torch.all(out == SENTINEL)
