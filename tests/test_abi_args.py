"""The C ABI's host-side argument checks (no GPU needed): every entry point
rejects the bad arguments include/dg.h lists with the documented status,
before it touches the device.  Pointers here are fake addresses that are
never dereferenced; every case fails validation before any CUDA call.  Also:
every binding entry point refuses host tensors (there is no CPU path)."""

import ctypes

import pytest
import torch

import moe_grouped_gemm_act_b200 as dg

OK, INV, ALN = dg.DG_OK, dg.DG_ERR_INVALID_ARG, dg.DG_ERR_ALIGNMENT
P = 0x10000        # 16-byte aligned, never dereferenced
ODD = 0x10004      # 4-byte aligned only


@pytest.fixture(scope="module")
def lib():
    return dg.load_library()


def test_quantize_1x128_checks(lib):
    q = lambda x=P, dt=0, b=1, m=4, k=128, ldx=128, qq=P, ldq=128, sf=P, ldsf=4, fl=0: \
        lib.dg_quantize_1x128(x, dt, b, m, k, ldx, qq, ldq, sf, ldsf, fl, None)
    assert q(x=None) == INV
    assert q(qq=None) == INV
    assert q(dt=2) == INV
    assert q(fl=4) == INV
    assert q(b=0) == INV
    assert q(k=100) == INV
    assert q(ldx=64) == INV
    assert q(ldsf=3) == INV
    assert q(ldq=136) == ALN
    assert q(m=5, ldsf=5) == ALN
    assert q(dt=1, ldx=132) == ALN            # BF16 rows of 264 bytes
    assert q(x=ODD) == ALN
    assert q(sf=ODD) == ALN


def test_quantize_128x128_checks(lib):
    q = lambda w=P, g=1, n=128, k=128, qq=P, sf=P, fl=0: \
        lib.dg_quantize_128x128(w, g, n, k, qq, sf, fl, None)
    assert q(w=None) == INV
    assert q(fl=2) == INV
    assert q(g=0) == INV
    assert q(k=0) == INV
    assert q(k=192) == INV
    assert q(n=-1) == INV
    assert q(w=ODD) == ALN


def test_pack_ue8m0_checks(lib):
    p = lambda sf=P, b=1, m=8, kg=4, ldsf=8, out=P, ldp=8: \
        lib.dg_pack_ue8m0(sf, b, m, kg, ldsf, out, ldp, None)
    assert p(b=0) == INV
    assert p(kg=0) == INV
    assert p(ldsf=4) == INV
    assert p(ldp=4) == INV
    assert p(m=0) == OK                       # nothing to do
    assert p(sf=None) == INV
    assert p(ldsf=10) == ALN
    assert p(out=ODD) == ALN


def gemm_args(**kw):
    a = dict(A=P, sfa=P, ld_sfa=128, B=P, sfb=P, D=P, M=128, N=256, K=512)
    a.update(kw)
    return a


def test_dense_gemm_checks(lib):
    def g(ws=None, nbytes=0, **kw):
        a = gemm_args(**kw)
        return lib.dg_fp8_gemm_nt(a["A"], a["sfa"], a["ld_sfa"], a["B"], a["sfb"], a["D"],
                                  a["M"], a["N"], a["K"], ws, nbytes, None)
    assert g(K=500) == INV
    assert g(N=260) == INV
    assert g(N=0) == INV
    assert g(M=-1) == INV
    assert g(A=None) == INV
    assert g(ld_sfa=64) == INV
    assert g(ld_sfa=130) == ALN
    assert g(D=ODD) == ALN
    assert g(sfb=ODD) == ALN
    assert g(ws=ODD, nbytes=64) == ALN


def test_accumulate_and_noalloc_checks(lib):
    def acc(C=P, **kw):
        a = gemm_args(**kw)
        return lib.dg_fp8_gemm_nt_accumulate(a["A"], a["sfa"], a["ld_sfa"], a["B"], a["sfb"], C,
                                             a["D"], a["M"], a["N"], a["K"], None, 0, None)
    assert acc(C=None) == INV
    assert acc(C=ODD) == ALN
    assert acc(K=64) == INV

    def na(**kw):
        a = gemm_args(**kw)
        return lib.dg_fp8_gemm_nt_noalloc(a["A"], a["sfa"], a["ld_sfa"], a["B"], a["sfb"],
                                          a["D"], a["M"], a["N"], a["K"], None)
    assert na(K=100) == INV
    assert na(N=12) == INV
    assert na(M=0) == OK


def test_grouped_gemm_checks(lib):
    def cont(idx=P, G=4, **kw):
        a = gemm_args(**kw)
        return lib.dg_m_grouped_fp8_gemm_nt_contiguous(a["A"], a["sfa"], a["ld_sfa"], a["B"],
                                                       a["sfb"], a["D"], idx, a["M"], a["N"],
                                                       a["K"], G, None)
    assert cont(idx=None) == INV
    assert cont(G=0) == INV
    assert cont(M=200, ld_sfa=200) == INV     # M_total not a multiple of 128
    assert cont(idx=ODD) == ALN

    def masked(mm=P, G=4, **kw):
        a = gemm_args(**kw)
        return lib.dg_m_grouped_fp8_gemm_nt_masked(a["A"], a["sfa"], a["ld_sfa"], a["B"],
                                                   a["sfb"], a["D"], mm, G, a["M"], a["N"],
                                                   a["K"], None)
    assert masked(mm=None) == INV
    assert masked(G=0) == INV
    assert masked(G=1025) == INV
    assert masked(K=130) == INV

    def kg(ks=P, G=4, C=None, ld_sfb=256, **kw):
        a = gemm_args(**kw)
        return lib.dg_k_grouped_fp8_gemm_nt_contiguous(a["A"], a["sfa"], a["ld_sfa"], a["B"],
                                                       a["sfb"], ld_sfb, C, a["D"], ks, G,
                                                       a["M"], a["N"], a["K"], None)
    assert kg(G=0) == INV
    assert kg(G=1025) == INV
    assert kg(ks=None) == INV
    assert kg(ld_sfb=128) == INV
    assert kg(ld_sfb=258) == ALN
    assert kg(ks=ODD) == ALN
    assert kg(C=ODD) == ALN
    assert kg(K=100) == INV
    assert kg(M=0) == OK                      # nothing to do


def test_device_status_needs_an_output(lib):
    assert lib.dg_get_device_status(None, ctypes.POINTER(ctypes.c_int)()) == INV


def test_every_tensor_entry_point_refuses_host_tensors():
    u8 = torch.zeros((128, 128), dtype=torch.uint8)
    f32 = torch.zeros((1, 128), dtype=torch.float32)
    d = torch.zeros((128, 128), dtype=torch.bfloat16)
    i32 = torch.zeros(128, dtype=torch.int32)
    calls = [
        lambda: dg.dg_quantize_1x128(torch.zeros(128, 128)),
        lambda: dg.dg_quantize_128x128(torch.zeros(128, 128)),
        lambda: dg.dg_pack_ue8m0(f32, 1),
        lambda: dg.dg_fp8_gemm_nt(u8, f32, u8, f32, d),
        lambda: dg.dg_fp8_gemm_nt_accumulate(u8, f32, u8, f32, torch.zeros(128, 128), d),
        lambda: dg.dg_fp8_gemm_nt_noalloc(u8, f32, u8, f32, d),
        lambda: dg.dg_m_grouped_fp8_gemm_nt_contiguous(u8, f32, u8.view(1, 128, 128), f32, d,
                                                       i32),
        lambda: dg.dg_m_grouped_fp8_gemm_nt_masked(u8.view(1, 128, 128), f32.view(1, 1, 128),
                                                   u8.view(1, 128, 128), f32, d.view(1, 128, 128),
                                                   i32[:1]),
        lambda: dg.dg_k_grouped_fp8_gemm_nt_contiguous(u8, f32, u8, f32,
                                                       torch.zeros((1, 128, 128)), i32[:1]),
    ]
    for call in calls:
        with pytest.raises(ValueError, match="CUDA"):
            call()
