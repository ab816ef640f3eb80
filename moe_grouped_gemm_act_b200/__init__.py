"""B200 (sm_100a) fine-grained block-scaled FP8 GEMM -- Python binding.

A thin ctypes layer over ``libdg.so`` (declared in ``include/dg.h``).  The
functions here only marshal torch tensors into pointers, sizes and the current
CUDA stream; every step of the computation runs in the library's CUDA kernels.
There is no CPU fallback: if the library is missing or the device is not
sm_100, the calls raise.

Entry points (same names as the C ABI):

* ``dg_quantize_1x128(x, pow2=False)`` -> (q, sf)    1 x 128 E4M3 activations
* ``dg_quantize_128x128(w, pow2=False)`` -> (q, sf)  128 x 128 E4M3 weights
* ``dg_quantize_128x1(x, pow2=False)`` -> (q, sf)  1 x 128-along-K groups of an
  operand stored [K, M] (K outermost)
* ``dg_pack_ue8m0(sf, m)`` -> packed int32 UE8M0 scales (4 K groups per word)
* ``dg_pack_ue8m0_128x128(sf, n)`` -> B's 128 x 128 block scales packed per row
* ``dg_fp8_gemm_nt(a, sfa, b, sfb, d, workspace=None)``
* ``dg_fp8_gemm_nt_accumulate(a, sfa, b, sfb, c, d, workspace=None)``  D = C + A B^T
* ``dg_fp8_gemm_nt_noalloc(a, sfa, b, sfb, d)``
* ``dg_fp8_gemm_nt_quantize(a, sfa, b, sfb, pow2=False)`` -> (dq, sfd)  the
  output quantized 1 x 128 in the epilogue (E4M3 codes and MN-major scales)
* ``dg_fp8_gemm_nn / _tn / _tt(a, sfa, b, sfb, d, workspace=None)``  the other
  operand layouts (A stored [K, M] for T, B stored [K, N] for N)
* ``dg_m_grouped_fp8_gemm_nt_contiguous(a, sfa, b, sfb, d, m_indices)``
* ``dg_m_grouped_fp8_gemm_nt_masked(a, sfa, b, sfb, d, masked_m)``
* ``dg_k_grouped_fp8_gemm_nt_contiguous(a, sfa, b, sfb, d, k_sizes, c=None)``
* ``dg_k_grouped_fp8_gemm_tn_contiguous(a, sfa, b, sfb, d, k_sizes, c=None)``
  (a [K, M] and b [K, N])
* ``dg_fp8_gemm_nt_ue8m0(a, sfa, b, sfb, d)``, ``dg_m_grouped_fp8_gemm_nt_masked_ue8m0(
  a, sfa, b, sfb, d, masked_m)``  power-of-two scales as packed UE8M0 words,
  applied by the tensor cores
* ``dg_get_device_status()``, helpers ``dg_get_tma_aligned_size``,
  ``dg_get_mk_alignment_for_contiguous_layout``, ``dg_set_num_sms``,
  ``dg_get_num_sms``, ``dg_fp8_gemm_nt_workspace_size``.

Layouts follow the header: A [M, K] uint8 (E4M3 codes), its scales MN-major
[K/128, ld] (``sf.t()`` of the logical [M, K/128]), B [N, K] uint8 with scales
[ceil(N/128), K/128], D [M, N] bfloat16.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdg.so")

DG_OK = 0
DG_DTYPE_F32, DG_DTYPE_BF16 = 0, 1
DG_SCALE_FP32, DG_SCALE_POW2 = 0, 1
DG_ERR_INVALID_ARG, DG_ERR_ALIGNMENT, DG_ERR_UNSUPPORTED_ARCH = -1, -2, -3
DG_ERR_CUDA, DG_ERR_WORKSPACE = -4, -5
DG_ERR_TIMEOUT, DG_ERR_DEVICE_DATA = -6, -7

EXPORTS = [
    "dg_status_string", "dg_get_mk_alignment_for_contiguous_layout",
    "dg_get_tma_aligned_size", "dg_set_num_sms", "dg_get_num_sms",
    "dg_quantize_1x128", "dg_quantize_128x1", "dg_quantize_128x128", "dg_pack_ue8m0",
    "dg_pack_ue8m0_128x128",
    "dg_fp8_gemm_nt", "dg_fp8_gemm_nt_ue8m0", "dg_m_grouped_fp8_gemm_nt_masked_ue8m0",
    "dg_fp8_gemm_nn", "dg_fp8_gemm_tn", "dg_fp8_gemm_tt", "dg_k_grouped_fp8_gemm_tn_contiguous",
    "dg_fp8_gemm_nt_quantize",
    "dg_fp8_gemm_nt_workspace_size", "dg_fp8_gemm_nt_noalloc", "dg_fp8_gemm_nt_accumulate",
    "dg_m_grouped_fp8_gemm_nt_contiguous",
    "dg_m_grouped_fp8_gemm_nt_masked", "dg_k_grouped_fp8_gemm_nt_contiguous",
    "dg_get_device_status",
]

_lib = None


class DGError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libdg.so (once) and declares the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing; build it with `python -m moe_grouped_gemm_act_b200.build`")
    lib = ctypes.CDLL(path)
    P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    sig = {
        "dg_status_string": (ctypes.c_char_p, [I]),
        "dg_get_mk_alignment_for_contiguous_layout": (I, []),
        "dg_get_tma_aligned_size": (I64, [I64, I]),
        "dg_set_num_sms": (I, [I]),
        "dg_get_num_sms": (I, []),
        "dg_quantize_1x128": (I, [P, I, I64, I64, I64, I64, P, I64, P, I64, I, P]),
        "dg_quantize_128x128": (I, [P, I64, I64, I64, P, P, I, P]),
        "dg_quantize_128x1": (I, [P, I, I64, I64, I64, P, I64, P, I64, I, P]),
        "dg_pack_ue8m0": (I, [P, I64, I64, I64, I64, P, I64, P]),
        "dg_pack_ue8m0_128x128": (I, [P, I64, I64, I64, P, I64, P]),
        "dg_fp8_gemm_nt_ue8m0": (I, [P, P, I64, P, P, I64, P, I64, I64, I64, P]),
        "dg_m_grouped_fp8_gemm_nt_masked_ue8m0":
            (I, [P, P, I64, P, P, I64, P, P, I, I64, I64, I64, P]),
        "dg_fp8_gemm_nt": (I, [P, P, I64, P, P, P, I64, I64, I64, P, SZ, P]),
        "dg_fp8_gemm_nn": (I, [P, P, I64, P, P, P, I64, I64, I64, P, SZ, P]),
        "dg_fp8_gemm_nt_quantize": (I, [P, P, I64, P, P, P, P, I64, I64, I64, I64, I, P]),
        "dg_fp8_gemm_tn": (I, [P, P, I64, P, P, P, I64, I64, I64, P, SZ, P]),
        "dg_fp8_gemm_tt": (I, [P, P, I64, P, P, P, I64, I64, I64, P, SZ, P]),
        "dg_k_grouped_fp8_gemm_tn_contiguous":
            (I, [P, P, I64, P, P, I64, P, P, P, I, I64, I64, I64, P]),
        "dg_fp8_gemm_nt_workspace_size": (SZ, [I64, I64, I64]),
        "dg_fp8_gemm_nt_noalloc": (I, [P, P, I64, P, P, P, I64, I64, I64, P]),
        "dg_fp8_gemm_nt_accumulate": (I, [P, P, I64, P, P, P, P, I64, I64, I64, P, SZ, P]),
        "dg_m_grouped_fp8_gemm_nt_contiguous":
            (I, [P, P, I64, P, P, P, P, I64, I64, I64, I, P]),
        "dg_m_grouped_fp8_gemm_nt_masked":
            (I, [P, P, I64, P, P, P, P, I, I64, I64, I64, P]),
        "dg_k_grouped_fp8_gemm_nt_contiguous":
            (I, [P, P, I64, P, P, I64, P, P, P, I, I64, I64, I64, P]),
        "dg_get_device_status": (I, [P, ctypes.POINTER(ctypes.c_int)]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().dg_status_string(int(status)).decode()


def _check(rc: int, what: str) -> None:
    if rc != DG_OK:
        raise DGError(rc, what)


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _need_cuda(*ts: torch.Tensor) -> None:
    for t in ts:
        if not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors (there is no CPU path)")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def _expect(t: torch.Tensor | None, name: str, dtype: torch.dtype, shape: tuple) -> None:
    """Raises ValueError unless t has this dtype and shape.  A shape entry of
    None accepts any extent; a pair (lo, "ld") accepts any multiple of 4 that
    is at least lo (the leading dimension of an MN-major scale tensor).  The C
    ABI takes raw pointers and cannot check extents, so every tensor is
    checked here before the call."""
    if t is None:
        raise ValueError(f"{name} is required")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != len(shape):
        raise ValueError(f"{name} must have {len(shape)} dimensions, got shape {tuple(t.shape)}")
    for i, (got, want) in enumerate(zip(t.shape, shape)):
        if want is None:
            continue
        if isinstance(want, tuple):
            lo = want[0]
            if got < lo or got % 4:
                raise ValueError(f"{name}: dimension {i} is {got}; it must be a multiple of 4 "
                                 f">= {lo} (shape {tuple(t.shape)})")
        elif got != want:
            raise ValueError(f"{name}: dimension {i} is {got}, expected {want} "
                             f"(shape {tuple(t.shape)})")


def _gemm_operands(a, sfa, b, sfb, m, n, k, groups=None, a_batch=None):
    """Checks the FP8 operands and their scales of an NT GEMM: A [.., M, K]
    uint8 with MN-major 1x128 scales [.., K/128, ld >= M], B [.., N, K] uint8
    with 128x128 scales [.., ceil(N/128), K/128]."""
    if k % 128:
        return  # the C ABI rejects it (DG_ERR_INVALID_ARG) before touching memory
    lead_a = () if a_batch is None else (a_batch,)
    lead_b = () if groups is None else (groups,)
    _expect(a, "a", torch.uint8, lead_a + (m, k))
    _expect(sfa, "sfa", torch.float32, lead_a + (k // 128, (m, "ld")))
    _expect(b, "b", torch.uint8, lead_b + (n, k))
    _expect(sfb, "sfb", torch.float32, lead_b + (-(-n // 128), k // 128))


# ------------------------------------------------------------------ helpers
def dg_get_mk_alignment_for_contiguous_layout() -> int:
    return load_library().dg_get_mk_alignment_for_contiguous_layout()


def dg_get_tma_aligned_size(n: int, elem_bytes: int) -> int:
    return load_library().dg_get_tma_aligned_size(n, elem_bytes)


def dg_set_num_sms(n: int) -> None:
    _check(load_library().dg_set_num_sms(n), "dg_set_num_sms")


def dg_get_num_sms() -> int:
    return load_library().dg_get_num_sms()


def dg_fp8_gemm_nt_workspace_size(m: int, n: int, k: int) -> int:
    return load_library().dg_fp8_gemm_nt_workspace_size(m, n, k)


def dg_get_device_status(stream=None) -> int:
    st = ctypes.c_int(0)
    _check(load_library().dg_get_device_status(_stream(stream), ctypes.byref(st)),
           "dg_get_device_status")
    return st.value


# ------------------------------------------------------------------ quantizers
def dg_quantize_1x128(x: torch.Tensor, pow2: bool = False, q=None, sf=None,
                      stream=None):
    """1 x 128 quantization of x [M, K] or [B, M, K] (float32 or bfloat16).

    Returns (q uint8 like x, sf float32 [K/128, ld] or [B, K/128, ld]) with
    ld = dg_get_tma_aligned_size(M, 4); sf[..., g, i] is the scale of row i,
    group g.
    """
    _need_cuda(x)
    batched = x.dim() == 3
    xb = x if batched else x.unsqueeze(0)
    b, m, k = xb.shape
    dtype = {torch.float32: DG_DTYPE_F32, torch.bfloat16: DG_DTYPE_BF16}.get(x.dtype)
    if dtype is None:
        raise ValueError("x must be float32 or bfloat16")
    ld = dg_get_tma_aligned_size(m, 4)
    if q is None:
        q = torch.empty(xb.shape, dtype=torch.uint8, device=x.device)
    if sf is None:
        sf = torch.empty((b, k // 128, ld), dtype=torch.float32, device=x.device)
    _need_cuda(q, sf)
    if k % 128 == 0:  # (otherwise the C ABI rejects the call)
        _expect(q if q.dim() == 3 else q.unsqueeze(0), "q", torch.uint8, (b, m, k))
        _expect(sf if sf.dim() == 3 else sf.unsqueeze(0), "sf", torch.float32,
                (b, k // 128, (m, "ld")))
    rc = load_library().dg_quantize_1x128(
        _ptr(xb), dtype, b, m, k, k, _ptr(q), k, _ptr(sf), sf.shape[-1],
        DG_SCALE_POW2 if pow2 else DG_SCALE_FP32, _stream(stream))
    _check(rc, "dg_quantize_1x128")
    if not batched:
        return q.view(m, k), sf.view(k // 128, sf.shape[-1])
    return q, sf


def dg_quantize_128x1(x: torch.Tensor, pow2: bool = False, q=None, sf=None, stream=None):
    """1 x 128-along-K quantization of an operand stored [K, M] (float32 or
    bfloat16): returns (q uint8 [K, M], sf float32 [K/128, ld]) with ld =
    dg_get_tma_aligned_size(M, 4); sf[g, m] is the scale of column m's K
    group g.  Bit-exact with dg_quantize_1x128 of x.T."""
    _need_cuda(x)
    k, m = x.shape
    dtype = {torch.float32: DG_DTYPE_F32, torch.bfloat16: DG_DTYPE_BF16}.get(x.dtype)
    if dtype is None:
        raise ValueError("x must be float32 or bfloat16")
    if q is None:
        q = torch.empty((k, m), dtype=torch.uint8, device=x.device)
    if sf is None:
        sf = torch.empty((k // 128, dg_get_tma_aligned_size(m, 4)), dtype=torch.float32,
                         device=x.device)
    _need_cuda(q, sf)
    if k % 128 == 0:
        _expect(q, "q", torch.uint8, (k, m))
        _expect(sf, "sf", torch.float32, (k // 128, (m, "ld")))
    rc = load_library().dg_quantize_128x1(
        _ptr(x), dtype, k, m, m, _ptr(q), m, _ptr(sf), sf.shape[-1],
        DG_SCALE_POW2 if pow2 else DG_SCALE_FP32, _stream(stream))
    _check(rc, "dg_quantize_128x1")
    return q, sf


def dg_quantize_128x128(w: torch.Tensor, pow2: bool = False, stream=None):
    """128 x 128 quantization of w [N, K] or [G, N, K] float32.

    Returns (q uint8 like w, sf float32 [ceil(N/128), K/128] or
    [G, ceil(N/128), K/128])."""
    _need_cuda(w)
    if w.dtype != torch.float32:
        raise ValueError("w must be float32")
    grouped = w.dim() == 3
    wb = w if grouped else w.unsqueeze(0)
    g, n, k = wb.shape
    q = torch.empty(wb.shape, dtype=torch.uint8, device=w.device)
    sf = torch.empty((g, -(-n // 128), k // 128), dtype=torch.float32, device=w.device)
    rc = load_library().dg_quantize_128x128(
        _ptr(wb), g, n, k, _ptr(q), _ptr(sf),
        DG_SCALE_POW2 if pow2 else DG_SCALE_FP32, _stream(stream))
    _check(rc, "dg_quantize_128x128")
    if not grouped:
        return q[0], sf[0]
    return q, sf


def dg_pack_ue8m0(sf: torch.Tensor, m: int, packed=None, stream=None) -> torch.Tensor:
    """Packs power-of-two scales sf (float32 [Kg, ld] or [B, Kg, ld], the
    MN-major layout dg_quantize_1x128 returns) of m rows into UE8M0 words:
    int32 [ceil(Kg/4), ld'] (or [B, ceil(Kg/4), ld']), ld' =
    dg_get_tma_aligned_size(m, 4); word (p, i) holds groups 4p .. 4p+3 of row
    i, one byte each, lowest group in the lowest byte.  Scales that are not +0
    or a normal power of two are reported through dg_get_device_status()."""
    _need_cuda(sf)
    if sf.dtype != torch.float32:
        raise ValueError("sf must be float32")
    batched = sf.dim() == 3
    sb = sf if batched else sf.unsqueeze(0)
    b, kg, ld = sb.shape
    words = -(-kg // 4)
    if m > ld:
        raise ValueError(f"m = {m} exceeds the scale rows' leading dimension {ld}")
    if packed is None:
        packed = torch.empty((b, words, dg_get_tma_aligned_size(m, 4)), dtype=torch.int32,
                             device=sf.device)
    _need_cuda(packed)
    _expect(packed if packed.dim() == 3 else packed.unsqueeze(0), "packed", torch.int32,
            (b, words, (m, "ld")))
    rc = load_library().dg_pack_ue8m0(_ptr(sb), b, m, kg, ld, _ptr(packed), packed.shape[-1],
                                      _stream(stream))
    _check(rc, "dg_pack_ue8m0")
    return packed if batched else packed.view(words, packed.shape[-1])


def dg_pack_ue8m0_128x128(sf: torch.Tensor, n: int, packed=None, stream=None) -> torch.Tensor:
    """B's 128 x 128 block scales sf (float32 power-of-two values,
    [ceil(n/128), Kg] or [G, ceil(n/128), Kg], as dg_quantize_128x128(pow2=True)
    returns) written out per row of B in the packed UE8M0 layout: int32
    [ceil(Kg/4), ld] (or [G, ceil(Kg/4), ld]), ld = dg_get_tma_aligned_size(n,
    4); word (p, j) holds groups 4p .. 4p+3 of row j's block."""
    _need_cuda(sf)
    if sf.dtype != torch.float32:
        raise ValueError("sf must be float32")
    grouped = sf.dim() == 3
    sb = sf if grouped else sf.unsqueeze(0)
    g, nb, kg = sb.shape
    if nb != -(-n // 128):
        raise ValueError(f"sf has {nb} row blocks; n = {n} needs {-(-n // 128)}")
    words = -(-kg // 4)
    if packed is None:
        packed = torch.empty((g, words, dg_get_tma_aligned_size(n, 4)), dtype=torch.int32,
                             device=sf.device)
    _need_cuda(packed)
    _expect(packed if packed.dim() == 3 else packed.unsqueeze(0), "packed", torch.int32,
            (g, words, (n, "ld")))
    rc = load_library().dg_pack_ue8m0_128x128(_ptr(sb), g, n, kg, _ptr(packed),
                                              packed.shape[-1], _stream(stream))
    _check(rc, "dg_pack_ue8m0_128x128")
    return packed if grouped else packed.view(words, packed.shape[-1])


# ------------------------------------------------------------------ GEMMs
def dg_fp8_gemm_nt(a, sfa, b, sfb, d, workspace: torch.Tensor | None = None,
                   stream=None) -> torch.Tensor:
    """D = A * B^T with 1x128 (sfa, MN-major [K/128, ld]) and 128x128 (sfb)
    scales; d is a preallocated bfloat16 [M, N] tensor, returned."""
    _need_cuda(a, sfa, b, sfb, d)
    m, k = a.shape
    n = b.shape[0]
    _gemm_operands(a, sfa, b, sfb, m, n, k)
    _expect(d, "d", torch.bfloat16, (m, n))
    if workspace is not None:
        _need_cuda(workspace)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = load_library().dg_fp8_gemm_nt(
        _ptr(a), _ptr(sfa), sfa.shape[-1], _ptr(b), _ptr(sfb), _ptr(d), m, n, k,
        _ptr(workspace), ws_bytes, _stream(stream))
    _check(rc, "dg_fp8_gemm_nt")
    return d


def _fp8_gemm_layout(name, a_t, b_t, a, sfa, b, sfb, d, workspace, stream):
    """The dense GEMM with A stored [K, M] when a_t, B stored [K, N] when b_t
    (else [M, K] and [N, K]); the scales keep their logical layouts."""
    _need_cuda(a, sfa, b, sfb, d)
    if a_t:
        k, m = a.shape
    else:
        m, k = a.shape
    n = b.shape[1] if b_t else b.shape[0]
    if k % 128 == 0:
        _expect(a, "a", torch.uint8, (k, m) if a_t else (m, k))
        _expect(b, "b", torch.uint8, (k, n) if b_t else (n, k))
        _expect(sfa, "sfa", torch.float32, (k // 128, (m, "ld")))
        _expect(sfb, "sfb", torch.float32, (-(-n // 128), k // 128))
    _expect(d, "d", torch.bfloat16, (m, n))
    if workspace is not None:
        _need_cuda(workspace)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = getattr(load_library(), name)(
        _ptr(a), _ptr(sfa), sfa.shape[-1], _ptr(b), _ptr(sfb), _ptr(d), m, n, k,
        _ptr(workspace), ws_bytes, _stream(stream))
    _check(rc, name)
    return d


def dg_fp8_gemm_nt_quantize(a, sfa, b, sfb, pow2: bool = False, dq=None, sfd=None,
                            stream=None):
    """D = A * B^T quantized 1 x 128 in the GEMM's epilogue: returns (dq uint8
    [M, N] E4M3 codes, sfd float32 [N/128, ld] MN-major scales, ld =
    dg_get_tma_aligned_size(M, 4)) -- bit-identical to dg_quantize_1x128 of
    the BF16 result of the same tile form.  N % 128 == 0."""
    _need_cuda(a, sfa, b, sfb)
    m, k = a.shape
    n = b.shape[0]
    _gemm_operands(a, sfa, b, sfb, m, n, k)
    if n % 128:
        raise ValueError(f"N = {n} must be a multiple of 128")
    if dq is None:
        dq = torch.empty((m, n), dtype=torch.uint8, device=a.device)
    if sfd is None:
        sfd = torch.empty((n // 128, dg_get_tma_aligned_size(m, 4)), dtype=torch.float32,
                          device=a.device)
    _need_cuda(dq, sfd)
    _expect(dq, "dq", torch.uint8, (m, n))
    _expect(sfd, "sfd", torch.float32, (n // 128, (m, "ld")))
    rc = load_library().dg_fp8_gemm_nt_quantize(
        _ptr(a), _ptr(sfa), sfa.shape[-1], _ptr(b), _ptr(sfb), _ptr(dq), _ptr(sfd),
        sfd.shape[-1], m, n, k, DG_SCALE_POW2 if pow2 else DG_SCALE_FP32, _stream(stream))
    _check(rc, "dg_fp8_gemm_nt_quantize")
    return dq, sfd


def dg_fp8_gemm_nn(a, sfa, b, sfb, d, workspace=None, stream=None) -> torch.Tensor:
    """D = A * B^T with A [M, K] and B stored [K, N] (N contiguous, N % 16 == 0)."""
    return _fp8_gemm_layout("dg_fp8_gemm_nn", False, True, a, sfa, b, sfb, d, workspace, stream)


def dg_fp8_gemm_tn(a, sfa, b, sfb, d, workspace=None, stream=None) -> torch.Tensor:
    """D = A * B^T with A stored [K, M] and B stored [K, N] (M, N % 16 == 0)."""
    return _fp8_gemm_layout("dg_fp8_gemm_tn", True, True, a, sfa, b, sfb, d, workspace, stream)


def dg_fp8_gemm_tt(a, sfa, b, sfb, d, workspace=None, stream=None) -> torch.Tensor:
    """D = A * B^T with A stored [K, M] (M % 16 == 0) and B [N, K]."""
    return _fp8_gemm_layout("dg_fp8_gemm_tt", True, False, a, sfa, b, sfb, d, workspace, stream)


def dg_fp8_gemm_nt_accumulate(a, sfa, b, sfb, c, d, workspace: torch.Tensor | None = None,
                              stream=None) -> torch.Tensor:
    """D = C + A * B^T: as dg_fp8_gemm_nt, with c a float32 [M, N] tensor added
    before the BF16 rounding of d; d is returned."""
    _need_cuda(a, sfa, b, sfb, c, d)
    m, k = a.shape
    n = b.shape[0]
    _gemm_operands(a, sfa, b, sfb, m, n, k)
    _expect(c, "c", torch.float32, (m, n))
    _expect(d, "d", torch.bfloat16, (m, n))
    if workspace is not None:
        _need_cuda(workspace)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = load_library().dg_fp8_gemm_nt_accumulate(
        _ptr(a), _ptr(sfa), sfa.shape[-1], _ptr(b), _ptr(sfb), _ptr(c), _ptr(d), m, n, k,
        _ptr(workspace), ws_bytes, _stream(stream))
    _check(rc, "dg_fp8_gemm_nt_accumulate")
    return d


def dg_fp8_gemm_nt_noalloc(a, sfa, b, sfb, d, stream=None) -> torch.Tensor:
    """dg_fp8_gemm_nt without a caller-provided workspace, for callers that
    cannot allocate device memory (see include/dg.h): the split-K scratch is
    the library's own fixed 32 MiB per-device array.  Shapes whose preferred
    split needs more raise DGError (DG_ERR_WORKSPACE).  Calls that overlap on
    the GPU share that array and must be ordered."""
    _need_cuda(a, sfa, b, sfb, d)
    m, k = a.shape
    n = b.shape[0]
    _gemm_operands(a, sfa, b, sfb, m, n, k)
    _expect(d, "d", torch.bfloat16, (m, n))
    rc = load_library().dg_fp8_gemm_nt_noalloc(
        _ptr(a), _ptr(sfa), sfa.shape[-1], _ptr(b), _ptr(sfb), _ptr(d), m, n, k,
        _stream(stream))
    _check(rc, "dg_fp8_gemm_nt_noalloc")
    return d


def dg_m_grouped_fp8_gemm_nt_contiguous(a, sfa, b, sfb, d, m_indices,
                                        stream=None) -> torch.Tensor:
    """Contiguous m-grouped GEMM: a [M_total, K], b [G, N, K], m_indices int32
    [M_total] (-1 = padding); padding rows of d are not written."""
    _need_cuda(a, sfa, b, sfb, d, m_indices)
    m_total, k = a.shape
    g, n, _ = b.shape
    _gemm_operands(a, sfa, b, sfb, m_total, n, k, groups=g)
    _expect(d, "d", torch.bfloat16, (m_total, n))
    _expect(m_indices, "m_indices", torch.int32, (m_total,))
    rc = load_library().dg_m_grouped_fp8_gemm_nt_contiguous(
        _ptr(a), _ptr(sfa), sfa.shape[-1], _ptr(b), _ptr(sfb), _ptr(d),
        _ptr(m_indices), m_total, n, k, g, _stream(stream))
    _check(rc, "dg_m_grouped_fp8_gemm_nt_contiguous")
    return d


def dg_m_grouped_fp8_gemm_nt_masked(a, sfa, b, sfb, d, masked_m,
                                    stream=None) -> torch.Tensor:
    """Masked m-grouped GEMM: a [G, M_max, K], sfa [G, K/128, ld], b [G, N, K],
    masked_m int32 [G] on the device; rows >= masked_m[g] of d untouched."""
    _need_cuda(a, sfa, b, sfb, d, masked_m)
    g, m_max, k = a.shape
    n = b.shape[1]
    _gemm_operands(a, sfa, b, sfb, m_max, n, k, groups=g, a_batch=g)
    _expect(d, "d", torch.bfloat16, (g, m_max, n))
    _expect(masked_m, "masked_m", torch.int32, (g,))
    rc = load_library().dg_m_grouped_fp8_gemm_nt_masked(
        _ptr(a), _ptr(sfa), sfa.shape[-1], _ptr(b), _ptr(sfb), _ptr(d),
        _ptr(masked_m), g, m_max, n, k, _stream(stream))
    _check(rc, "dg_m_grouped_fp8_gemm_nt_masked")
    return d


def dg_k_grouped_fp8_gemm_tn_contiguous(a, sfa, b, sfb, d, k_sizes, c=None,
                                        stream=None) -> torch.Tensor:
    """The k-grouped GEMM with both operands stored with the token axis K
    outermost: a [K, M], b [K, N] uint8 (M, N % 16 == 0), scales and the rest
    as in dg_k_grouped_fp8_gemm_nt_contiguous."""
    _need_cuda(a, sfa, b, sfb, d, k_sizes)
    if c is not None:
        _need_cuda(c)
    k, m = a.shape
    n = b.shape[1]
    g = k_sizes.numel()
    if k % 128 == 0:
        _expect(a, "a", torch.uint8, (k, m))
        _expect(sfa, "sfa", torch.float32, (k // 128, (m, "ld")))
        _expect(b, "b", torch.uint8, (k, n))
        _expect(sfb, "sfb", torch.float32, (k // 128, (n, "ld")))
    _expect(d, "d", torch.float32, (g, m, n))
    _expect(k_sizes, "k_sizes", torch.int32, (g,))
    if c is not None:
        _expect(c, "c", torch.float32, (g, m, n))
    rc = load_library().dg_k_grouped_fp8_gemm_tn_contiguous(
        _ptr(a), _ptr(sfa), sfa.shape[-1], _ptr(b), _ptr(sfb), sfb.shape[-1], _ptr(c),
        _ptr(d), _ptr(k_sizes), g, m, n, k, _stream(stream))
    _check(rc, "dg_k_grouped_fp8_gemm_tn_contiguous")
    return d


def dg_k_grouped_fp8_gemm_nt_contiguous(a, sfa, b, sfb, d, k_sizes, c=None,
                                        stream=None) -> torch.Tensor:
    """K-grouped GEMM (MoE weight gradient): a [M, K] and b [N, K] uint8 with
    1x128 scales sfa [K/128, ld_a] and sfb [K/128, ld_b] (both from
    dg_quantize_1x128), k_sizes int32 [G] on the device (multiples of 128
    summing to K), d float32 [G, M, N]; d[g] = c[g] + a_g b_g^T over group
    g's K segment (c float32 [G, M, N] or None).  d is returned."""
    _need_cuda(a, sfa, b, sfb, d, k_sizes)
    if c is not None:
        _need_cuda(c)
    m, k = a.shape
    n = b.shape[0]
    g = k_sizes.numel()
    if k % 128 == 0:  # (otherwise the C ABI rejects the call)
        _expect(a, "a", torch.uint8, (m, k))
        _expect(sfa, "sfa", torch.float32, (k // 128, (m, "ld")))
        _expect(b, "b", torch.uint8, (n, k))
        _expect(sfb, "sfb", torch.float32, (k // 128, (n, "ld")))
    _expect(d, "d", torch.float32, (g, m, n))
    _expect(k_sizes, "k_sizes", torch.int32, (g,))
    if c is not None:
        _expect(c, "c", torch.float32, (g, m, n))
    rc = load_library().dg_k_grouped_fp8_gemm_nt_contiguous(
        _ptr(a), _ptr(sfa), sfa.shape[-1], _ptr(b), _ptr(sfb), sfb.shape[-1], _ptr(c),
        _ptr(d), _ptr(k_sizes), g, m, n, k, _stream(stream))
    _check(rc, "dg_k_grouped_fp8_gemm_nt_contiguous")
    return d


def _ue8m0_scales(sfa, sfb, m, n, k, lead=()):
    """Checks packed UE8M0 scale words: sfa [.., ceil(K/512), ld >= m],
    sfb [.., ceil(K/512), ld >= n], int32."""
    if k % 128:
        return
    words = -(-(k // 128) // 4)
    _expect(sfa, "sfa", torch.int32, lead + (words, (m, "ld")))
    _expect(sfb, "sfb", torch.int32, lead + (words, (n, "ld")))


def dg_fp8_gemm_nt_ue8m0(a, sfa, b, sfb, d, stream=None) -> torch.Tensor:
    """D = A * B^T with power-of-two scales as packed UE8M0 words applied by
    the tensor cores: a [M, K] and b [N, K] uint8, sfa int32 [ceil(K/512),
    ld_a] (dg_pack_ue8m0 of the 1x128 scales), sfb int32 [ceil(K/512), ld_b]
    per row of B (dg_pack_ue8m0_128x128 of the 128x128 block scales); d a
    preallocated bfloat16 [M, N] tensor, returned."""
    _need_cuda(a, sfa, b, sfb, d)
    m, k = a.shape
    n = b.shape[0]
    if k % 128 == 0:
        _expect(a, "a", torch.uint8, (m, k))
        _expect(b, "b", torch.uint8, (n, k))
    _ue8m0_scales(sfa, sfb, m, n, k)
    _expect(d, "d", torch.bfloat16, (m, n))
    rc = load_library().dg_fp8_gemm_nt_ue8m0(
        _ptr(a), _ptr(sfa), sfa.shape[-1], _ptr(b), _ptr(sfb), sfb.shape[-1], _ptr(d), m, n, k,
        _stream(stream))
    _check(rc, "dg_fp8_gemm_nt_ue8m0")
    return d


def dg_m_grouped_fp8_gemm_nt_masked_ue8m0(a, sfa, b, sfb, d, masked_m,
                                          stream=None) -> torch.Tensor:
    """The masked m-grouped GEMM with packed UE8M0 scales: a [G, M_max, K],
    sfa int32 [G, ceil(K/512), ld_a], b [G, N, K], sfb int32 [G, ceil(K/512),
    ld_b] per row of B, masked_m int32 [G] on the device; rows >= masked_m[g]
    of d are untouched."""
    _need_cuda(a, sfa, b, sfb, d, masked_m)
    g, m_max, k = a.shape
    n = b.shape[1]
    if k % 128 == 0:
        _expect(a, "a", torch.uint8, (g, m_max, k))
        _expect(b, "b", torch.uint8, (g, n, k))
    _ue8m0_scales(sfa, sfb, m_max, n, k, lead=(g,))
    _expect(d, "d", torch.bfloat16, (g, m_max, n))
    _expect(masked_m, "masked_m", torch.int32, (g,))
    rc = load_library().dg_m_grouped_fp8_gemm_nt_masked_ue8m0(
        _ptr(a), _ptr(sfa), sfa.shape[-1], _ptr(b), _ptr(sfb), sfb.shape[-1], _ptr(d),
        _ptr(masked_m), g, m_max, n, k, _stream(stream))
    _check(rc, "dg_m_grouped_fp8_gemm_nt_masked_ue8m0")
    return d
