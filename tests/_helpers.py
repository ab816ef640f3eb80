"""Shared helpers for the parity tests: moving oracle-layout arrays to the
device layouts of the C ABI and the GEMM acceptance check.

Acceptance (the library's stated bar for the GEMM): relative Frobenius error
<= 4e-3 and, per element, |d - o| <= 8e-3 |o| + 2e-3 rms(o).  The bound comes
from the arithmetic: BF16 output rounding is a relative 2**-9 ~ 2e-3 per
element, and the FP32 promotion plus the tensor cores' internal accumulation
order add far less; the rms term absorbs cancellation near zero.
"""

import os

import numpy as np
import torch

from oracle import bf16

REL_FRO = 4e-3
REL_ELEM = 8e-3
ABS_RMS = 2e-3


def sfa_to_device(alpha: np.ndarray, ld: int | None = None) -> torch.Tensor:
    """Logical alpha [M, Kg] -> MN-major device tensor [Kg, ld]."""
    m, kg = alpha.shape
    ld = ld or (-(-m // 4) * 4)
    out = np.zeros((kg, ld), np.float32)
    out[:, :m] = alpha.T
    return torch.from_numpy(out).cuda()


def sfa_batched_to_device(alpha: np.ndarray, ld: int | None = None) -> torch.Tensor:
    """[G, M, Kg] -> [G, Kg, ld]."""
    g, m, kg = alpha.shape
    ld = ld or (-(-m // 4) * 4)
    out = np.zeros((g, kg, ld), np.float32)
    out[:, :, :m] = alpha.transpose(0, 2, 1)
    return torch.from_numpy(out).cuda()


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bits_of(d: torch.Tensor) -> np.ndarray:
    """uint16 bit patterns of a bfloat16 device tensor."""
    return d.view(torch.int16).cpu().numpy().view(np.uint16)


def check_gemm(got_bits: np.ndarray, want_f64: np.ndarray, what: str = "") -> None:
    got = bf16.from_bits(got_bits)
    want = np.asarray(want_f64, np.float64)
    assert got.shape == want.shape
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    diff = got - want
    fro = np.linalg.norm(diff) / max(np.linalg.norm(want), 1e-300)
    rms = np.sqrt(np.mean(want ** 2))
    bound = REL_ELEM * np.abs(want) + ABS_RMS * rms
    worst = np.max(np.abs(diff) - bound)
    assert fro <= REL_FRO, f"{what}: relative Frobenius error {fro:.3e}"
    assert worst <= 0, f"{what}: element bound exceeded by {worst:.3e}"


def check_f32(got: np.ndarray, want_f64: np.ndarray, what: str = "") -> None:
    """The same acceptance bound for an FP32 result."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want_f64, np.float64)
    assert got.shape == want.shape
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    diff = got - want
    fro = np.linalg.norm(diff) / max(np.linalg.norm(want), 1e-300)
    rms = np.sqrt(np.mean(want ** 2))
    worst = np.max(np.abs(diff) - (REL_ELEM * np.abs(want) + ABS_RMS * rms))
    assert fro <= REL_FRO, f"{what}: relative Frobenius error {fro:.3e}"
    assert worst <= 0, f"{what}: element bound exceeded by {worst:.3e}"


class env:
    """Temporarily set library tuning variables (read at each call)."""

    def __init__(self, **kv):
        self.kv = {k: str(v) for k, v in kv.items()}

    def __enter__(self):
        self.old = {k: os.environ.get(k) for k in self.kv}
        os.environ.update(self.kv)

    def __exit__(self, *a):
        for k, v in self.old.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v
