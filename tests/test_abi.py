"""CPU checks of the C ABI boundary: the library loads, exports every entry
point that include/dg.h declares, and its host-only helpers behave as
documented.  No compute call is made (there may be no GPU here)."""

import ctypes
import os
import re

import pytest

import moe_grouped_gemm_act_b200 as dg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "dg.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dg_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from moe_grouped_gemm_act_b200 import build
    build.build()
    return dg.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), f"{n} declared in dg.h but not exported"
    assert sorted(names) == sorted(dg.EXPORTS)


def test_binding_has_every_entry_point():
    for n in declared_functions():
        if n != "dg_status_string":
            assert callable(getattr(dg, n)), n


def test_host_helpers(lib):
    assert dg.dg_get_mk_alignment_for_contiguous_layout() == 128
    assert dg.dg_get_tma_aligned_size(5, 4) == 8
    assert dg.dg_get_tma_aligned_size(8, 4) == 8
    assert dg.dg_get_tma_aligned_size(17, 1) == 32
    assert dg.dg_get_tma_aligned_size(3, 2) == 8
    assert dg.dg_get_tma_aligned_size(-1, 4) == -1
    assert dg.dg_get_tma_aligned_size(4, 3) == -1
    assert dg.status_string(0) == "ok"
    assert "timed out" in dg.status_string(-6)
    assert dg.status_string(12345) == "unknown status"
    assert lib.dg_fp8_gemm_nt_workspace_size(0, 128, 128) == 0
    # 32 x 96 tiles of 128 x 256 fill whole waves closely enough: no split
    assert lib.dg_fp8_gemm_nt_workspace_size(4096, 24576, 1536) == 0
    # 32 x 28 = 896 tiles = 6 waves of 148 + 8: the last 8 tiles split 16 ways
    # (8 x 16 FP32 partial tiles of 128 x 256, then 8 counters, 256-aligned)
    assert lib.dg_fp8_gemm_nt_workspace_size(4096, 7168, 7168) == \
        (8 * 16 * 128 * 256 * 4 + 8 * 4 + 255) // 256 * 256
    assert lib.dg_fp8_gemm_nt_workspace_size(64, 7168, 16384) % 256 == 0


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(dg, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        dg.load_library(str(tmp_path / "nope.so"))


def test_product_path_has_no_cpu_fallback():
    import torch
    x = torch.zeros(128, 128)
    with pytest.raises((ValueError, RuntimeError)):
        dg.dg_quantize_1x128(x)


def test_product_does_not_import_oracle():
    for f in os.listdir(os.path.join(ROOT, "moe_grouped_gemm_act_b200")):
        if f.endswith(".py"):
            src = open(os.path.join(ROOT, "moe_grouped_gemm_act_b200", f)).read()
            assert "oracle" not in re.sub(r'""".*?"""', "", src, flags=re.S), f
