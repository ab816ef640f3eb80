"""Host-side pieces of bench.py that run without a GPU: the oracle samples
behind `cpu_baseline` and the reference arm, on tiny versions of the grouped
workloads."""

import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from moe_grouped_gemm_act_b200 import inputs  # noqa: E402


@pytest.mark.parametrize("kind", ["masked", "contiguous"])
def test_grouped_oracle_sample_counts_valid_rows(kind):
    spec = dict(kind=kind, groups=4, n=256, k=256, seed=3, m_max=64, tokens=300)
    s = bench.GroupedOracleSample(spec, rows=8, cols=128)
    secs, flops = s.run()
    assert secs > 0
    n_rows = sum(len(xr) for xr, _, _ in s.prepared)
    assert 0 < n_rows <= 8 * bench.GroupedOracleSample.EXPERTS
    assert flops == 2.0 * n_rows * 128 * 256


def test_grouped_oracle_sample_takes_experts_with_rows():
    # masked: experts with zero valid rows are skipped
    spec = dict(kind="masked", groups=6, n=128, k=128, seed=0, m_max=32)
    counts = inputs.masked_counts(6, 32, seed=0)
    s = bench.GroupedOracleSample(spec, rows=64, cols=128)
    want = [int(c) for c in counts if c > 0][:bench.GroupedOracleSample.EXPERTS]
    assert [len(xr) for xr, _, _ in s.prepared] == [min(c, 64) for c in want]


def test_workload_specs_name_their_bound():
    for name, bound in [("prefill", "tensor"), ("prefill_acc", "tensor"), ("decode64", "hbm"),
                        ("decode128", "hbm"), ("contiguous", "tensor"), ("masked", "hbm"),
                        ("kgrouped", "tensor")]:
        assert bench.workload_spec(name)["bound"] == bound
    with pytest.raises(SystemExit):
        bench.workload_spec("nope")


def test_measured_traffic_follows_the_source_hash(monkeypatch):
    monkeypatch.setitem(bench.GEMM_TRAFFIC, "prefill", (bench.gemm_source_hash(), 1.5e8))
    assert bench.measured_traffic("prefill") == 1.5e8
    monkeypatch.setitem(bench.GEMM_TRAFFIC, "prefill", ("0" * 16, 1.5e8))
    assert bench.measured_traffic("prefill") is None
    assert bench.measured_traffic("no such workload") is None
    assert np.isfinite(bench.job_throughput(1.0, 1, 1, 1.0))


def test_default_workload_traffic_matches_the_current_sources():
    # the bench's default line must carry the traffic of the sources it runs
    assert bench.measured_traffic("prefill") is not None


def test_code_key_ignores_comments_but_not_code():
    src = 'int f(int x) {  // doubles\n  /* the "// value" */ return 2 * x; }\nconst char *s = "a // b";\n'
    same = 'int f(int x) {\n  return 2 * x;  // changed comment\n}\nconst char *s = "a // b";'
    other = 'int f(int x) { return 3 * x; }\nconst char *s = "a // b";'
    lit = 'int f(int x) { return 2 * x; }\nconst char *s = "a // c";'
    key = bench.gemm_source_hash([src])
    assert bench.gemm_source_hash([same]) == key
    assert bench.gemm_source_hash([other]) != key
    assert bench.gemm_source_hash([lit]) != key       # text inside a literal is code
    assert bench.strip_comments("a/*x*/b") == "a b"


def test_k_grouped_oracle_sample():
    spec = dict(kind="kgrouped", groups=3, m=40, n=136, tokens=300, seed=5)
    a, b, lay = bench.KGroupedOracleSample.generate(spec)
    assert a.shape == (40, lay.k_total) and b.shape == (136, lay.k_total)
    # padding tokens are zero in both operands
    start = 0
    for cnt, size in zip(lay.counts, lay.k_sizes):
        assert not a[:, start + int(cnt):start + int(size)].any()
        assert not b[:, start + int(cnt):start + int(size)].any()
        start += int(size)
    s = bench.make_sampler(spec, rows=8, cols=64)
    secs, flops = s.run()
    assert secs > 0 and flops == 2.0 * 8 * 64 * 300
    # the GPU arm's host slices give the same sample
    s2 = bench.KGroupedOracleSample(spec, 8, 64, src=bench.KGroupedOracleSample.source(a, b))
    assert np.array_equal(s2.a, s.a) and np.array_equal(s2.b, s.b)


def test_per_shape_report_fractions():
    from types import SimpleNamespace
    shapes = [dict(n=256, k=1024), dict(n=512, k=2048)]
    data = SimpleNamespace(m=128, shapes=shapes, acc=False)
    data.shape_bytes = lambda s: bench.DenseData.shape_bytes(data, s)
    rows = bench.per_shape_report(data, [0.5, 2.0], "tensor", 1000.0)
    assert rows[0]["tflops"] == pytest.approx(2 * 128 * 256 * 1024 / 0.5e-3 / 1e12)
    assert rows[1]["frac"] == pytest.approx(rows[1]["tflops"] / 1000.0)
    assert rows[0]["gemm_us_alone"] == pytest.approx(500.0)
    hb = bench.per_shape_report(data, [0.5, 2.0], "hbm", 6000.0)
    want = 128 * 1024 + 4 * 128 * 8 + 256 * 1024 + 4 * 2 * 8 + 2 * 128 * 256
    assert hb[0]["gbs"] == pytest.approx(want / 0.5e-3 / 1e9)
    assert hb[0]["frac"] == pytest.approx(hb[0]["gbs"] / 6000.0)


def test_k_grouped_bench_data_on_the_host(monkeypatch):
    # the weight-gradient workload's host logic, with a stand-in for the
    # library (records the calls) and CPU tensors: no kernel runs here
    import torch
    calls = []

    class FakeDG:
        @staticmethod
        def dg_get_tma_aligned_size(n, e):
            return -(-n // 4) * 4

        @staticmethod
        def dg_quantize_1x128(x, q=None, sf=None):
            calls.append(("quantize", tuple(x.shape)))
            m, k = x.shape
            return (torch.zeros((m, k), dtype=torch.uint8) if q is None else q,
                    torch.zeros((k // 128, -(-m // 4) * 4)) if sf is None else sf)

        @staticmethod
        def dg_k_grouped_fp8_gemm_nt_contiguous(a, sfa, b, sfb, d, k_sizes, c=None):
            calls.append(("kgrouped", tuple(a.shape), tuple(b.shape), tuple(d.shape),
                          tuple(k_sizes.tolist())))
            return d

    import moe_grouped_gemm_act_b200 as dg_mod
    for name in ("dg_get_tma_aligned_size", "dg_quantize_1x128",
                 "dg_k_grouped_fp8_gemm_nt_contiguous"):
        monkeypatch.setattr(dg_mod, name, getattr(FakeDG, name))
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a: None)
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self: self)
    spec = dict(name="kgrouped", kind="kgrouped", bound="tensor", groups=3, m=64, n=136,
                tokens=300, seed=5, desc="test")
    data = bench.KGroupedData(spec, torch.device("cpu"))
    lay = inputs.k_grouped_layout(300, 3, seed=5)
    k = lay.k_total
    assert data.flops() == 2.0 * 64 * 136 * 300
    assert data.gemm_bytes() == (64 + 136) * k + 4 * (64 + 136) * (k // 128) + \
        4 * 3 * 64 * 136 + 4 * 3
    assert data.input_bytes() == (64 + 136) * k * 4
    assert data.launches_per_step() == 3
    data.step()
    assert calls == [("quantize", (64, k)), ("quantize", (136, k)),
                     ("kgrouped", (64, k), (136, k), (3, 64, 136), tuple(lay.k_sizes))]
    calls.clear()
    data.make_host()
    assert data.h2d == ((64 + 136) * k + 3) * 4 and data.d2h == 3 * 64 * 136 * 4
    data.e2e_step(torch.device("cpu"))
    assert [c[0] for c in calls] == ["quantize", "quantize", "kgrouped"]
    rows = bench.per_shape_report(data, [1.0], "tensor", 1000.0)
    assert rows[0]["k"] == 300 and rows[0]["tflops"] == pytest.approx(2 * 64 * 136 * 300 / 1e-3 / 1e12)
    sampler = bench.make_sampler(spec, 8, 16, data)
    assert isinstance(sampler, bench.KGroupedOracleSample)
    assert sampler.a.shape == (8, k) and sampler.b.shape == (16, k)


def test_dense_and_grouped_byte_helpers():
    import torch
    d = object.__new__(bench.DenseData)
    d.m, d.acc = 64, True
    d.shapes = [dict(n=256, k=512, a32=torch.zeros(64, 512), qb=torch.zeros(256, 512,
                                                                             dtype=torch.uint8))]
    s = d.shapes[0]
    base = 64 * 512 + 4 * 64 * 4 + 256 * 512 + 4 * 2 * 4 + 2 * 64 * 256
    assert d.shape_bytes(s) == base + 4 * 64 * 256
    assert d.gemm_bytes() == d.shape_bytes(s)
    assert d.input_bytes() == 64 * 512 * 4 + 256 * 512
    g = object.__new__(bench.GroupedData)
    g.m, g.active = 100, 2
    g.shapes = [dict(n=256, k=512, index=torch.zeros(3, dtype=torch.int32),
                     a32=torch.zeros(128, 512), qb=torch.zeros(4, 256, 512, dtype=torch.uint8))]
    assert g.shape_bytes(g.shapes[0]) == g.gemm_bytes()
    rows = bench.per_shape_report(g, [0.01], "hbm", 6540.0)
    assert rows[0]["gbs"] == pytest.approx(g.gemm_bytes() / 1e-5 / 1e9)
