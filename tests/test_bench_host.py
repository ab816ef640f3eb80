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
    assert rows[0]["gemm_us"] == pytest.approx(500.0)
    hb = bench.per_shape_report(data, [0.5, 2.0], "hbm", 6000.0)
    want = 128 * 1024 + 4 * 128 * 8 + 256 * 1024 + 4 * 2 * 8 + 2 * 128 * 256
    assert hb[0]["gbs"] == pytest.approx(want / 0.5e-3 / 1e9)
    assert hb[0]["frac"] == pytest.approx(hb[0]["gbs"] / 6000.0)
