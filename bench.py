"""Benchmark of the fine-grained block-scaled FP8 GEMM hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload W]
                    [--impl reference]

One step = one pass of the whole hot path over one batch of synthetic input:
for every (N, K) pair of the workload, quantize the FP32 activations A with the
1x128 quantizer kernel, then run the FP8 GEMM against the pre-quantized
(128x128) weights B.  Weights are quantized once before timing (they are
offline-quantized model parameters).  The headline workload is the dense
prefill set: M = 4096 and (N, K) in {(7168, 16384), (4096, 7168),
(24576, 1536), (2112, 7168)}.  By default every workload of the metric is
measured, one after the other: prefill (the line's value), decode at M = 64
and 128, the contiguous and masked MoE layouts, the masked layout with
power-of-two scales, the k-grouped weight gradient and D = C + A B^T; each
of the others is listed under config.workloads with its own roofline,
end-to-end rate and oracle sample.  ``--workload W`` measures one.

Reported (one JSON line on rank 0):
* value       whole-job TFLOP/s (2 M N K per GEMM, summed over shapes and
              ranks) with inputs resident in HBM, CUDA events on the launch
              stream, max over ranks;
* e2e         the same metric through the public API with pinned host buffers:
              host->device copy of A, B and scales, quantize, GEMM, and the
              device->host copy of D, all inside the timed region;
* roofline    the GEMM kernel's achieved TFLOP/s (or GB/s for the memory-bound
              workloads) over the measured peak;
* cpu_baseline the CPU oracle timed on a bounded row sample of the same work.

With --gpus N > 1 (launched by torch.distributed.run) every rank runs an
independent replica of the workload on its own GPU (the method has no
cross-GPU exchange): scaling is weak and the only collectives are the timing
barrier and the max-over-ranks reduction.

``--impl reference`` times the CPU oracle (the reference of this library) on
the host cores instead, one bounded row sample per step.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from moe_grouped_gemm_act_b200 import inputs  # noqa: E402

METRIC = "FP8 block-scaled GEMM TFLOPS & % of B200 FP8 peak / HBM roofline, per shape"
FP8_OVER_BF16 = 2.0  # nominal dense FP8 / BF16 tensor throughput ratio on B200

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per GEMM launch,
# averaged over the workload's launches, from ncu captures of this bench
# (profiles/fp8_gemm_*.md give the commands).  Each figure is valid only for
# the GEMM code it was taken on (gemm_source_hash, stored beside it); on a
# mismatch the bench reports null.
GEMM_TRAFFIC = {
    "prefill": ("54a8c4c38565ba2a", 209.7e6),
    "decode64": ("54a8c4c38565ba2a", 50.5e6),
    "decode128": ("54a8c4c38565ba2a", 51.1e6),
    "contiguous": ("54a8c4c38565ba2a", 987.4e6),
    "masked": ("54a8c4c38565ba2a", 531.0e6),
    "masked_pow2": ("54a8c4c38565ba2a", 531.2e6),
    "masked_ue8m0": ("54a8c4c38565ba2a", 535.2e6),
    "kgrouped": ("54a8c4c38565ba2a", 1437.5e6),
    "kgrouped_tn": ("54a8c4c38565ba2a", 1423.8e6),
    "prefill_acc": ("54a8c4c38565ba2a", 403.5e6),
    "prefill_quant": ("54a8c4c38565ba2a", 220.4e6),
    "prefill_ue8m0": ("54a8c4c38565ba2a", 213.4e6),
}


def strip_comments(src: str) -> str:
    """C/C++ source without comments and with whitespace runs collapsed, so
    that the traffic key follows the code, not its comments.  String and
    character literals are kept verbatim."""
    out, i, n = [], 0, len(src)
    while i < n:
        ch = src[i]
        if src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        elif ch in "\"'":
            j = i + 1
            while j < n and src[j] != ch:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        else:
            out.append(ch)
            i += 1
    return " ".join("".join(out).split())


def gemm_source_hash(texts=None) -> str:
    """Key of the GEMM's code: SHA-256 (first 16 hex digits) of csrc/gemm.cu,
    csrc/ptx.cuh and csrc/internal.h without comments."""
    import hashlib
    h = hashlib.sha256()
    if texts is None:
        texts = []
        for f in ("gemm.cu", "ptx.cuh", "internal.h"):
            with open(os.path.join(ROOT, "moe_grouped_gemm_act_b200", "csrc", f)) as fh:
                texts.append(fh.read())
    for t in texts:
        h.update(strip_comments(t).encode())
    return h.hexdigest()[:16]


def measured_traffic(workload: str):
    entry = GEMM_TRAFFIC.get(workload)
    if entry is None:
        return None
    try:
        return entry[1] if gemm_source_hash() == entry[0] else None
    except OSError:
        return None


# ---------------------------------------------------------------- workloads
def workload_spec(name: str) -> dict:
    if name == "prefill":
        return dict(name=name, kind="dense", m=inputs.PREFILL_M, nk=inputs.PREFILL_NK,
                    seeds=inputs.PREFILL_SEEDS, bound="tensor",
                    desc="dense NT prefill, M=4096, (N,K) in "
                         "{(7168,16384),(4096,7168),(24576,1536),(2112,7168)}; "
                         "A~N(0,1) with 0.1% x50 outliers, B~N(0,0.02); "
                         "1x128 / 128x128 FP32 scales, BF16 out")
    if name == "prefill_acc":
        return dict(name=name, kind="dense", m=inputs.PREFILL_M, nk=inputs.PREFILL_NK,
                    seeds=inputs.PREFILL_SEEDS, bound="tensor", acc=True,
                    desc="dense NT prefill with D = C + A*B^T, C FP32 ~ N(0,16) [M,N], "
                         "M=4096, (N,K) in {(7168,16384),(4096,7168),(24576,1536),"
                         "(2112,7168)}; A, B and scales as prefill")
    if name in ("decode64", "decode128"):
        m = 64 if name == "decode64" else 128
        return dict(name=name, kind="dense", m=m, nk=inputs.PREFILL_NK,
                    seeds=inputs.DECODE_SEEDS, bound="hbm",
                    desc=f"dense NT decode, M={m}, same four (N,K) pairs")
    if name == "contiguous":
        return dict(name=name, kind="contiguous", bound="tensor", **inputs.CONTIGUOUS,
                    desc="m-grouped contiguous, G=8, N=4096 K=7168, 32768 tokens "
                         "multinomial over experts, segments padded to 128")
    if name == "masked":
        return dict(name=name, kind="masked", bound="hbm", **inputs.MASKED,
                    desc="m-grouped masked, G=32, M_max=256, N=7168 K=2048, "
                         "masked_m ~ U{0..256}")
    if name == "masked_pow2":
        return dict(name=name, kind="masked", bound="hbm", pow2=True, **inputs.MASKED,
                    desc="m-grouped masked, G=32, M_max=256, N=7168 K=2048, "
                         "masked_m ~ U{0..256}, every scale rounded up to a power of two "
                         "(UE8M0-representable)")
    if name == "masked_ue8m0":
        return dict(name=name, kind="masked", bound="hbm", pow2=True, ue8m0=True,
                    **inputs.MASKED,
                    desc="m-grouped masked, G=32, M_max=256, N=7168 K=2048, "
                         "masked_m ~ U{0..256}, power-of-two scales as packed UE8M0 words "
                         "applied by the tensor cores (block-scaled MMA)")
    if name == "prefill_ue8m0":
        return dict(name=name, kind="dense", m=inputs.PREFILL_M, nk=inputs.PREFILL_NK,
                    seeds=inputs.PREFILL_SEEDS, bound="tensor", pow2=True, ue8m0=True,
                    desc="dense NT prefill with power-of-two scales as packed UE8M0 words "
                         "applied by the tensor cores (block-scaled MMA), M=4096, (N,K) in "
                         "{(7168,16384),(4096,7168),(24576,1536),(2112,7168)}; A, B as prefill")
    if name == "prefill_quant":
        # the prefill shapes whose N is a whole number of 128-wide groups (an
        # output quantized 1x128 is the next GEMM's A, whose K must be)
        return dict(name=name, kind="dense", m=inputs.PREFILL_M,
                    nk=[nk for nk in inputs.PREFILL_NK if nk[0] % 128 == 0],
                    seeds=inputs.PREFILL_SEEDS, bound="tensor", quant_out=True,
                    desc="dense NT prefill with the output quantized 1x128 in the epilogue "
                         "(E4M3 codes + FP32 scales), M=4096, (N,K) in "
                         "{(7168,16384),(4096,7168),(24576,1536)}; A, B and scales as prefill")
    if name == "kgrouped_tn":
        return dict(name=name, kind="kgrouped", bound="tensor", tn=True, **inputs.K_GROUPED,
                    desc="k-grouped contiguous TN (MoE weight gradient, operands stored "
                         "token-major: A [K, M], B [K, N]), G=8, M=4096 N=7168, 32768 "
                         "tokens multinomial over experts along K, segments padded to 128; "
                         "1x128-along-K FP32 scales on both, FP32 D[g] out")
    if name == "kgrouped":
        return dict(name=name, kind="kgrouped", bound="tensor", **inputs.K_GROUPED,
                    desc="k-grouped contiguous (MoE weight gradient), G=8, M=4096 N=7168, "
                         "32768 tokens multinomial over experts along K, segments padded "
                         "to 128; A~N(0,1) with 0.1% x50 outliers, B~N(0,1); 1x128 FP32 "
                         "scales on both, FP32 D[g] out")
    raise SystemExit(f"unknown workload {name}")


def peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                    source="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """Samples nvidia-smi every 50 ms; ``summary`` keeps the samples taken
    between ``mark_start`` and ``mark_stop`` (the timed region)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines: list[tuple[float, str]] = []
        self.t0 = self.t1 = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)  # let the first samples arrive
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark_start(self):
        self.t0 = time.time()

    def mark_stop(self):
        self.t1 = time.time()

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, ln in self.lines:
            if self.t0 is not None and not (self.t0 <= ts <= (self.t1 or ts) + 0.1):
                continue
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = max(mx, float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- device data
class DenseData:
    def __init__(self, spec, device):
        import torch
        import moe_grouped_gemm_act_b200 as dg
        self.dg = dg
        m = spec["m"]
        self.m = m
        self.acc = bool(spec.get("acc"))
        self.quant_out = bool(spec.get("quant_out"))
        # UE8M0: power-of-two scales packed for the block-scaled MMA (B's once,
        # A's every step after the quantizer)
        self.ue8m0 = bool(spec.get("ue8m0"))
        self.pow2 = bool(spec.get("pow2"))
        self.shapes = []
        gen = torch.Generator(device=device)
        for n, k in spec["nk"]:
            x = inputs.activations(m, k, seed=spec["seeds"]["seed_a"] + k, outliers=True)
            w = inputs.weights((n, k), seed=spec["seeds"]["seed_b"] + n + k)
            a32 = torch.from_numpy(x).to(device)
            qb, sfb = dg.dg_quantize_128x128(torch.from_numpy(w).to(device), pow2=self.pow2)
            ld = dg.dg_get_tma_aligned_size(m, 4)
            qa = torch.empty((m, k), dtype=torch.uint8, device=device)
            sfa = torch.empty((k // 128, ld), dtype=torch.float32, device=device)
            if self.quant_out:   # E4M3 codes and MN-major 1x128 scales of D
                d = (torch.empty((m, n), dtype=torch.uint8, device=device),
                     torch.empty((n // 128, ld), dtype=torch.float32, device=device))
            else:
                d = torch.empty((m, n), dtype=torch.bfloat16, device=device)
            wsb = dg.dg_fp8_gemm_nt_workspace_size(m, n, k)
            ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=device) if wsb else None
            c = None
            if self.acc:  # D = C + A B^T: a seeded FP32 C per shape
                gen.manual_seed(spec["seeds"]["seed_a"] + 7 * k + n)
                c = torch.randn((m, n), generator=gen, device=device, dtype=torch.float32) * 4
            pb = dg.dg_pack_ue8m0_128x128(sfb, n) if self.ue8m0 else None
            pa = dg.dg_pack_ue8m0(sfa.zero_(), m) if self.ue8m0 else None
            self.shapes.append(dict(n=n, k=k, a32=a32, qb=qb, sfb=sfb, qa=qa, sfa=sfa, d=d,
                                    ws=ws, x_host=x, w_host=w, c=c, pa=pa, pb=pb))
        torch.cuda.synchronize()

    def flops(self) -> float:
        return sum(2.0 * self.m * s["n"] * s["k"] for s in self.shapes)

    def shape_bytes(self, s) -> float:
        """Algorithmic bytes of one shape's GEMM launch (A, alpha, B, beta, D,
        and C when accumulating)."""
        n, k = s["n"], s["k"]
        out = (self.m * n + 4 * self.m * (n // 128)) if getattr(self, "quant_out", False) \
            else 2 * self.m * n
        if getattr(self, "ue8m0", False):
            # packed words: 4 K groups per int32, per row of A and of B
            words = -(-(k // 128) // 4)
            return self.m * k + 4 * self.m * words + n * k + 4 * n * words + out
        tot = self.m * k + 4 * self.m * (k // 128) + n * k + \
            4 * (-(-n // 128)) * (k // 128) + out
        if self.acc:
            tot += 4 * self.m * n  # C
        return tot

    def gemm_bytes(self) -> float:
        """Algorithmic bytes of the GEMM launches of one step."""
        return sum(self.shape_bytes(s) for s in self.shapes)

    def gemm(self, s):
        if self.ue8m0:
            self.dg.dg_fp8_gemm_nt_ue8m0(s["qa"], s["pa"], s["qb"], s["pb"], s["d"])
        elif self.quant_out:
            self.dg.dg_fp8_gemm_nt_quantize(s["qa"], s["sfa"], s["qb"], s["sfb"], dq=s["d"][0],
                                            sfd=s["d"][1])
        elif self.acc:
            self.dg.dg_fp8_gemm_nt_accumulate(s["qa"], s["sfa"], s["qb"], s["sfb"], s["c"], s["d"],
                                              workspace=s["ws"])
        else:
            self.dg.dg_fp8_gemm_nt(s["qa"], s["sfa"], s["qb"], s["sfb"], s["d"],
                                   workspace=s["ws"])

    def step(self):
        """One pass of the hot path: for every shape, quantize A, then GEMM."""
        for s in self.shapes:
            self.dg.dg_quantize_1x128(s["a32"], pow2=self.pow2, q=s["qa"], sf=s["sfa"])
            if self.ue8m0:
                self.dg.dg_pack_ue8m0(s["sfa"], self.m, packed=s["pa"])
            self.gemm(s)

    def capture(self):
        """CUDA graphs of one step and of each shape's GEMM alone.  The
        library is called once eagerly first (its per-device set-up must not
        happen inside a capture); replaying removes host launch overhead, as a
        serving loop would."""
        import torch
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self.step()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        self.step_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.step_graph):
            self.step()
        self.gemm_graphs = []
        for s in self.shapes:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self.gemm(s)
            self.gemm_graphs.append(g)
        # the step's GEMM launches alone, back to back as in the step
        self.gemm_step_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.gemm_step_graph):
            for s in self.shapes:
                self.gemm(s)
        torch.cuda.synchronize()

    def launches_per_step(self) -> int:
        # this library's kernels per step: one quantizer and one GEMM per
        # shape, plus the UE8M0 form's scale packing (a split-K call also
        # enqueues a runtime memset, not counted)
        return (3 if self.ue8m0 else 2) * len(self.shapes)

    def input_bytes(self) -> float:
        """Bytes of inputs a step streams (FP32 activations and FP8 B)."""
        return sum(s["a32"].numel() * 4 + s["qb"].numel() for s in self.shapes)

    # end-to-end through the public API from pinned host buffers
    def make_host(self):
        import torch
        self.host = []
        for s in self.shapes:
            self.host.append(dict(
                a=torch.from_numpy(s["x_host"]).pin_memory(),
                qb=s["qb"].cpu().pin_memory(), sfb=s["sfb"].cpu().pin_memory(),
                c=None if s["c"] is None else s["c"].cpu().pin_memory(),
                d=tuple(torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in s["d"])
                if self.quant_out else
                torch.empty(s["d"].shape, dtype=torch.bfloat16).pin_memory()))
        self.h2d = sum(h["a"].numel() * 4 + h["qb"].numel() + h["sfb"].numel() * 4 +
                       (0 if h["c"] is None else h["c"].numel() * 4) for h in self.host)
        self.d2h = sum((sum(t.numel() * t.element_size() for t in h["d"]) if self.quant_out
                        else h["d"].numel() * 2) for h in self.host)

    def e2e_step(self, device):
        dg = self.dg
        for s, h in zip(self.shapes, self.host):
            a = h["a"].to(device, non_blocking=True)
            qb = h["qb"].to(device, non_blocking=True)
            sfb = h["sfb"].to(device, non_blocking=True)
            qa, sfa = dg.dg_quantize_1x128(a, pow2=self.pow2)
            if self.ue8m0:
                pa = dg.dg_pack_ue8m0(sfa, qa.shape[0])
                pb = dg.dg_pack_ue8m0_128x128(sfb, qb.shape[0])
                dg.dg_fp8_gemm_nt_ue8m0(qa, pa, qb, pb, s["d"])
                h["d"].copy_(s["d"], non_blocking=True)
                continue
            if self.quant_out:
                dg.dg_fp8_gemm_nt_quantize(qa, sfa, qb, sfb, dq=s["d"][0], sfd=s["d"][1])
                for dst, src in zip(h["d"], s["d"]):
                    dst.copy_(src, non_blocking=True)
                continue
            if h["c"] is not None:
                c = h["c"].to(device, non_blocking=True)
                dg.dg_fp8_gemm_nt_accumulate(qa, sfa, qb, sfb, c, s["d"], workspace=s["ws"])
            else:
                dg.dg_fp8_gemm_nt(qa, sfa, qb, sfb, s["d"], workspace=s["ws"])
            h["d"].copy_(s["d"], non_blocking=True)


class GroupedData(DenseData):
    """The MoE layouts: one grouped GEMM per step (quantize all activation
    rows of the fixed buffer, then the contiguous or masked GEMM).  FLOPs
    and algorithmic bytes count valid rows and active experts only."""

    def __init__(self, spec, device):
        import torch
        import moe_grouped_gemm_act_b200 as dg
        self.dg = dg
        self.kind = spec["kind"]
        G, n, k = spec["groups"], spec["n"], spec["k"]
        if self.kind == "masked":
            m_max = spec["m_max"]
            counts = inputs.masked_counts(G, m_max, seed=spec["seed"])
            x = inputs.activations(G * m_max, k, seed=spec["seed"] + 1,
                                   outliers=True).reshape(G, m_max, k)
            index = torch.from_numpy(counts).to(device)
            rows_valid = int(counts.sum())
            active = int((counts > 0).sum())
            d_shape = (G, m_max, n)
            self.rows_total = G * m_max
        else:
            lay = inputs.contiguous_layout(spec["tokens"], G, seed=spec["seed"])
            x = inputs.activations(lay.m_total, k, seed=spec["seed"] + 1, outliers=True)
            x[lay.m_indices < 0] = 0.0   # padding rows (their content is never read back)
            index = torch.from_numpy(lay.m_indices).to(device)
            rows_valid = int((lay.m_indices >= 0).sum())
            active = int(len(np.unique(lay.m_indices[lay.m_indices >= 0])))
            d_shape = (lay.m_total, n)
            self.rows_total = lay.m_total
        w = inputs.weights((G, n, k), seed=spec["seed"] + 2)
        a32 = torch.from_numpy(x).to(device)
        self.pow2 = bool(spec.get("pow2"))
        qb, sfb = dg.dg_quantize_128x128(torch.from_numpy(w).to(device), pow2=self.pow2)
        # host inputs for the oracle's timed sample (a few experts' rows and
        # the first columns of their weights)
        self.sample_src = GroupedOracleSample.source(spec, x, w, index.cpu().numpy())
        del w
        qa, sfa = dg.dg_quantize_1x128(a32, pow2=self.pow2)
        # UE8M0: B's block scales packed once (weights); A's are packed
        # every step after the quantizer
        self.ue8m0 = bool(spec.get("ue8m0"))
        self.pb = dg.dg_pack_ue8m0_128x128(sfb, n) if self.ue8m0 else None
        self.pa = dg.dg_pack_ue8m0(sfa, qa.shape[-2]) if self.ue8m0 else None
        d = torch.empty(d_shape, dtype=torch.bfloat16, device=device)
        self.m = rows_valid
        self.active = active
        self.groups = G
        self.shapes = [dict(n=n, k=k, a32=a32, qb=qb, sfb=sfb, qa=qa, sfa=sfa, d=d, ws=None,
                            index=index, x_host=x)]
        torch.cuda.synchronize()

    def shape_bytes(self, s) -> float:
        return self.gemm_bytes()

    def gemm_bytes(self) -> float:
        s = self.shapes[0]
        n, k, v = s["n"], s["k"], self.m
        if getattr(self, "ue8m0", False):
            # packed words: 4 K groups per int32, per row of A and of B
            words = -(-(k // 128) // 4)
            return (v * k + 4 * v * words + self.active * (n * k + 4 * n * words)
                    + 2 * v * n + 4 * s["index"].numel())
        return (v * k + 4 * v * (k // 128) + self.active * (n * k + 4 * (-(-n // 128)) * (k // 128))
                + 2 * v * n + 4 * s["index"].numel())

    def gemm(self, s):
        if self.ue8m0:
            self.dg.dg_m_grouped_fp8_gemm_nt_masked_ue8m0(s["qa"], self.pa, s["qb"], self.pb,
                                                          s["d"], s["index"])
        elif self.kind == "masked":
            self.dg.dg_m_grouped_fp8_gemm_nt_masked(s["qa"], s["sfa"], s["qb"], s["sfb"], s["d"],
                                                    s["index"])
        else:
            self.dg.dg_m_grouped_fp8_gemm_nt_contiguous(s["qa"], s["sfa"], s["qb"], s["sfb"],
                                                        s["d"], s["index"])

    def step(self):
        """One pass of the hot path: quantize the activations (and, for the
        UE8M0 form, pack their scales), then GEMM."""
        s = self.shapes[0]
        self.dg.dg_quantize_1x128(s["a32"], pow2=self.pow2, q=s["qa"], sf=s["sfa"])
        if self.ue8m0:
            self.dg.dg_pack_ue8m0(s["sfa"], s["qa"].shape[-2], packed=self.pa)
        self.gemm(s)

    def launches_per_step(self) -> int:
        return 3 if self.ue8m0 else 2

    def make_host(self):
        s = self.shapes[0]
        self.host = [dict(a=torch_pin(s["x_host"]), qb=s["qb"].cpu().pin_memory(),
                          sfb=s["sfb"].cpu().pin_memory(), index=s["index"].cpu().pin_memory(),
                          d=torch_empty_pinned(s["d"]))]
        h = self.host[0]
        self.h2d = (h["a"].numel() * 4 + h["qb"].numel() + h["sfb"].numel() * 4
                    + h["index"].numel() * 4)
        self.d2h = h["d"].numel() * 2

    def e2e_step(self, device):
        s, h = self.shapes[0], self.host[0]
        a = h["a"].to(device, non_blocking=True)
        qb = h["qb"].to(device, non_blocking=True)
        sfb = h["sfb"].to(device, non_blocking=True)
        index = h["index"].to(device, non_blocking=True)
        qa, sfa = self.dg.dg_quantize_1x128(a, pow2=self.pow2)
        if self.ue8m0:
            pa = self.dg.dg_pack_ue8m0(sfa, qa.shape[-2])
            pb = self.dg.dg_pack_ue8m0_128x128(sfb, qb.shape[-2])
            self.dg.dg_m_grouped_fp8_gemm_nt_masked_ue8m0(qa, pa, qb, pb, s["d"], index)
            h["d"].copy_(s["d"], non_blocking=True)
            return
        if self.kind == "masked":
            self.dg.dg_m_grouped_fp8_gemm_nt_masked(qa, sfa, qb, sfb, s["d"], index)
        else:
            self.dg.dg_m_grouped_fp8_gemm_nt_contiguous(qa, sfa, qb, sfb, s["d"], index)
        h["d"].copy_(s["d"], non_blocking=True)


class KGroupedData(DenseData):
    """The MoE weight gradient: one step quantizes the activation gradient A
    [M, K] and the activations B [N, K] (1x128 along the token axis K), then
    runs the k-grouped GEMM into FP32 D [G, M, N].  FLOPs count the valid
    tokens (not the padding of the segments).  The TN form stores both
    operands token-major (A [K, M], B [K, N]), quantizes them with the
    K-outermost quantizer and runs the TN k-grouped GEMM."""

    def __init__(self, spec, device):
        import torch
        import moe_grouped_gemm_act_b200 as dg
        self.dg = dg
        a, b, lay = KGroupedOracleSample.generate(spec)
        self.sample_src = KGroupedOracleSample.source(a, b)
        G, m, n, k = spec["groups"], spec["m"], spec["n"], lay.k_total
        self.tn = bool(spec.get("tn"))
        if self.tn:   # token-major storage (set-up, untimed)
            a32 = torch.from_numpy(np.ascontiguousarray(a.T)).to(device)
            b32 = torch.from_numpy(np.ascontiguousarray(b.T)).to(device)
        else:
            a32 = torch.from_numpy(a).to(device)
            b32 = torch.from_numpy(b).to(device)
        qa = torch.empty(tuple(a32.shape), dtype=torch.uint8, device=device)
        sfa = torch.empty((k // 128, dg.dg_get_tma_aligned_size(m, 4)), dtype=torch.float32,
                          device=device)
        qb = torch.empty(tuple(b32.shape), dtype=torch.uint8, device=device)
        sfb = torch.empty((k // 128, dg.dg_get_tma_aligned_size(n, 4)), dtype=torch.float32,
                          device=device)
        d = torch.empty((G, m, n), dtype=torch.float32, device=device)
        ks = torch.from_numpy(lay.k_sizes).to(device)
        self.m = m
        self.groups = G
        self.k_total = k
        tokens = int(lay.counts.sum())
        self.shapes = [dict(n=n, k=tokens, a32=a32, b32=b32, qa=qa, sfa=sfa, qb=qb, sfb=sfb,
                            d=d, k_sizes=ks, x_host=a.T if self.tn else a,
                            b_host=b.T if self.tn else b, ws=None)]
        torch.cuda.synchronize()

    def shape_bytes(self, s) -> float:
        return self.gemm_bytes()

    def gemm_bytes(self) -> float:
        s = self.shapes[0]
        m, n, k = self.m, s["n"], self.k_total
        return (m + n) * k + 4 * (m + n) * (k // 128) + 4 * self.groups * m * n + 4 * self.groups

    def gemm(self, s):
        f = (self.dg.dg_k_grouped_fp8_gemm_tn_contiguous if self.tn
             else self.dg.dg_k_grouped_fp8_gemm_nt_contiguous)
        f(s["qa"], s["sfa"], s["qb"], s["sfb"], s["d"], s["k_sizes"])

    def quantize(self, x, q=None, sf=None):
        if self.tn:
            return self.dg.dg_quantize_128x1(x, q=q, sf=sf)
        return self.dg.dg_quantize_1x128(x, q=q, sf=sf)

    def step(self):
        s = self.shapes[0]
        self.quantize(s["a32"], q=s["qa"], sf=s["sfa"])
        self.quantize(s["b32"], q=s["qb"], sf=s["sfb"])
        self.gemm(s)

    def launches_per_step(self) -> int:
        return 3

    def input_bytes(self) -> float:
        s = self.shapes[0]
        return (s["a32"].numel() + s["b32"].numel()) * 4

    def make_host(self):
        s = self.shapes[0]
        self.host = [dict(a=torch_pin(s["x_host"]), b=torch_pin(s["b_host"]),
                          k_sizes=s["k_sizes"].cpu().pin_memory(),
                          d=torch_empty_pinned(s["d"]))]
        h = self.host[0]
        self.h2d = (h["a"].numel() + h["b"].numel() + h["k_sizes"].numel()) * 4
        self.d2h = h["d"].numel() * 4

    def e2e_step(self, device):
        s, h = self.shapes[0], self.host[0]
        a = h["a"].to(device, non_blocking=True)
        b = h["b"].to(device, non_blocking=True)
        ks = h["k_sizes"].to(device, non_blocking=True)
        qa, sfa = self.quantize(a)
        qb, sfb = self.quantize(b)
        f = (self.dg.dg_k_grouped_fp8_gemm_tn_contiguous if self.tn
             else self.dg.dg_k_grouped_fp8_gemm_nt_contiguous)
        f(qa, sfa, qb, sfb, s["d"], ks)
        h["d"].copy_(s["d"], non_blocking=True)


def per_shape_report(data, per_shape_ms, bound: str, peak: float) -> list:
    """Each shape's GEMM time when launched alone (its own graph: the launch
    latency the step hides is included), TFLOP/s and fraction of the roofline
    peak: TFLOP/s over the FP8 peak for tensor-bound work, algorithmic GB/s
    over the copy bandwidth for HBM-bound work."""
    out = []
    for s, ms in zip(data.shapes, per_shape_ms):
        secs = ms * 1e-3
        row = {"n": s["n"], "k": s["k"], "gemm_us_alone": 1e3 * ms,
               "tflops": 2.0 * data.m * s["n"] * s["k"] / secs / 1e12}
        if bound == "tensor":
            row["frac"] = row["tflops"] / peak
        else:
            row["gbs"] = data.shape_bytes(s) / secs / 1e9
            row["frac"] = row["gbs"] / peak
        out.append(row)
    return out


def torch_pin(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).pin_memory()


def torch_empty_pinned(t):
    import torch
    return torch.empty(t.shape, dtype=t.dtype).pin_memory()


class OracleSample:
    """The CPU oracle on a bounded sample of the workload: for every (N, K)
    pair, the first ``rows`` rows of A and the first ``cols`` columns of D over
    the full K.  One run = quantize the sampled A rows (1x128) and compute the
    sampled block of every GEMM.  Weights are quantized once beforehand, as on
    the GPU (the first 128-aligned rows of B quantize exactly as in full)."""

    def __init__(self, spec, rows: int, cols: int):
        from oracle import quant as oq
        self.prepared = []
        self.acc = bool(spec.get("acc"))
        self.quant_out = bool(spec.get("quant_out"))
        self.pow2 = bool(spec.get("pow2"))
        g = np.random.default_rng(spec["seeds"]["seed_a"])
        for n, k in spec["nk"]:
            x = inputs.activations(spec["m"], k, seed=spec["seeds"]["seed_a"] + k,
                                   outliers=True)
            w = inputs.weights((n, k), seed=spec["seeds"]["seed_b"] + n + k)
            c = min(n, cols)
            qb, beta = oq.quantize_128x128(w[:c], pow2=self.pow2)
            cs = (g.standard_normal((rows, c)) * 4).astype(np.float32) if self.acc else None
            self.prepared.append((x[:rows].copy(), qb, beta, c, k, cs))
        self.desc = (f"{rows} rows of A x first {cols} columns of D per (N,K) pair, "
                     f"full K" + (", D = C + A B^T" if self.acc else "") +
                     (", D quantized 1x128" if self.quant_out else "") +
                     (", power-of-two scales" if self.pow2 else ""))

    def run(self) -> tuple[float, float]:
        """Returns (seconds, FLOPs) of one pass."""
        from oracle import gemm as og, quant as oq
        t0 = time.perf_counter()
        flops = 0.0
        for xs, qb, beta, c, k, cs in self.prepared:
            qa, alpha = oq.quantize_1x128(xs, pow2=self.pow2)
            if self.quant_out:
                from oracle import bf16 as ob
                d = ob.from_bits(og.fp8_gemm_nt(qa, alpha, qb, beta)).astype(np.float32)
                oq.quantize_1x128(d)
            elif cs is None:
                og.fp8_gemm_nt(qa, alpha, qb, beta)
            else:
                og.fp8_gemm_nt_accumulate(qa, alpha, qb, beta, cs)
            flops += 2.0 * xs.shape[0] * c * k
        return time.perf_counter() - t0, flops


class GroupedOracleSample:
    """The CPU oracle on a bounded sample of a grouped workload: the first
    ``experts`` experts holding rows, up to ``rows`` of each expert's rows and
    the first ``cols`` columns of D over the full K.  One run = quantize the
    sampled A rows (1x128) and run the oracle's masked or contiguous GEMM on
    that sub-problem (weights quantized once beforehand, as on the GPU)."""

    EXPERTS = 2

    @staticmethod
    def source(spec, x, w, index):
        """The slices the sample needs, from the workload's host inputs."""
        cols = 1024
        picked = []
        for e in range(spec["groups"]):
            if spec["kind"] == "masked":
                rows = x[e, :int(index[e])]
            else:
                rows = x[index == e]
            if len(rows):
                picked.append((rows[:64].copy(), w[e, :cols].copy()))
            if len(picked) == GroupedOracleSample.EXPERTS:
                break
        return picked

    def __init__(self, spec, rows: int, cols: int, src=None):
        from oracle import quant as oq
        self.kind = spec["kind"]
        self.k = spec["k"]
        self.pow2 = bool(spec.get("pow2"))
        if src is None:
            src = self.source(spec, *self._generate(spec))
        self.prepared = []
        for xr, wc in src:
            xr, wc = xr[:rows], wc[:cols]
            qb, beta = oq.quantize_128x128(wc, pow2=self.pow2)
            self.prepared.append((xr, qb, beta))
        c = min(cols, spec["n"])
        self.desc = (f"{rows} rows of each of the first {len(self.prepared)} experts with rows "
                     f"x first {c} columns of D, full K ({self.kind} oracle)")

    @staticmethod
    def _generate(spec):
        G, k = spec["groups"], spec["k"]
        w = inputs.weights((G, spec["n"], k), seed=spec["seed"] + 2)
        if spec["kind"] == "masked":
            counts = inputs.masked_counts(G, spec["m_max"], seed=spec["seed"])
            x = inputs.activations(G * spec["m_max"], k, seed=spec["seed"] + 1,
                                   outliers=True).reshape(G, spec["m_max"], k)
            return x, w, counts
        lay = inputs.contiguous_layout(spec["tokens"], G, seed=spec["seed"])
        x = inputs.activations(lay.m_total, k, seed=spec["seed"] + 1, outliers=True)
        return x, w, lay.m_indices

    def run(self) -> tuple[float, float]:
        """Returns (seconds, FLOPs) of one pass."""
        from oracle import gemm as og, quant as oq
        t0 = time.perf_counter()
        qas = [oq.quantize_1x128(xr, pow2=self.pow2) for xr, _, _ in self.prepared]
        qb = np.stack([q for _, q, _ in self.prepared])
        beta = np.stack([b for _, _, b in self.prepared])
        n_rows = [len(xr) for xr, _, _ in self.prepared]
        c = qb.shape[1]
        if self.kind == "masked":
            m = max(n_rows)
            qa = np.zeros((len(qas), m, self.k), np.uint8)
            alpha = np.zeros((len(qas), m, self.k // 128), np.float32)
            for e, (q, a) in enumerate(qas):
                qa[e, :len(q)], alpha[e, :len(a)] = q, a
            og.m_grouped_masked(qa, alpha, qb, beta, np.array(n_rows, np.int32),
                                np.zeros((len(qas), m, c), np.uint16))
        else:
            qa = np.concatenate([q for q, _ in qas])
            alpha = np.concatenate([a for _, a in qas])
            idx = np.concatenate([np.full(r, e, np.int32) for e, r in enumerate(n_rows)])
            og.m_grouped_contiguous(qa, alpha, qb, beta, idx,
                                    np.zeros((len(idx), c), np.uint16))
        flops = 2.0 * sum(n_rows) * c * self.k
        return time.perf_counter() - t0, flops


class KGroupedOracleSample:
    """The CPU oracle on a bounded sample of the weight gradient: the first
    ``rows`` rows of A and ``cols`` rows of B (rows and columns of every
    D[g]) over the full K.  One run = quantize both samples (1x128) and run
    the oracle's k-grouped GEMM; both operands are quantized per step on the
    GPU too."""

    @staticmethod
    def generate(spec):
        """The workload's host inputs: A [M, K], B [N, K] with zeros on the
        padding tokens of every segment, and the layout."""
        lay = inputs.k_grouped_layout(spec["tokens"], spec["groups"], seed=spec["seed"])
        a = inputs.activations(spec["m"], lay.k_total, seed=spec["seed"] + 1, outliers=True)
        b = inputs.activations(spec["n"], lay.k_total, seed=spec["seed"] + 2)
        valid = np.zeros(lay.k_total, bool)
        start = 0
        for cnt, size in zip(lay.counts, lay.k_sizes):
            valid[start:start + int(cnt)] = True
            start += int(size)
        a[:, ~valid] = 0.0
        b[:, ~valid] = 0.0
        return a, b, lay

    @staticmethod
    def source(a, b, rows: int = 64, cols: int = 1024):
        return a[:rows].copy(), b[:cols].copy()

    def __init__(self, spec, rows: int, cols: int, src=None):
        lay = inputs.k_grouped_layout(spec["tokens"], spec["groups"], seed=spec["seed"])
        if src is None:
            a, b, _ = self.generate(spec)
            src = self.source(a, b, rows, cols)
        self.a, self.b = src[0][:rows], src[1][:cols]
        self.k_sizes = lay.k_sizes
        self.tokens = int(lay.counts.sum())
        self.desc = (f"{len(self.a)} rows x {len(self.b)} columns of every D[g], full K "
                     f"({self.tokens} tokens, k-grouped oracle)")

    def run(self) -> tuple[float, float]:
        """Returns (seconds, FLOPs) of one pass."""
        from oracle import gemm as og, quant as oq
        t0 = time.perf_counter()
        qa, alpha = oq.quantize_1x128(self.a)
        qb, beta = oq.quantize_1x128(self.b)
        og.k_grouped_contiguous_f64(qa, alpha, qb, beta, self.k_sizes)
        return time.perf_counter() - t0, 2.0 * len(self.a) * len(self.b) * self.tokens


def make_sampler(spec, rows: int, cols: int, data=None):
    """The oracle sample of a workload (from the GPU arm's host inputs when
    ``data`` is given)."""
    if spec["kind"] == "dense":
        return OracleSample(spec, rows, cols)
    src = None if data is None else data.sample_src
    if spec["kind"] == "kgrouped":
        return KGroupedOracleSample(spec, rows, cols, src=src)
    return GroupedOracleSample(spec, rows, cols, src=src)


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        if info:
            return max(int(i.get("num_threads", 1)) for i in info)
    except Exception:
        pass
    return os.cpu_count() or 1


# ---------------------------------------------------------------- arms
def run_reference(args, rank: int) -> None:
    """The oracle arm: rank 0 times the CPU oracle on bounded samples."""
    if rank != 0:
        return
    # the headline workload when all are measured
    spec = workload_spec("prefill" if args.workload == "all" else args.workload)
    sampler = make_sampler(spec, args.ref_rows, args.ref_cols)
    for _ in range(args.warmup):
        sampler.run()
    secs, flops = 0.0, 0.0
    for _ in range(args.steps):
        s, f = sampler.run()
        secs += s
        flops += f
    value = flops / secs / 1e12
    cores = blas_threads()
    sample = sampler.desc
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": spec["desc"], "sample": sample},
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


def max_over_ranks(values, world: int, device) -> list:
    """Element-wise maximum of per-rank timings over all ranks (every rank
    gets the result).  With one rank, the values themselves."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(work_per_step: float, steps: int, world: int, ms: float) -> float:
    """Whole-job rate: the work all ranks did (each rank runs the same steps
    on its own replica) over the slowest rank's time, per second."""
    return work_per_step * steps * world / (ms * 1e-3)


ALL_WORKLOADS = ["prefill", "decode64", "decode128", "contiguous", "masked", "masked_pow2",
                 "masked_ue8m0", "kgrouped", "kgrouped_tn", "prefill_acc", "prefill_quant",
                 "prefill_ue8m0"]


def measure_workload(name: str, args, rank: int, world: int, device, cpu_secs: float) -> dict:
    """Times one workload on this rank and returns its bench fields (rank 0's
    are the ones printed): whole-step throughput from CUDA-graph replays, the
    GEMM kernel alone against its roofline, the end-to-end rate from pinned
    host buffers, and the oracle on a bounded sample of the same work (rank 0,
    N = 1 only, about ``cpu_secs`` of CPU time)."""
    import torch
    import torch.distributed as dist

    spec = workload_spec(name)
    data = {"dense": DenseData, "kgrouped": KGroupedData}.get(spec["kind"], GroupedData)(
        spec, device)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    # ------------------------------------------------ device-resident timing
    # Each step replays a CUDA graph of the whole step (quantize + GEMM for
    # every shape); events on the replay stream bracket exactly K steps.
    data.capture()
    nshape = len(data.shapes)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(device.index or 0) as clocks:
        for _ in range(args.warmup):
            data.step_graph.replay()
        barrier()
        clocks.mark_start()
        start.record()
        for _ in range(args.steps):
            data.step_graph.replay()
        stop.record()
        torch.cuda.synchronize()
        clocks.mark_stop()
    barrier()
    total_ms = start.elapsed_time(stop)
    # The dominant kernel, launched as in the step: a graph of the step's GEMM
    # launches without the quantizers, back to back (programmatic dependent
    # launch lets each one's set-up overlap the previous one's tail, as it
    # does in the step), K replays between one event pair.  Each pass streams
    # several hundred MB of operands and outputs (> L2).
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(args.warmup):
        data.gemm_step_graph.replay()
    torch.cuda.synchronize()
    g0.record()
    for _ in range(args.steps):
        data.gemm_step_graph.replay()
    g1.record()
    torch.cuda.synchronize()
    gemm_ms = g0.elapsed_time(g1)
    # Per shape, each GEMM timed alone (its own graph and event pair, shapes
    # round-robin so that each launch finds the other shapes' operands in L2):
    # includes the launch latency the step hides, reported per shape only.
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)] for _ in range(nshape)]
    for g in data.gemm_graphs:
        g.replay()
    for i in range(args.steps):
        for j, g in enumerate(data.gemm_graphs):
            ev[j][i][0].record()
            g.replay()
            ev[j][i][1].record()
    torch.cuda.synchronize()
    per_shape_ms = [statistics.mean(a.elapsed_time(b) for a, b in ev[j]) for j in range(nshape)]

    # ------------------------------------------------ end-to-end timing
    data.make_host()
    for _ in range(max(1, args.warmup // 2)):
        data.e2e_step(device)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = max(3, min(args.steps, 25))  # PCIe-bound; fewer steps suffice
    e0.record()
    for _ in range(e2e_steps):
        data.e2e_step(device)
    e1.record()
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e0.elapsed_time(e1) * args.steps / e2e_steps

    # ------------------------------------------------ max over ranks
    total_ms, e2e_ms, gemm_total_ms = max_over_ranks([total_ms, e2e_ms, gemm_ms], world, device)

    flops_step = data.flops()
    value = job_throughput(flops_step, args.steps, world, total_ms) / 1e12
    e2e = job_throughput(flops_step, args.steps, world, e2e_ms) / 1e12
    pk = peaks()
    # dominant kernel: the GEMM
    if spec["bound"] == "tensor":
        achieved = flops_step * args.steps / (gemm_total_ms * 1e-3) / 1e12
        peak = pk["bf16"] * FP8_OVER_BF16
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak,
                "peak_source": f"{pk['source']} bf16 burst x {FP8_OVER_BF16} (nominal FP8/BF16)"}
    else:
        achieved = data.gemm_bytes() * args.steps / (gemm_total_ms * 1e-3) / 1e9
        peak = pk["hbm"]
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "peak_source": f"{pk['source']} copy bandwidth"}
    roof["traffic"] = (args.traffic if args.traffic is not None and args.workload == name
                       else measured_traffic(name))
    roof["traffic_unit"] = "bytes per GEMM launch (ncu dram read + write)"
    per_shape = per_shape_report(data, per_shape_ms, spec["bound"], peak)

    cpu = None
    if rank == 0 and world == 1 and cpu_secs > 0:
        sampler = make_sampler(spec, args.ref_rows, args.ref_cols, data)
        sampler.run()
        secs, fl = 0.0, 0.0
        while secs < cpu_secs:
            s_, f_ = sampler.run()
            secs += s_
            fl += f_
        cpu = {"value": fl / secs / 1e12, "unit": "TFLOPS", "cores": blas_threads(),
               "kind": "oracle", "sample": f"{sampler.desc} ({secs:.1f} s on the host)"}
    out = {
        "workload": name, "desc": spec["desc"], "value": value, "unit": "TFLOPS",
        "ms_per_step": total_ms / args.steps,
        "config": {"workload": spec["desc"],
                   "valid_rows" if spec["kind"] in ("contiguous", "masked") else "m": data.m,
                   "nk": [[sh["n"], sh["k"]] for sh in data.shapes],
                   "l2": "not flushed: each step streams %.0f MB of inputs (> 126 MB L2)"
                         % (data.input_bytes() / 1e6),
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "per_shape": per_shape},
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e, "unit": "TFLOPS", "h2d_bytes_per_step": data.h2d,
                "d2h_bytes_per_step": data.d2h},
        "gpu_launches": data.launches_per_step() * args.steps,
        "clocks": clocks.summary(),
    }
    del data
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def run_gpu(args, rank: int, world: int, local_rank: int) -> None:
    import torch

    import moe_grouped_gemm_act_b200 as dg

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    dg.load_library()
    names = ALL_WORKLOADS if args.workload == "all" else [args.workload]
    cpu_secs = 0.0 if args.no_cpu_baseline else 10.0
    results = []
    for i, name in enumerate(names):
        # the headline workload gets about 10 s of oracle time, the others 3 s
        results.append(measure_workload(name, args, rank, world, device,
                                        cpu_secs if i == 0 else min(cpu_secs, 3.0)))
    if rank != 0:
        return
    head = results[0]
    line = {
        "metric": METRIC, "value": head["value"], "unit": "TFLOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3", "data": "synthetic",
        "config": dict(head["config"]),
        "roofline": head["roofline"],
        "cpu_baseline": head["cpu_baseline"],
        "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"],
        "clocks": head["clocks"],
    }
    if len(results) > 1:
        # every other workload of the metric, each with its own roofline,
        # end-to-end rate, oracle sample and clocks
        line["config"]["workloads"] = results[1:]
    print(json.dumps(line))


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="all", choices=["all", *ALL_WORKLOADS],
                    help="one workload, or all of them (the default: the line's value is the "
                         "prefill workload's, the others are listed under config.workloads)")
    ap.add_argument("--impl", default="dg", choices=["dg", "reference"])
    ap.add_argument("--ref-rows", type=int, default=16,
                    help="rows of A per shape in the oracle's timed sample")
    ap.add_argument("--ref-cols", type=int, default=1024,
                    help="columns of D per shape in the oracle's timed sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--traffic", type=float, default=None,
                    help="ncu DRAM bytes per GEMM launch, when measured on the current sources")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        run_gpu(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
