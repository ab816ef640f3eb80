"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module only draws random numbers and builds index arrays; it contains no
step of the method (no scaling, rounding or GEMM arithmetic), so the oracle and
the CUDA path can both be fed from it without sharing any of the method's code.

Value distributions follow the workloads the library is measured on (the
DeepSeek-V3/R1 inference shapes named by the DeepGEMM launch article, which no
public dataset stands in for):

* activations A ~ N(0, 1), optionally with outliers: each entry independently
  multiplied by 50 with probability 0.001;
* weights B ~ N(0, 0.02);
* contiguous MoE layout: token counts ~ Multinomial(T, uniform over G experts),
  each expert segment padded up to a multiple of 128 rows, a per-row int32
  expert index with -1 on padding rows;
* masked MoE layout: masked_m[g] ~ Uniform{0, ..., M_max}.
* k-grouped MoE layout (weight gradient): token counts ~ Multinomial(T,
  uniform over G experts) along K, each segment padded up to a multiple of
  128 tokens.

All generators are numpy PCG64 streams with explicit seeds.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

ALIGN_M = 128


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def activations(m: int, k: int, seed: int, outliers: bool = False) -> np.ndarray:
    """float32 [m, k] ~ N(0, 1); with ``outliers`` each entry is multiplied by
    50 with probability 0.001."""
    g = rng(seed)
    x = g.standard_normal((m, k), dtype=np.float32)
    if outliers:
        hit = g.random((m, k), dtype=np.float32) < np.float32(0.001)
        x[hit] *= np.float32(50.0)
    return x


def weights(shape, seed: int, std: float = 0.02) -> np.ndarray:
    """float32 array of the given shape ~ N(0, std**2)."""
    g = rng(seed)
    return (g.standard_normal(shape, dtype=np.float32) * np.float32(std))


@dataclass
class ContiguousLayout:
    counts: np.ndarray      # int64 [G]: valid tokens per expert
    m_indices: np.ndarray   # int32 [M_total]: expert per row, -1 = padding
    m_total: int


def contiguous_layout(num_tokens: int, num_groups: int, seed: int,
                      align: int = ALIGN_M) -> ContiguousLayout:
    """Multinomial split of ``num_tokens`` over ``num_groups`` experts, each
    segment padded up to a multiple of ``align`` rows."""
    g = rng(seed)
    counts = g.multinomial(num_tokens, np.full(num_groups, 1.0 / num_groups))
    padded = [(-(-int(c) // align)) * align for c in counts]
    m_total = int(sum(padded))
    m_indices = np.full(m_total, -1, dtype=np.int32)
    row = 0
    for e, (c, p) in enumerate(zip(counts, padded)):
        m_indices[row:row + int(c)] = e
        row += p
    return ContiguousLayout(counts=np.asarray(counts), m_indices=m_indices,
                            m_total=m_total)


@dataclass
class KGroupedLayout:
    counts: np.ndarray      # int64 [G]: tokens per expert
    k_sizes: np.ndarray     # int32 [G]: K segment per expert, counts padded to 128
    k_total: int


def k_grouped_layout(num_tokens: int, num_groups: int, seed: int,
                     align: int = ALIGN_M) -> KGroupedLayout:
    """Multinomial split of ``num_tokens`` over ``num_groups`` experts along
    the K axis, each segment padded up to a multiple of ``align`` tokens (an
    expert with no tokens gets an empty segment).  The padding tokens are
    for the caller to fill with zeros."""
    g = rng(seed)
    counts = g.multinomial(num_tokens, np.full(num_groups, 1.0 / num_groups))
    k_sizes = np.array([(-(-int(c) // align)) * align for c in counts], dtype=np.int32)
    return KGroupedLayout(counts=np.asarray(counts), k_sizes=k_sizes,
                          k_total=int(k_sizes.sum()))


def masked_counts(num_groups: int, m_max: int, seed: int) -> np.ndarray:
    """int32 [G] ~ Uniform{0, ..., m_max}."""
    return rng(seed).integers(0, m_max + 1, size=num_groups).astype(np.int32)


# Workload table: the shapes the library is tested and measured on.
DENSE_PARITY = dict(m=128, n=256, k=512, seed_a=0, seed_b=1)
PREFILL_M = 4096
PREFILL_NK = [(7168, 16384), (4096, 7168), (24576, 1536), (2112, 7168)]
PREFILL_SEEDS = dict(seed_a=2, seed_b=3)
DECODE_M = [64, 128]
DECODE_SEEDS = dict(seed_a=4, seed_b=5)
CONTIGUOUS = dict(groups=8, n=4096, k=7168, tokens=32768, seed=6)
MASKED = dict(groups=32, m_max=256, n=7168, k=2048, seed=7)
# the weight gradient of the contiguous workload's GEMM: D[g] [4096, 7168] over
# each expert's tokens
K_GROUPED = dict(groups=8, m=4096, n=7168, tokens=32768, seed=8)
