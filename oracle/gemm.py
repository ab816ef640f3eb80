"""The fine-grained block-scaled FP8 NT GEMM and its MoE grouped forms.

Lesson 13, Fig. 13-1: for A [M, K] with 1x128 scales alpha and B with 128x128
scales beta,

    C[i, j] = sum_g alpha[i, g] * beta[g, floor(j / 128)]
                    * sum_{k < 128} A[i, 128 g + k] * B[128 g + k, j].

The page writes B as K x N; the exercise (Lesson 13 practice task) and the NT
convention (Deep dive, section 3: ``fp8_gemm_nt`` computes A @ B.T) store it as
[N, K], which is what is used here: B[128 g + k, j] above is ``qb[j, 128 g + k]``.

The oracle follows the exercise's order: for each 128-wide K block, the block's
partial product of the decoded codes (a float64 matmul), times the outer
product of the block's scales, added into a float64 accumulator.  Then the
result is rounded once to BF16 (Lesson 13, Fig. 13-1: the epilogue only
converts and writes back).

Grouped forms (Lesson 13, Fig. 13-3 and the answer to Q3; Deep dive,
section 3, the grouped GEMM table):

* m-grouped contiguous: the tokens of all experts are concatenated along M;
  each expert segment is aligned to the M tile; a per-row expert index names
  the expert, -1 on padding rows; N and K are shared by all experts.
* m-grouped masked: A is [G, M_max, K]; masked_m[g] rows of expert g are
  valid; only those rows are computed.
* k-grouped contiguous (the MoE weight gradient): the groups split the K
  axis (tokens) instead of M; M and N are shared by all groups and every
  group has its own [M, N] output.

Rows that are not computed (padding, rows >= masked_m[g]) are left exactly as
they were in the output (the pages do not say; this is the reading taken);
the oracle copies the caller's initial output for them.
"""

from __future__ import annotations

import numpy as np

from . import bf16, e4m3

GROUP = 128


def fp8_gemm_nt_f64(qa: np.ndarray, alpha: np.ndarray,
                    qb: np.ndarray, beta: np.ndarray) -> np.ndarray:
    """float64 D [M, N] of the Fig. 13-1 formula.

    qa uint8 [M, K] E4M3 codes, alpha float32 [M, K/128];
    qb uint8 [N, K] E4M3 codes, beta float32 [ceil(N/128), K/128].
    """
    M, K = qa.shape
    N, Kb = qb.shape
    if K != Kb or K % GROUP:
        raise ValueError("K mismatch or K not a multiple of 128")
    kg = K // GROUP
    if alpha.shape != (M, kg) or beta.shape != (-(-N // GROUP), kg):
        raise ValueError("scale shapes do not match the 1x128 / 128x128 grids")
    n_block_of_col = np.arange(N) // GROUP
    a_vals = e4m3.decode(qa)
    b_vals = e4m3.decode(qb)
    alpha64 = np.asarray(alpha, np.float64)
    beta64 = np.asarray(beta, np.float64)
    d = np.zeros((M, N), dtype=np.float64)
    for g in range(kg):
        ks = slice(g * GROUP, (g + 1) * GROUP)
        partial = a_vals[:, ks] @ b_vals[:, ks].T  # exact: small integers x 2^k
        scale = alpha64[:, g][:, None] * beta64[n_block_of_col, g][None, :]
        d += partial * scale
    return d


def fp8_gemm_nt_rowscaled_f64(qa: np.ndarray, alpha: np.ndarray,
                              qb: np.ndarray, beta_rows: np.ndarray) -> np.ndarray:
    """float64 D [M, N] of the Fig. 13-1 formula with one scale per row of B
    and 128-wide K group, beta_rows float [N, K/128], instead of one per
    128 x 128 block (the scaling Fig. 13-1 gives A, applied to both operands;
    a 128 x 128 block scale is the special case in which the 128 rows of a
    block share their values).  alpha float [M, K/128] as in fp8_gemm_nt_f64.
    Same order: per 128-wide K block, the block's partial product of the
    decoded codes times the outer product of the block's scales, added in
    float64."""
    M, K = qa.shape
    N, Kb = qb.shape
    if K != Kb or K % GROUP:
        raise ValueError("K mismatch or K not a multiple of 128")
    kg = K // GROUP
    if alpha.shape != (M, kg) or beta_rows.shape != (N, kg):
        raise ValueError("scale shapes do not match the 1x128 grids of A and B")
    a_vals = e4m3.decode(qa)
    b_vals = e4m3.decode(qb)
    alpha64 = np.asarray(alpha, np.float64)
    beta64 = np.asarray(beta_rows, np.float64)
    d = np.zeros((M, N), dtype=np.float64)
    for g in range(kg):
        ks = slice(g * GROUP, (g + 1) * GROUP)
        d += (a_vals[:, ks] @ b_vals[:, ks].T) * (alpha64[:, g][:, None] * beta64[:, g][None, :])
    return d


def fp8_gemm_nt_ue8m0_f64(qa, sfa_packed, qb, sfb_packed) -> np.ndarray:
    """float64 D [M, N] of the block-scaled GEMM whose scales are UE8M0 codes
    in the packed layout (Lesson 13, Fig. 13-1 text: newer versions take
    UE8M0 scales; Deep dive, section 3: four per 32-bit word, MN-major):
    sfa_packed int32 [ceil(K/512), ld_a >= M] for the rows of A,
    sfb_packed int32 [ceil(K/512), ld_b >= N] for the rows of B.  The codes
    are decoded to their powers of two and the formula is evaluated as in
    fp8_gemm_nt_rowscaled_f64."""
    from . import ue8m0
    M, K = qa.shape
    N = qb.shape[0]
    kg = K // GROUP
    alpha = ue8m0.unpack_1x128(sfa_packed, M, kg)
    beta_rows = ue8m0.unpack_1x128(sfb_packed, N, kg)
    return fp8_gemm_nt_rowscaled_f64(qa, alpha, qb, beta_rows)


def fp8_gemm_nt(qa, alpha, qb, beta) -> np.ndarray:
    """BF16 bit patterns (uint16 [M, N]) of the dense NT GEMM."""
    return bf16.to_bits(fp8_gemm_nt_f64(qa, alpha, qb, beta))


LAYOUTS = ("nt", "nn", "tn", "tt")


def fp8_gemm_f64(layout: str, qa_stored, alpha, qb_stored, beta) -> np.ndarray:
    """The Fig. 13-1 formula for the four operand layouts of the Deep dive,
    section 3 (D = A @ B.T for "nt"; the first letter says whether A is used
    as stored or transposed, the second whether B is).  Stored shapes:
    "nt" A [M, K], B [N, K]; "nn" A [M, K], B [K, N]; "tn" A [K, M],
    B [K, N]; "tt" A [K, M], B [N, K].  The scales do not depend on the
    layout: alpha [M, K/128] per row of A and 128-wide K group, beta
    [ceil(N/128), K/128] per 128 x 128 block of B (in its [N, K] view).
    Reading: the layouts only change how A and B are stored; D is still
    [M, N] = sum over K, so the oracle views both operands as [M, K] and
    [N, K] and evaluates the NT formula."""
    if layout not in LAYOUTS:
        raise ValueError(f"layout must be one of {LAYOUTS}")
    qa = qa_stored.T if layout[0] == "t" else qa_stored
    qb = qb_stored if layout[1] == "t" else qb_stored.T
    return fp8_gemm_nt_f64(np.ascontiguousarray(qa), alpha, np.ascontiguousarray(qb), beta)


def fp8_gemm_nt_accumulate_f64(qa, alpha, qb, beta, c) -> np.ndarray:
    """float64 C + A B^T (Deep dive, section 3: the NT GEMM's D = C + A @ B.T
    form), with C float32 [M, N] taken exactly and added to the float64
    result of the Fig. 13-1 formula."""
    d = fp8_gemm_nt_f64(qa, alpha, qb, beta)
    c64 = np.asarray(c, np.float64)
    if c64.shape != d.shape:
        raise ValueError("C must be [M, N]")
    return c64 + d


def fp8_gemm_nt_accumulate(qa, alpha, qb, beta, c) -> np.ndarray:
    """BF16 bit patterns of D = C + A B^T, rounded once."""
    return bf16.to_bits(fp8_gemm_nt_accumulate_f64(qa, alpha, qb, beta, c))


def m_grouped_contiguous_f64(qa, alpha, qb, beta, m_indices, d_init):
    """Contiguous m-grouped GEMM in float64.

    qa [M_total, K], alpha [M_total, K/128]; qb [G, N, K], beta
    [G, ceil(N/128), K/128]; m_indices int [M_total] (expert of each row, -1 =
    padding); d_init float64 [M_total, N]: returned unchanged on padding rows.
    """
    m_indices = np.asarray(m_indices)
    d = np.array(d_init, dtype=np.float64, copy=True)
    for e in np.unique(m_indices[m_indices >= 0]):
        rows = np.nonzero(m_indices == e)[0]
        d[rows] = fp8_gemm_nt_f64(qa[rows], alpha[rows], qb[e], beta[e])
    return d


def m_grouped_contiguous(qa, alpha, qb, beta, m_indices, d_init_bits):
    """BF16 bits of the contiguous form; padding rows keep ``d_init_bits``."""
    m_indices = np.asarray(m_indices)
    out = np.array(d_init_bits, dtype=np.uint16, copy=True)
    d = m_grouped_contiguous_f64(qa, alpha, qb, beta, m_indices,
                                 np.zeros(out.shape))
    valid = m_indices >= 0
    out[valid] = bf16.to_bits(d[valid])
    return out


def m_grouped_masked_f64(qa, alpha, qb, beta, masked_m, d_init):
    """Masked m-grouped GEMM in float64.

    qa [G, M_max, K], alpha [G, M_max, K/128]; qb [G, N, K], beta
    [G, ceil(N/128), K/128]; masked_m int [G]; d_init [G, M_max, N]: rows
    >= masked_m[g] are returned unchanged.  A masked_m outside [0, M_max] is
    clamped into that range.
    """
    d = np.array(d_init, dtype=np.float64, copy=True)
    G, m_max, _ = qa.shape
    for e in range(G):
        m = int(min(max(int(masked_m[e]), 0), m_max))
        if m:
            d[e, :m] = fp8_gemm_nt_f64(qa[e, :m], alpha[e, :m], qb[e], beta[e])
    return d


def m_grouped_masked(qa, alpha, qb, beta, masked_m, d_init_bits):
    """BF16 bits of the masked form; rows >= masked_m keep ``d_init_bits``."""
    out = np.array(d_init_bits, dtype=np.uint16, copy=True)
    G, m_max, _ = qa.shape
    for e in range(G):
        m = int(min(max(int(masked_m[e]), 0), m_max))
        if m:
            out[e, :m] = fp8_gemm_nt(qa[e, :m], alpha[e, :m], qb[e], beta[e])
    return out


def k_grouped_contiguous_f64(qa, alpha, qb, beta, k_sizes, c=None):
    """K-grouped contiguous GEMM in float64: for every group g,
    D[g] = C[g] + A_g B_g^T, where A_g and B_g are group g's segment of the
    shared K axis (Deep dive, section 3, the grouped GEMM table: the group
    axis is K, M and N are fixed, used for the MoE weight gradient; NT form).

    qa uint8 [M, K_total], alpha float32 [M, K_total/128]; qb uint8
    [N, K_total], beta float32 [N, K_total/128]: both operands are
    token-indexed activations here, so both carry the 1x128 scaling of
    Fig. 13-1's A (one scale per row per 128 K elements).  k_sizes int [G]:
    group g owns the K segment starting at sum(k_sizes[:g]); every size is a
    multiple of 128, so a scale group never spans two experts (zero is
    allowed: that group's D is its C).  c float [G, M, N] or None (zeros).

    Within a segment the Fig. 13-1 order is kept: per 128-wide K block, the
    block's partial product of the decoded codes, times the outer product of
    the block's row scales of A and of B, added in float64.
    """
    M, K = qa.shape
    N, Kb = qb.shape
    k_sizes = np.asarray(k_sizes, dtype=np.int64)
    if K != Kb or K % GROUP:
        raise ValueError("K mismatch or K not a multiple of 128")
    if np.any(k_sizes < 0) or np.any(k_sizes % GROUP) or int(k_sizes.sum()) != K:
        raise ValueError("group sizes must be multiples of 128 that sum to K")
    kg = K // GROUP
    if alpha.shape != (M, kg) or beta.shape != (N, kg):
        raise ValueError("scale shapes do not match the 1x128 grids of A and B")
    G = len(k_sizes)
    d = np.zeros((G, M, N), dtype=np.float64)
    if c is not None:
        c64 = np.asarray(c, np.float64)
        if c64.shape != d.shape:
            raise ValueError("C must be [G, M, N]")
        d += c64
    a_vals = e4m3.decode(qa)
    b_vals = e4m3.decode(qb)
    alpha64 = np.asarray(alpha, np.float64)
    beta64 = np.asarray(beta, np.float64)
    first_block = 0
    for g in range(G):
        blocks = int(k_sizes[g]) // GROUP
        for b in range(first_block, first_block + blocks):
            ks = slice(b * GROUP, (b + 1) * GROUP)
            partial = a_vals[:, ks] @ b_vals[:, ks].T
            d[g] += partial * (alpha64[:, b][:, None] * beta64[:, b][None, :])
        first_block += blocks
    return d
