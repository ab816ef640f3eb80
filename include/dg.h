/*
 * dg.h -- C ABI of the B200 (sm_100a) fine-grained block-scaled FP8 GEMM
 * library (libdg.so).
 *
 * What is computed (sources named by page title and figure/section):
 *
 *   "Lesson 13: DeepSeek DeepGEMM core architecture and Hopper FP8 kernel
 *   breakdown" (hpc.payai.win), Fig. 13-1:
 *       D[i, j] = sum_g alpha[i, g] * beta[g, j / 128]
 *                       * sum_{k < 128} A[i, 128 g + k] * B[j, 128 g + k]
 *   with A, B in E4M3, alpha one FP32 scale per row per 128-wide K group
 *   (alpha = max|group| / 448), beta one FP32 scale per 128 x 128 block of B,
 *   each 128-K block's partial product scaled and promoted into an FP32
 *   accumulator inside the main loop, and D written as BF16.
 *
 *   "DeepGEMM architecture deep dive" (blog.123qwe.co.kr), section 3: NT
 *   layout (A row-major [M, K], B row-major [N, K], D = A * B^T), LHS scales
 *   stored transposed (MN-major) and TMA-aligned, contiguous grouped layout
 *   with expert segments aligned to the M block, masked grouped layout with a
 *   per-expert valid row count; every GEMM as D = C + A @ B (the accumulating
 *   NT form), the K-grouped contiguous form of the MoE weight gradient, and
 *   sm_100's packed UE8M0 scale layout.
 *
 * Conventions shared by every entry point:
 *   - Every pointer argument marked "device" must point to device memory of
 *     the current CUDA device; the caller owns all buffers and the stream.
 *   - All calls are asynchronous on `stream` (NULL = the legacy default
 *     stream) unless stated otherwise; none allocates device memory.
 *   - The return value is a dg_status code.  Argument errors are detected on
 *     the host before anything is launched and leave outputs untouched.
 *     Errors found by a kernel on the device (bad expert index, masked_m out
 *     of range, k-grouped sizes off the rules, a scale UE8M0 cannot hold, a
 *     pipeline wait that timed out) are recorded in a device status word
 *     read by dg_get_device_status().
 *   - The library keeps a small amount of per-device state (device
 *     properties, the device status word), created by the first call on that
 *     device.  Make one call before capturing any call into a CUDA graph.
 *   - E4M3 here is the FN variant: max 448, no infinities, 0x7F/0xFF NaN.
 *   - BF16 outputs are round-to-nearest-even.
 */
#ifndef DG_H_
#define DG_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (CUstream); NULL selects the legacy default stream. */
typedef struct CUstream_st *dg_stream_t;

/* Status codes. */
#define DG_OK 0
#define DG_ERR_INVALID_ARG -1      /* bad shape, null pointer, bad flag       */
#define DG_ERR_ALIGNMENT -2        /* pointer or leading dim not 16-B aligned */
#define DG_ERR_UNSUPPORTED_ARCH -3 /* current device is not sm_100            */
#define DG_ERR_CUDA -4             /* a CUDA runtime/driver call failed        */
#define DG_ERR_WORKSPACE -5        /* workspace missing or too small           */
#define DG_ERR_TIMEOUT -6          /* device: a pipeline wait gave up          */
#define DG_ERR_DEVICE_DATA -7      /* device: bad index / count / size / scale */

/* Input element types for the quantizers. */
#define DG_DTYPE_F32 0
#define DG_DTYPE_BF16 1

/* Quantizer flags. */
#define DG_SCALE_FP32 0 /* scale = fl32(amax / 448)                          */
#define DG_SCALE_POW2 1 /* scale rounded up to a power of two (UE8M0-exact)  */

/* Text for a status code (static string, never NULL). */
const char *dg_status_string(int status);

/* Row alignment each expert segment must have in the contiguous grouped
 * layout (Deep dive, section 3: get_mk_alignment_for_contiguous_layout).
 * Always 128, the M block of every kernel here. */
int dg_get_mk_alignment_for_contiguous_layout(void);

/* Smallest n' >= n such that n' * elem_bytes is a multiple of 16 bytes, the
 * TMA alignment of a leading dimension (DeepGEMM launch article: "get TMA
 * aligned size" utility).  Returns -1 for n < 0 or elem_bytes not in
 * {1, 2, 4, 8}.  Use it for ld_sf / ld_sfa. */
int64_t dg_get_tma_aligned_size(int64_t n, int elem_bytes);

/* Cap the number of SMs the GEMM kernels use (DeepGEMM launch article:
 * "set max SM count").  n <= 0 restores "all SMs".  Returns DG_OK.  The
 * setting is process-wide and read at each launch. */
int dg_set_num_sms(int n);

/* The SM cap in effect for the current device (all SMs when unset). */
int dg_get_num_sms(void);

/*
 * dg_quantize_1x128 -- 1 x 128 activation quantization (Lesson 13,
 * Fig. 13-1; answer to Q1).
 *
 * For every batch b, row i < M and group g < K/128 of x:
 *     amax  = max_k |x[b, i, 128 g + k]|
 *     alpha = fl32(amax / 448)            (DG_SCALE_POW2: rounded up to 2^e)
 *     q[b, i, 128 g + k] = E4M3_RNE_satfinite(fl32(x / alpha))
 * A group with amax == 0 gets alpha = 0 and all codes 0x00.  A negative value
 * that rounds to zero keeps its sign (0x80).  NaN/Inf inputs are unsupported.
 *
 *   x      device, dtype x_dtype (DG_DTYPE_F32 or DG_DTYPE_BF16),
 *          [batch][M][ld_x] row-major; batch stride M * ld_x elements.
 *   batch  >= 1; M >= 0 (M == 0 is a no-op); K > 0, K % 128 == 0.
 *   ld_x   >= K, elements; the row stride must be 16-byte aligned.
 *   q      device uint8 [batch][M][ld_q] (E4M3 codes); ld_q >= K, ld_q % 16 == 0.
 *   sf     device float [batch][K/128][ld_sf], MN-major (scale of row i, group
 *          g of batch b at sf[(b * K/128 + g) * ld_sf + i]);
 *          ld_sf >= M, ld_sf % 4 == 0 (see dg_get_tma_aligned_size).
 *   flags  DG_SCALE_FP32 or DG_SCALE_POW2.
 * All pointers 16-byte aligned.  Output is bit-exact (deterministic).
 */
int dg_quantize_1x128(const void *x, int x_dtype, int64_t batch, int64_t M,
                      int64_t K, int64_t ld_x, uint8_t *q, int64_t ld_q,
                      float *sf, int64_t ld_sf, int flags, dg_stream_t stream);

/*
 * dg_quantize_128x1 -- the 1 x 128 activation quantization of Lesson 13,
 * Fig. 13-1 (groups of 128 consecutive K elements of one row of the logical
 * [M][K] operand) for an operand stored with K outermost, x [K][M]: the
 * group of column m and K group g is x[128 g .. 128 g + 127][m].  This is how
 * the TN / TT GEMMs and the TN k-grouped GEMM take their transposed operands.
 *
 *   x       device float or BF16 (x_dtype) [K][ld_x], ld_x >= M.
 *   q       device uint8 [K][ld_q] E4M3 codes, ld_q >= M.
 *   sf      device float [K/128][ld_sf], MN-major (sf[g * ld_sf + m]), the
 *           layout the GEMMs read; ld_sf >= M, % 4 == 0.
 *   flags   DG_SCALE_FP32 or DG_SCALE_POW2.
 *   M >= 0 (0 is a no-op), K % 128 == 0, K / 128 <= 65535; pointers
 *   16-byte aligned.
 * Bit-exact with dg_quantize_1x128 applied to the transposed operand.
 */
int dg_quantize_128x1(const void *x, int x_dtype, int64_t K, int64_t M,
                      int64_t ld_x, uint8_t *q, int64_t ld_q, float *sf,
                      int64_t ld_sf, int flags, dg_stream_t stream);

/*
 * dg_quantize_128x128 -- 128 x 128 weight block quantization (Lesson 13,
 * Fig. 13-1: "one scale beta per 128 x 128 block, quantized offline").
 *
 * For every group b < G, block (nb, g) of w[b] (rows 128 nb .. min(N, 128 nb
 * + 128), columns 128 g .. 128 g + 128): beta = fl32(amax / 448) (or its
 * power-of-two round-up), q = E4M3_RNE_satfinite(fl32(w / beta)); amax == 0
 * gives beta = 0 and codes 0x00.
 *
 *   w      device float [G][N][K] row-major, 16-byte aligned.
 *   q      device uint8 [G][N][K].
 *   sf     device float [G][ceil(N/128)][K/128] row-major.
 *   G >= 1, N >= 0, K % 128 == 0, K > 0.
 */
int dg_quantize_128x128(const float *w, int64_t G, int64_t N, int64_t K,
                        uint8_t *q, float *sf, int flags, dg_stream_t stream);

/*
 * dg_pack_ue8m0 -- the packed UE8M0 scale layout ("DeepGEMM architecture deep
 * dive", section 3: on sm_100 the LHS scales are four UE8M0 values per 32-bit
 * integer, transposed and TMA-aligned; UE8M0 itself: Lesson 13, Fig. 13-1
 * text).  UE8M0 code e stands for 2^(e - 127); for a power-of-two FP32 scale
 * it is the FP32 exponent field, and +0 is coded 0.
 *
 *   sf      device float [batch][Kg][ld_sf], MN-major: the scale of row i,
 *           K group g at sf[(b * Kg + g) * ld_sf + i] -- the layout
 *           dg_quantize_1x128 writes; with DG_SCALE_POW2 every scale is +0
 *           or a normal power of two.
 *   packed  device int32 [batch][ceil(Kg/4)][ld_packed], MN-major: word
 *           (b, p, i) holds groups 4p .. 4p+3 of row i, group 4p+t in bits
 *           8t .. 8t+7; groups past Kg are zero bytes.  Entries i >= M are
 *           not written.
 *   batch >= 1, M >= 0 (M == 0 is a no-op), Kg >= 1; ld_sf >= M and
 *   ld_packed >= M, both multiples of 4; both pointers 16-byte aligned.
 * A scale that is not +0 or a positive normal power of two (a signed value,
 * a non-power of two, a subnormal, inf or NaN) is recorded in the device
 * status word as DG_ERR_DEVICE_DATA (see dg_get_device_status); its byte is
 * then its exponent field.  Output is bit-exact.  Memory is caller-owned.
 */
int dg_pack_ue8m0(const float *sf, int64_t batch, int64_t M, int64_t Kg,
                  int64_t ld_sf, int32_t *packed, int64_t ld_packed,
                  dg_stream_t stream);

/*
 * dg_pack_ue8m0_128x128 -- 128 x 128 block scales of B (Lesson 13, Fig. 13-1)
 * written out in the packed UE8M0 layout one word row per row of B, the form
 * the UE8M0 GEMMs read B's scales in (each of the 128 rows of a block repeats
 * the block's words).
 *
 *   sf      device float [G][ceil(N/128)][Kg] row-major, as written by
 *           dg_quantize_128x128 with DG_SCALE_POW2 (every scale +0 or a
 *           normal power of two).
 *   packed  device int32 [G][ceil(Kg/4)][ld_packed]: word (g, p, n) holds
 *           groups 4p .. 4p+3 of block n/128 of expert g, group 4p+t in bits
 *           8t .. 8t+7; groups past Kg are zero bytes.  Entries n >= N are not
 *           written.
 *   G >= 1, N >= 0 (0 is a no-op), Kg >= 1, ld_packed >= N and % 4 == 0;
 *   both pointers 16-byte aligned.
 * Scales UE8M0 cannot hold are recorded as DG_ERR_DEVICE_DATA, as in
 * dg_pack_ue8m0.  Output is bit-exact.  Memory is caller-owned.
 */
int dg_pack_ue8m0_128x128(const float *sf, int64_t G, int64_t N, int64_t Kg,
                          int32_t *packed, int64_t ld_packed, dg_stream_t stream);

/*
 * dg_fp8_gemm_nt -- dense NT GEMM, D = A * B^T with 1x128 / 128x128 scales
 * (Lesson 13, Fig. 13-1; DeepGEMM launch article: gemm_fp8_fp8_bf16_nt).
 *
 *   A      device uint8 [M][K] E4M3, row-major (K-major), 16-byte aligned.
 *   sfa    device float [K/128][ld_sfa] MN-major alpha (as written by
 *          dg_quantize_1x128 with batch 1); ld_sfa >= M, ld_sfa % 4 == 0.
 *   B      device uint8 [N][K] E4M3, row-major (K-major).
 *   sfb    device float [ceil(N/128)][K/128] row-major beta.
 *   D      device BF16 [M][N] row-major, written for all i < M, j < N.
 *   workspace, workspace_bytes
 *          optional device scratch (may be NULL / 0).  When at least
 *          dg_fp8_gemm_nt_workspace_size(M, N, K) bytes are given, the GEMM
 *          may split K across CTAs: small-M (decode) shapes split every tile,
 *          large shapes only the tiles of a last, partial wave of CTAs.  A
 *          decode tile's splits usually form one thread-block cluster and
 *          sum their partials in on-chip shared memory, leaving the workspace
 *          unused; otherwise FP32 partials go to the workspace and the splits
 *          of a tile sum them there.  Either way the splits are added in a
 *          fixed order.  The workspace must not be used by another call that
 *          runs at the same time; its contents between calls do not matter.
 *   M >= 0 (0 is a no-op), N > 0 with N % 8 == 0, K > 0 with K % 128 == 0.
 * Deterministic: repeated calls give identical bits (also with split K).
 */
int dg_fp8_gemm_nt(const uint8_t *A, const float *sfa, int64_t ld_sfa,
                   const uint8_t *B, const float *sfb, void *D, int64_t M,
                   int64_t N, int64_t K, void *workspace,
                   size_t workspace_bytes, dg_stream_t stream);

/*
 * dg_fp8_gemm_nn, dg_fp8_gemm_tn, dg_fp8_gemm_tt -- the dense GEMM with the
 * other operand layouts ("DeepGEMM architecture deep dive", section 3: every
 * GEMM is D = C + A @ B, NT by default, and sm_100 supports NT, TN, NN and
 * TT).  The first letter says how A is used, the second how B is: N as
 * stored, T transposed, with D = A * B^T always [M][N]:
 *   NN  A [M][K] (K-major) and B stored [K][N] (N contiguous);
 *   TN  A stored [K][M] (M contiguous) and B stored [K][N];
 *   TT  A stored [K][M] and B [N][K] (K-major).
 * The scales keep their logical meaning: sfa is alpha per row of A and
 * 128-wide K group (device float [K/128][ld_sfa], MN-major, as for NT) and
 * sfb is beta per 128 x 128 block of B's [N][K] view ([ceil(N/128)][K/128]).
 * An operand stored with K outermost is loaded as MN-major tiles, so its row
 * stride must be a multiple of 16 bytes: M % 16 == 0 for TN and TT, N % 16
 * == 0 for NN and TN (DG_ERR_ALIGNMENT otherwise).  Everything else --
 * arguments, workspace use, errors, determinism -- is as in dg_fp8_gemm_nt
 * (the tile is 128 or 256 columns wide).
 */
int dg_fp8_gemm_nn(const uint8_t *A, const float *sfa, int64_t ld_sfa,
                   const uint8_t *B, const float *sfb, void *D, int64_t M,
                   int64_t N, int64_t K, void *workspace,
                   size_t workspace_bytes, dg_stream_t stream);
int dg_fp8_gemm_tn(const uint8_t *A, const float *sfa, int64_t ld_sfa,
                   const uint8_t *B, const float *sfb, void *D, int64_t M,
                   int64_t N, int64_t K, void *workspace,
                   size_t workspace_bytes, dg_stream_t stream);
int dg_fp8_gemm_tt(const uint8_t *A, const float *sfa, int64_t ld_sfa,
                   const uint8_t *B, const float *sfb, void *D, int64_t M,
                   int64_t N, int64_t K, void *workspace,
                   size_t workspace_bytes, dg_stream_t stream);

/* Workspace size in bytes with which dg_fp8_gemm_nt (and the NN, TN, TT
 * forms) use the K split the tile heuristic prefers for this shape on the
 * current device (0 when that choice does not split K; the result depends on
 * the SM count in effect, see dg_set_num_sms).  A multiple of 256 bytes. */
size_t dg_fp8_gemm_nt_workspace_size(int64_t M, int64_t N, int64_t K);

/*
 * dg_fp8_gemm_nt_noalloc -- dg_fp8_gemm_nt for callers that cannot allocate
 * device memory.  The pages have no counterpart to this entry point.
 *
 * Who needs it: a runtime that reserves all device memory at start-up and
 * forbids later allocation, a plugin whose host framework owns every buffer
 * and passes in only inputs and outputs, or a latency-critical loop that
 * cannot pay for cudaMalloc's implicit device-wide synchronisation.  Such a
 * caller cannot supply the split-K workspace dg_fp8_gemm_nt takes; here the
 * scratch is a fixed 32 MiB array inside the library, placed on each device
 * that loads the library's code and kept there until the process exits.
 *
 * Same computation, arguments, layouts and errors as dg_fp8_gemm_nt, minus
 * the workspace.  Nothing is allocated and no allocating routine is called.
 *   - Returns DG_ERR_WORKSPACE (nothing launched) when the shape's preferred
 *     K split needs more than 32 MiB, i.e. when
 *     dg_fp8_gemm_nt_workspace_size(M, N, K) > 32 MiB.  The split tiles
 *     times their splits never exceed the SM count, so the need is at most
 *     SMs x 128 KiB plus 4 bytes per SM (about 19.4 MB on a 148-SM B200):
 *     devices of up to 256 SMs never see this error.
 *   - Uses exactly the tile form and split that dg_fp8_gemm_nt picks when
 *     given dg_fp8_gemm_nt_workspace_size(M, N, K) bytes of workspace, so
 *     both give identical bits.
 *   - The first call on a device looks up the array's device address (and
 *     loads that code on the device); make that first call before any stream
 *     capture.  A lookup that fails returns DG_ERR_CUDA and is retried by
 *     the next call.
 *   - All calls share the one array and leave their partial sums in it; each
 *     call clears the part that must start at zero before its kernel runs.
 *     Calls whose kernels overlap on the GPU (unordered streams) race on the
 *     array: order them.
 */
int dg_fp8_gemm_nt_noalloc(const uint8_t *A, const float *sfa, int64_t ld_sfa,
                           const uint8_t *B, const float *sfb, void *D, int64_t M,
                           int64_t N, int64_t K, dg_stream_t stream);

/*
 * dg_fp8_gemm_nt_quantize -- dg_fp8_gemm_nt with the FP8 cast of its output
 * fused into the epilogue ("DeepGEMM architecture deep dive", section 3:
 * users should fuse the FP8 cast into the kernel that produces the data).
 * D is not written as BF16; each row's 128-column groups leave the GEMM
 * already quantized 1 x 128 (Lesson 13, Fig. 13-1), in the layouts the next
 * GEMM takes as its A and alpha.  The result is bit-identical to rounding D
 * to BF16 and then calling dg_quantize_1x128 on it (DG_DTYPE_BF16, the same
 * flags), for the tile form this call uses (256-wide tiles, K not split; a
 * dg_fp8_gemm_nt that splits K may round a few elements of D differently).
 *
 *   A, sfa, ld_sfa, B, sfb, M, K   as in dg_fp8_gemm_nt.
 *   N      N % 128 == 0 (whole groups).
 *   Dq     device uint8 [M][N] E4M3 codes, 16-byte aligned.
 *   sfd    device float [N/128][ld_sfd], MN-major: the scale of row i, column
 *          group g at sfd[g * ld_sfd + i]; ld_sfd >= M, % 4 == 0, 16-byte
 *          aligned.
 *   flags  DG_SCALE_FP32 or DG_SCALE_POW2 (scales rounded up to powers of
 *          two, UE8M0-representable).
 * No workspace: K is never split.  Deterministic.
 */
int dg_fp8_gemm_nt_quantize(const uint8_t *A, const float *sfa, int64_t ld_sfa,
                            const uint8_t *B, const float *sfb, uint8_t *Dq,
                            float *sfd, int64_t ld_sfd, int64_t M, int64_t N,
                            int64_t K, int flags, dg_stream_t stream);

/*
 * dg_fp8_gemm_nt_accumulate -- D = C + A * B^T (Deep dive, section 3: the NT
 * GEMM's accumulating form): the block-scaled product of dg_fp8_gemm_nt plus
 * an FP32 matrix C, added to the FP32 accumulator before the single rounding
 * of D to BF16.
 *
 * Same arguments, layouts, workspace use and errors as dg_fp8_gemm_nt, plus
 *   C      device float [M][N] row-major, 16-byte aligned, read only; must
 *          not overlap D.  NULL is DG_ERR_INVALID_ARG (unless M == 0).
 * Decode-sized splits of K go through the workspace (not through clusters);
 * the 2-CTA pair form is not used.  Deterministic.
 */
int dg_fp8_gemm_nt_accumulate(const uint8_t *A, const float *sfa,
                              int64_t ld_sfa, const uint8_t *B,
                              const float *sfb, const float *C, void *D,
                              int64_t M, int64_t N, int64_t K, void *workspace,
                              size_t workspace_bytes, dg_stream_t stream);

/*
 * dg_m_grouped_fp8_gemm_nt_contiguous -- MoE m-grouped GEMM, contiguous
 * layout (Lesson 13, Fig. 13-3 "contiguous"; Deep dive, section 3).
 *
 * The tokens of all experts are concatenated along M.  Row i belongs to
 * expert m_indices[i] (-1 = padding row).  Every aligned block of 128 rows
 * belongs to at most one expert; blocks holding only padding are skipped.
 *   D[i, :] = A[i, :] * B[m_indices[i]]^T  (with the scales of that expert)
 * for m_indices[i] >= 0; padding rows of D are not written.
 *
 *   A          device uint8 [M_total][K]; sfa device float [K/128][ld_sfa]
 *              (ld_sfa >= M_total, % 4 == 0).
 *   B          device uint8 [G][N][K]; sfb device float [G][ceil(N/128)][K/128].
 *   D          device BF16 [M_total][N].
 *   m_indices  device int32 [M_total].
 *   M_total % 128 == 0 (dg_get_mk_alignment_for_contiguous_layout), G >= 1,
 *   N % 8 == 0, K % 128 == 0.
 * Device-side errors (recorded, the offending rows are skipped):
 *   an index >= G, or two different experts inside one 128-row block.
 */
int dg_m_grouped_fp8_gemm_nt_contiguous(const uint8_t *A, const float *sfa,
                                        int64_t ld_sfa, const uint8_t *B,
                                        const float *sfb, void *D,
                                        const int32_t *m_indices,
                                        int64_t M_total, int64_t N, int64_t K,
                                        int G, dg_stream_t stream);

/*
 * dg_m_grouped_fp8_gemm_nt_masked -- MoE m-grouped GEMM, masked layout
 * (Lesson 13, Fig. 13-3 "masked" and the answer to Q3; Deep dive, section 3).
 *
 * Expert g owns the fixed slab A[g] of M_max rows; only its first
 * masked_m[g] rows are valid.  masked_m is read on the device, so launch
 * parameters do not depend on it and the call can be replayed from a CUDA
 * graph with new counts.
 *   D[g, i, :] = A[g, i, :] * B[g]^T  for i < masked_m[g];
 * rows i >= masked_m[g] of D are not written.
 *
 *   A         device uint8 [G][M_max][K]; sfa device float [G][K/128][ld_sfa]
 *             (ld_sfa >= M_max, % 4 == 0).
 *   B         device uint8 [G][N][K]; sfb device float [G][ceil(N/128)][K/128].
 *   D         device BF16 [G][M_max][N].
 *   masked_m  device int32 [G]; values outside [0, M_max] are clamped and
 *             recorded as DG_ERR_DEVICE_DATA.
 *   1 <= G <= 1024, M_max >= 1, N % 8 == 0, K % 128 == 0.
 */
int dg_m_grouped_fp8_gemm_nt_masked(const uint8_t *A, const float *sfa,
                                    int64_t ld_sfa, const uint8_t *B,
                                    const float *sfb, void *D,
                                    const int32_t *masked_m, int G,
                                    int64_t M_max, int64_t N, int64_t K,
                                    dg_stream_t stream);

/*
 * dg_fp8_gemm_nt_ue8m0 -- dense NT GEMM with power-of-two scales given as
 * packed UE8M0 codes (Lesson 13, Fig. 13-1 text: newer versions accept UE8M0
 * scales; Deep dive, section 3: on sm_100 the scales are four UE8M0 values
 * per 32-bit word, MN-major, TMA-aligned).  The formula is Fig. 13-1's with
 * alpha = 2^(code_A - 127) per row of A and 128-wide K group and
 * beta = 2^(code_B - 127) per row of B and K group.  Because every scale is a
 * power of two, the tensor cores apply them (block-scaled MMA, one scale per
 * row and 32-wide K slice) and the tile accumulates in FP32 over the whole of
 * K; there is no per-block promotion on the CUDA cores.  A code of 0 stands
 * for 2^-127 and may only scale an all-zero group (the quantizer's +0 scale).
 *
 *   A      device uint8 [M][K] E4M3, row-major (K-major).
 *   sfa    device int32 [ceil(K/512)][ld_sfa], the layout dg_pack_ue8m0
 *          writes: word (p, i) holds K groups 4p .. 4p+3 of row i;
 *          ld_sfa >= M, % 4 == 0.
 *   B      device uint8 [N][K] E4M3, row-major (K-major).
 *   sfb    device int32 [ceil(K/512)][ld_sfb], one word row per row of B
 *          (dg_pack_ue8m0 of per-row scales, or dg_pack_ue8m0_128x128 of
 *          128 x 128 block scales); ld_sfb >= N, % 4 == 0.
 *   D      device BF16 [M][N] row-major, written for all i < M, j < N.
 *   M >= 0 (0 is a no-op), N > 0 with N % 8 == 0, K > 0 with K % 128 == 0;
 *   A, B, D, sfa, sfb 16-byte aligned.
 * No workspace: K is never split.  Deterministic.
 */
int dg_fp8_gemm_nt_ue8m0(const uint8_t *A, const int32_t *sfa, int64_t ld_sfa,
                         const uint8_t *B, const int32_t *sfb, int64_t ld_sfb,
                         void *D, int64_t M, int64_t N, int64_t K,
                         dg_stream_t stream);

/*
 * dg_m_grouped_fp8_gemm_nt_masked_ue8m0 -- the masked MoE GEMM of
 * dg_m_grouped_fp8_gemm_nt_masked with packed UE8M0 scales as in
 * dg_fp8_gemm_nt_ue8m0: sfa device int32 [G][ceil(K/512)][ld_sfa]
 * (ld_sfa >= M_max, % 4 == 0), sfb device int32 [G][ceil(K/512)][ld_sfb]
 * (ld_sfb >= N, % 4 == 0).  Rows >= masked_m[g] of D are not written;
 * masked_m outside [0, M_max] is clamped and recorded as DG_ERR_DEVICE_DATA.
 *   1 <= G <= 1024, M_max >= 1, N % 8 == 0, K % 128 == 0.
 */
int dg_m_grouped_fp8_gemm_nt_masked_ue8m0(const uint8_t *A, const int32_t *sfa,
                                          int64_t ld_sfa, const uint8_t *B,
                                          const int32_t *sfb, int64_t ld_sfb, void *D,
                                          const int32_t *masked_m, int G,
                                          int64_t M_max, int64_t N, int64_t K,
                                          dg_stream_t stream);

/*
 * dg_k_grouped_fp8_gemm_nt_contiguous -- the K-grouped contiguous GEMM of
 * the MoE weight gradient ("DeepGEMM architecture deep dive", section 3, the
 * grouped GEMM table: the group axis is K, M and N are shared).  The K axis
 * (tokens) is cut into G consecutive segments; for every group g,
 *
 *   D[g][i][j] = C[g][i][j] + sum over the 128-K blocks b of segment g of
 *                alpha[i][b] * beta[j][b] * sum_{k < 128} A[i][128b+k] B[j][128b+k]
 *
 * in FP32: both operands carry 1x128 scales along K (Lesson 13, Fig. 13-1's
 * activation scaling; here A and B are both token-indexed).
 *
 *   A        device E4M3 [M][K] row-major (K-major); B device E4M3 [N][K].
 *   sfa      device float [K/128][ld_sfa], MN-major (dg_quantize_1x128 of A);
 *            ld_sfa >= M, ld_sfa % 4 == 0.
 *   sfb      device float [K/128][ld_sfb], MN-major (dg_quantize_1x128 of B);
 *            ld_sfb >= N, ld_sfb % 4 == 0.
 *   C        device float [G][M][N] added to the product, or NULL (zero).
 *   D        device float [G][M][N], written whole (an empty group gets C,
 *            or zeros).
 *   k_sizes  device int32 [G]: K of each segment, each a multiple of 128,
 *            summing to K (0 allowed).  Sizes off the 128 grid or not adding
 *            up to K are recorded in the device status word as
 *            DG_ERR_DEVICE_DATA; the kernel then clamps every segment into
 *            [0, K) and reads nothing outside the operands.
 *   1 <= G <= 1024, M >= 0 (M == 0 is a no-op), N > 0, N % 8 == 0,
 *   K > 0, K % 128 == 0.  All pointers 16-byte aligned.
 * Memory is caller-owned; nothing is allocated.  Results are deterministic.
 */
int dg_k_grouped_fp8_gemm_nt_contiguous(const uint8_t *A, const float *sfa,
                                        int64_t ld_sfa, const uint8_t *B,
                                        const float *sfb, int64_t ld_sfb,
                                        const float *C, float *D,
                                        const int32_t *k_sizes, int G,
                                        int64_t M, int64_t N, int64_t K,
                                        dg_stream_t stream);

/*
 * dg_get_device_status -- synchronizes `stream`, then reads and clears the
 * current device's status word.  *status receives DG_OK or the first device
 * error recorded since the last read (DG_ERR_TIMEOUT, DG_ERR_DEVICE_DATA).
 * Returns DG_OK, or DG_ERR_CUDA if the synchronization itself failed.
 */
/*
 * dg_k_grouped_fp8_gemm_tn_contiguous -- the K-grouped GEMM of
 * dg_k_grouped_fp8_gemm_nt_contiguous with both operands stored with the
 * token axis K outermost, as a weight gradient's activations and output
 * gradients are ("DeepGEMM architecture deep dive", section 3, the grouped
 * GEMM table: K-grouped, FP8 TN):
 *   A  device uint8 [K][M] (M contiguous), M % 16 == 0;
 *   B  device uint8 [K][N] (N contiguous), N % 16 == 0;
 * sfa [K/128][ld_sfa] and sfb [K/128][ld_sfb], C, D, k_sizes and everything
 * else as in the NT form: D[g][i][j] = C[g][i][j] + the sum over group g's
 * K segment (per 128-wide K block, scaled by alpha[i] and beta[j] of the
 * block) of A[k][i] * B[k][j].
 */
int dg_k_grouped_fp8_gemm_tn_contiguous(const uint8_t *A, const float *sfa,
                                        int64_t ld_sfa, const uint8_t *B,
                                        const float *sfb, int64_t ld_sfb,
                                        const float *C, float *D,
                                        const int32_t *k_sizes, int G, int64_t M,
                                        int64_t N, int64_t K, dg_stream_t stream);

int dg_get_device_status(dg_stream_t stream, int *status);

#ifdef __cplusplus
}
#endif

#endif /* DG_H_ */
