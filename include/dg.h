/*
 * dg.h -- C ABI of libdg.so: FP8 (E4M3) GEMMs with fine-grained FP32 scaling
 * and two-level (promoted) accumulation, for NVIDIA B200 (sm_100a).
 *
 * Operation (DeepGEMM README summary, ja.news.hada.io topic 19459, section
 * "GEMMインターフェースとレイアウト制約"): D = C + A @ B.T, with NT as the base
 * layout; scaling factors are FP32 and the LHS scales are stored transposed
 * (MN-major) with a TMA-aligned leading dimension. Scale granularity: one
 * scale per 1x128 K-strip of A and per 128x128 block of B; the per-K-block
 * tensor-core partial sums are promoted into an FP32 accumulator with
 * sfa * sfb applied ("DeepSeek開源新突破：DeepGEMM庫揭秘", paragraph 2: two-level
 * accumulation because the FP8 tensor-core accumulator is imprecise).
 *
 * Conventions for every entry point below:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the
 *     library never frees or retains them. Row-major, densely packed, unless
 *     a leading dimension is stated.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Calls are
 *     asynchronous on it: no host synchronisation, no device-to-host reads,
 *     no memory allocation. They are therefore safe to capture in a CUDA graph.
 *   - Every base pointer must be 16-byte aligned. Arguments are validated on
 *     the host before anything is launched; a violation returns an error code
 *     and launches nothing.
 *   - Device-side waits are bounded: a wait that exceeds the timeout (default
 *     2 s) records DG_ERR_TIMEOUT in a per-device error word, and the kernel
 *     exits cleanly; read it with dg_get_last_device_error(). The output of a
 *     launch that timed out is undefined (some tiles may be written, others
 *     not); inputs are never written.
 *   - E4M3 bytes are the OCP OFP8 "E4M3FN" encoding (torch.float8_e4m3fn).
 */
#ifndef DG_H
#define DG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DG_OK = 0,
  DG_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad enum */
  DG_ERR_UNSUPPORTED_SHAPE = 2, /* K % 128 != 0, N % 8 != 0, too many groups, ... */
  DG_ERR_MISALIGNED = 3,        /* a pointer is not 16-byte aligned */
  DG_ERR_CUDA = 4,              /* a CUDA runtime / driver call failed */
  DG_ERR_TIMEOUT = 5            /* a bounded device wait ran out (see above) */
} dg_status;

/* Human-readable name of a status code (static string). */
const char* dg_status_string(dg_status s);

/* ---------------------------------------------------------------------------
 * Quantiser: BF16/FP32 -> E4M3 codes + FP32 scales.
 * Source: same README summary, section "GEMMインターフェースとレイアウト制約"
 * (casting and scale layout are the caller's job; the library ships helpers),
 * and the scale rule fixed for this library: scale = max(amax, 1e-4f) / 448,
 * code = E4M3_RN_satfinite(x / scale), both IEEE FP32 divisions.
 *
 *   x       [batch][rows][cols], FP32 (in_dtype = DG_IN_F32) or BF16
 *           (DG_IN_BF16). Read only.
 *   codes   [batch][rows][cols] E4M3 bytes (written).
 *   scales  written per mode:
 *     DG_QUANT_ROW_1x128     one per (row, 128-col strip): cols % 128 == 0;
 *                            scales[b][cols/128][ld_scales], transposed
 *                            (MN-major); ld_scales >= rows, ld_scales % 4 == 0.
 *                            This is the sfa layout every NT GEMM below reads.
 *     DG_QUANT_BLOCK_128x128 one per 128x128 block, rows and columns may
 *                            be ragged: scales[b][ceil(rows/128)]
 *                            [ceil(cols/128)]; cols % 4 == 0; ld_scales
 *                            ignored. This is the sfb layout (of B [N][K],
 *                            and of B [K][N] for the NN / TN layouts).
 *     DG_QUANT_COL_128x1     one per (128-row strip, column): rows % 128 == 0;
 *                            scales[b][rows/128][cols]; ld_scales ignored.
 *                            This is the layout the K-grouped TN GEMM reads.
 *   amax is taken over the elements that exist (a ragged last block reads only
 *   its real rows and columns).
 * ------------------------------------------------------------------------- */
enum { DG_IN_F32 = 0, DG_IN_BF16 = 1 };
enum { DG_QUANT_ROW_1x128 = 0, DG_QUANT_BLOCK_128x128 = 1, DG_QUANT_COL_128x1 = 2 };

dg_status dg_quantize_fp8(const void* x, int in_dtype, int batch, int rows, int cols,
                          int mode, void* codes, float* scales, int ld_scales,
                          void* stream);

/* ---------------------------------------------------------------------------
 * Dense NT GEMM: D[m][n] = C[m][n] + sum_kb sfa[kb][m] * sfb[n/128][kb] *
 *                          sum_{k in kb} A[m][k] * B[n][k]
 * Source: README summary, "GEMMインターフェースとレイアウト制約" (fp8_gemm_nt).
 *
 *   A    [M][K] E4M3            sfa [K/128][align4(M)] FP32 (ROW_1x128 layout)
 *   B    [N][K] E4M3            sfb [ceil(N/128)][K/128] FP32 (BLOCK layout)
 *   C    [M][N] BF16 or NULL (C may alias D)
 *   D    [M][N] BF16, rounded to nearest even from the FP32 accumulator.
 * Shapes: M >= 0, N >= 0 (either 0: no-op), K % 128 == 0 (K == 0: D = C),
 * N % 8 == 0.
 * M <= 128 (decode) runs a swap-AB kernel with split-K over a thread-block
 * cluster, or, for 65..128 rows where a cost model expects it to be faster,
 * 128 x 256 tiles with each tile split along K over a cluster (both
 * reductions add the partial sums in a fixed order, so results repeat bit
 * for bit from run to run). The test hook dg_debug_drop_next_arrive does not
 * apply to such split tiles.
 * ------------------------------------------------------------------------- */
dg_status dg_fp8_gemm_nt(const void* A, const float* sfa, const void* B, const float* sfb,
                         const void* C, void* D, int M, int N, int K, void* stream);

/* ---------------------------------------------------------------------------
 * Dense GEMM with the other operand layouts (README summary, "GEMMインター
 * フェースとレイアウト制約": NT is the base layout, NN / TN / TT are offered
 * besides). Same operation and scale granularity as dg_fp8_gemm_nt; the
 * letters are named as NT is: A [M][K] = N, A [K][M] = T; B [N][K] = T (as
 * in D = A @ B.T), B [K][N] = N:
 *   NN  A [M][K], sfa [K/128][align4(M)];  B [K][N], sfb [K/128][ceil(N/128)]
 *   TN  A [K][M], sfa [K/128][M];          B [K][N], sfb [K/128][ceil(N/128)]
 *   TT  A [K][M], sfa [K/128][M];          B [N][K], sfb [ceil(N/128)][K/128]
 * (the quantiser's COL_128x1 mode on A [K][M] and BLOCK_128x128 mode on
 * B [K][N] produce exactly these scale layouts). C / D [M][N] BF16 as NT.
 * K % 128 == 0, N % 8 == 0; M % 16 == 0 when A is [K][M]; N % 16 == 0 when
 * B is [K][N]. The small-M (decode) strategy is NT-only: these run the
 * persistent kernel for every M.
 * A dense weight gradient (dW = dY^T X, both operands K-outer, FP32 output,
 * accumulation onto C) is dg_k_grouped_fp8_gemm_tn_contiguous with G = 1.
 * ------------------------------------------------------------------------- */
dg_status dg_fp8_gemm_nn(const void* A, const float* sfa, const void* B, const float* sfb,
                         const void* C, void* D, int M, int N, int K, void* stream);
dg_status dg_fp8_gemm_tn(const void* A, const float* sfa, const void* B, const float* sfb,
                         const void* C, void* D, int M, int N, int K, void* stream);
dg_status dg_fp8_gemm_tt(const void* A, const float* sfa, const void* B, const float* sfb,
                         const void* C, void* D, int M, int N, int K, void* stream);

/* ---------------------------------------------------------------------------
 * M-grouped GEMM, contiguous layout (MoE prefill / training forward).
 * Source: README summary, section "DenseとGrouped GEMM": experts share N and K;
 * each expert's tokens are concatenated along M, each segment aligned to the
 * M block size (dg_get_mk_alignment_for_contiguous_layout()).
 *
 *   A         [Mt][K] E4M3, Mt % 128 == 0
 *   sfa       [K/128][align4(Mt)] FP32
 *   B         [G][N][K] E4M3      sfb [G][ceil(N/128)][K/128] FP32
 *   m_indices [Mt] int32 device array: expert id of each row, -1 on padding.
 *             Each 128-row block must belong to a single expert (or be all
 *             padding). A block whose first row is -1 is skipped entirely.
 *   C         [Mt][N] BF16 or NULL     D [Mt][N] BF16
 * Rows with m_indices == -1 (and rows whose id is >= G) are left untouched.
 * ------------------------------------------------------------------------- */
dg_status dg_m_grouped_fp8_gemm_nt_contiguous(const void* A, const float* sfa, const void* B,
                                              const float* sfb, const int32_t* m_indices,
                                              const void* C, void* D, int Mt, int N, int K,
                                              int G, void* stream);

/* ---------------------------------------------------------------------------
 * M-grouped GEMM, masked layout (MoE decode under CUDA graphs, where the host
 * does not know per-expert token counts).
 * Source: README summary, "DenseとGrouped GEMM" (m_grouped_fp8_gemm_nt_masked:
 * given a mask tensor the kernel computes only the valid region).
 *
 *   A        [G][max_m][K] E4M3     sfa [G][K/128][align4(max_m)] FP32
 *   B        [G][N][K] E4M3         sfb [G][ceil(N/128)][K/128] FP32
 *   masked_m [G] int32 device array, read on the device; values are clamped
 *            to [0, max_m].
 *   D        [G][max_m][N] BF16; rows m >= masked_m[g] are left untouched.
 *   expected_m  host-side hint, the typical number of valid rows per group
 *            (same section: the call takes an expected M because the counts
 *            are only known on the device). It only steers the tile-width
 *            choice; results do not depend on it. <= 0 means unknown (plan for
 *            max_m); values above max_m count as max_m.
 * G <= 1024.
 * ------------------------------------------------------------------------- */
dg_status dg_m_grouped_fp8_gemm_nt_masked(const void* A, const float* sfa, const void* B,
                                          const float* sfb, const int32_t* masked_m, void* D,
                                          int G, int max_m, int expected_m, int N, int K,
                                          void* stream);

/* ---------------------------------------------------------------------------
 * K-grouped GEMM, TN, contiguous along K (MoE weight gradient).
 * Source: README summary, "DenseとGrouped GEMM" (k_grouped_fp8_gemm_tn_contiguous:
 * M and N fixed, groups along K). Reading of "TN": both operands are stored
 * K-outer (M or N contiguous), groups concatenated along K.
 *
 *   A      [sumK][M] E4M3   sfa [sumK/128][M] FP32 (COL_128x1 layout)
 *   B      [sumK][N] E4M3   sfb [sumK/128][N] FP32 (COL_128x1 layout)
 *   ks     HOST array of G per-group K sizes, each a multiple of 128 (0
 *          allowed); read during the call only.
 *   C      [G][M][N] FP32 or NULL (may alias D)     D [G][M][N] FP32
 *   D_g[m][n] = C_g[m][n] + sum_{kb in group g} sfa[kb][m] * sfb[kb][n] *
 *               sum_{k in kb} A[k][m] * B[k][n]
 * M % 16 == 0, N % 16 == 0, 1 <= G <= 256.
 * ------------------------------------------------------------------------- */
dg_status dg_k_grouped_fp8_gemm_tn_contiguous(const void* A, const float* sfa, const void* B,
                                              const float* sfb, const int* ks, const float* C,
                                              float* D, int G, int M, int N, void* stream);

/* ---------------------------------------------------------------------------
 * Power-of-two (UE8M0) scales and the tensor core's block-scaled MMA.
 * Source: README summary, "GEMMインターフェースとレイアウト制約" (UE8M0 scales,
 * four packed per int32); the hardware path replaces the per-K-block
 * promotion with tcgen05.mma kind::mxf8f6f4 block scaling, so it relies on
 * the tensor core's own FP32 accumulation across K-blocks.
 *
 * dg_quantize_fp8_ue8m0: as dg_quantize_fp8 (batch 1, modes ROW_1x128 or
 * BLOCK_128x128, cols % 128 == 0), but every scale is rounded up to a power
 * of two, s = 2^ceil(log2(max(amax, 1e-4f) / 448)), and code = E4M3_RN(x / s)
 * (exact division, never saturating).
 *   scales  optional (NULL allowed): FP32 scales in dg_quantize_fp8's layout
 *           for that mode (usable by dg_fp8_gemm_nt, the promotion path).
 *   packed  int32 [ceil(cols/512)][ceil(rows/128)][32][4] (written): byte b of
 *           word [q][rb][i][j] = biased exponent (log2 s + 127) of row
 *           128 rb + 32 j + i for K-block 4 q + b. BLOCK mode writes its block
 *           scale for all 128 rows of the block (rows past `rows` included).
 *           Bytes of K-blocks past cols/128, and of rows past `rows` in ROW
 *           mode, are not written.
 * ------------------------------------------------------------------------- */
dg_status dg_quantize_fp8_ue8m0(const void* x, int in_dtype, int rows, int cols, int mode,
                                void* codes, float* scales, int ld_scales, int32_t* packed,
                                void* stream);

/* Dense NT GEMM on the block-scaled MMA: D = C + A @ B.T with sfa / sfb the
 * packed UE8M0 scales of A (ROW mode, rows = M) and B (BLOCK mode, rows = N)
 * from dg_quantize_fp8_ue8m0. A [M][K], B [N][K] E4M3; C [M][N] BF16 or NULL
 * (may alias D); D [M][N] BF16. K % 128 == 0, N % 8 == 0. M <= 128 runs a
 * swap-AB kernel with split-K over a cluster (partials added in rank order). */
dg_status dg_fp8_gemm_nt_ue8m0(const void* A, const int32_t* sfa, const void* B,
                               const int32_t* sfb, const void* C, void* D, int M, int N, int K,
                               void* stream);

/* ---------------------------------------------------------------------------
 * FP8 x FP4 (mixed precision): E4M3 activations times E2M1 weights.
 * Sources: README summary (ja.news.hada.io topic 19459), the 2026-04 update
 * (FP8xFP4 GEMM on SM100) and "GEMMインターフェースとレイアウト制約" (SM100
 * scaling factors are packed UE8M0); "DeepGEMM技术解析" (mlqm.cn), section
 * 5.2 (FP8xFP4 -> BF16). The pages fix neither the 4-bit format nor its scale
 * granularity; this library takes E2M1 of the OCP Microscaling Formats
 * specification v1.0 (section 5.3.3: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6)
 * with one power-of-two scale per 32 consecutive K elements of a row, the
 * block size of that specification and the 1X scale vector of the tensor
 * core's block-scaled MMA.
 *
 * dg_quantize_fp4_e2m1: x [rows][cols] (in_dtype F32 or BF16), cols % 128 == 0.
 *   s = 2^ceil(log2(max(amax, 1e-4f) / 6)) per (row, 32-column strip),
 *   code = E2M1_RN(x / s) (exact division, ties to the even code).
 *   codes   uint8 [rows][cols/2] (written): element 2j in the low nibble of
 *           byte j, element 2j+1 in the high nibble. 16-byte aligned.
 *   scales  optional (NULL allowed): FP32 scales [rows][cols/32].
 *   packed  int32 [cols/128][ceil(rows/128)][32][4] (written): byte b of word
 *           [kb][rb][i][j] = biased exponent (log2 s + 127) of row
 *           128 rb + 32 j + i for strip 4 kb + b -- the UE8M0 layout of
 *           dg_quantize_fp8_ue8m0 with 32-wide strips in place of K-blocks.
 *           Bytes of rows past `rows` are not written.
 *   Inputs must be finite. Allocates nothing; asynchronous on `stream`.
 *
 * dg_fp8_fp4_gemm_nt: D = C + A @ B.T on the block-scaled MMA,
 *   D[m][n] = C[m][n] + sum_kb sa(m, kb) * sum_{c<4} sb(n, 4 kb + c) *
 *             sum_{k in strip 4 kb + c} A[m][k] * B[n][k]
 *   A   [M][K] E4M3, sfa its packed UE8M0 scales from dg_quantize_fp8_ue8m0
 *       in ROW_1x128 mode (rows = M);
 *   B   [N][K/2] packed E2M1 and sfb its packed scales, both from
 *       dg_quantize_fp4_e2m1 (rows = N); B 32-byte aligned;
 *   C   [M][N] BF16 or NULL (may alias D); D [M][N] BF16.
 *   K % 128 == 0, N % 8 == 0. Accumulation is the tensor core's FP32 across
 *   all K (no per-K-block promotion). M <= 128 runs the block-scaled swap-AB
 *   split-K kernel, as dg_fp8_gemm_nt_ue8m0 does. Errors as
 *   dg_fp8_gemm_nt_ue8m0.
 * ------------------------------------------------------------------------- */
dg_status dg_quantize_fp4_e2m1(const void* x, int in_dtype, int rows, int cols, void* codes,
                               float* scales, int32_t* packed, void* stream);
dg_status dg_fp8_fp4_gemm_nt(const void* A, const int32_t* sfa, const void* B,
                             const int32_t* sfb, const void* C, void* D, int M, int N, int K,
                             void* stream);

/* ---------------------------------------------------------------------------
 * K-grouped GEMM with the per-group K sizes in DEVICE memory (a training
 * backward captured in a CUDA graph, where the sizes are produced on the GPU
 * and the host cannot read them). Source: README summary, "DenseとGrouped
 * GEMM" (the K-grouped operation); the device-side sizes are this library's
 * extension of it.
 *
 *   ks_dev      [G] int32 DEVICE array of per-group K sizes, read on the
 *               device after the previous kernel on the stream completes.
 *   k_capacity  K rows that A, B (and K/128 rows that sfa, sfb) hold; a
 *               multiple of 128. The groups occupy rows [0, sum ks) of it.
 *   Everything else as dg_k_grouped_fp8_gemm_tn_contiguous. Groups with
 *   K = 0 get D_g = C_g (or 0).
 * Device-side validation: a size that is negative or not a multiple of 128
 * counts as 0, and the running sum is clamped to k_capacity; either case
 * records DG_ERR_INVALID_ARG (site 9) for dg_get_last_device_error(). The
 * call itself reads nothing on the host, so it can be captured in a graph.
 * ------------------------------------------------------------------------- */
dg_status dg_k_grouped_fp8_gemm_tn_contiguous_dev_ks(const void* A, const float* sfa,
                                                     const void* B, const float* sfb,
                                                     const int32_t* ks_dev, int k_capacity,
                                                     const float* C, float* D, int G, int M, int N,
                                                     void* stream);

/* ---------------------------------------------------------------------------
 * Utilities (README summary, section "ユーティリティと環境変数").
 * ------------------------------------------------------------------------- */
/* M alignment every contiguous-layout segment must have: 128. */
int dg_get_mk_alignment_for_contiguous_layout(void);
/* Smallest x >= mn with x * elem_bytes a multiple of 16 (TMA row alignment). */
int dg_get_tma_aligned_size(int mn, int elem_bytes);
/* Cap on the SMs the GEMM kernels use (0 = all SMs of the device). */
void dg_set_num_sms(int n);
int dg_get_num_sms(void);
/* Bounded-wait limit in nanoseconds for subsequent launches (0 = default 2 s). */
void dg_set_wait_timeout_ns(uint64_t ns);
/* Programmatic dependent launch (default on): each launch may start its
 * prologue while the previous kernel on the stream finishes; every kernel of
 * this library waits for its predecessor before reading global memory.
 * Source: README summary, section "ユーティリティと環境変数" (set_pdl / get_pdl). */
void dg_set_pdl(int enable);
int dg_get_pdl(void);

/* Synchronises `stream`, then reads and clears this device's error word.
 * Returns DG_OK, DG_ERR_TIMEOUT (a bounded wait ran out; *site gets the code
 * of the wait that gave up, if site != NULL), DG_ERR_INVALID_ARG (device-side
 * sizes were invalid, site 9) or DG_ERR_CUDA. Debug/test use.
 * The error word is one per device, shared by every stream: it holds the
 * first error any launch on the device recorded since the last read. Call
 * this when no other stream has work of this library in flight; otherwise an
 * error recorded by a launch on another stream may be reported here (or
 * recorded between the read and the clear and lost). */
dg_status dg_get_last_device_error(void* stream, int* site);

/* Test hook: when nonzero, the next GEMM launch drops one producer arrive so
 * that its consumers' bounded waits run out (used to test the timeout path).
 * Reset to 0 after one launch. */
void dg_debug_drop_next_arrive(int enable);

/* Number of kernels this library has launched since load (all devices). */
uint64_t dg_get_launch_count(void);

/* Environment variables (README summary, section "ユーティリティと環境変数",
 * names its DG_PRINT_CONFIGS; the rest override this library's planner, for
 * comparisons; none is needed for correct results):
 *   DG_PRINT_CONFIGS=1   print each launch's plan (tiles, widths, splits) to
 *                        stderr; read once.
 *   DG_FORCE_BN=128|256  tile width of the M > 128 dense and grouped kernels;
 *                        read once.
 *   DG_TAIL_SPLIT=0      no split-K launch for a dense call's partial last
 *                        wave; read once.
 *   DG_PAIR=1            dense M > 128 on CTA pairs (256-row tiles); read once.
 *   DG_PAIR_BN=128|256   tile width of the pair kernel; read once.
 *   DG_DECODE_MINB=1|2, DG_DECODE_SPLITS=s
 *                        CTAs per SM and split count of the M <= 128 kernels;
 *                        read on every call.
 *   DG_DECODE_BNP=64     65..128 tokens as two 64-token tiles on half an SM
 *                        each instead of one 128-token tile (FP8 M <= 128
 *                        kernel); read on every call.
 *   DG_DECODE_PAIR=0|1   128-token tiles of the FP8 M <= 128 kernel on tcgen05
 *                        CTA pairs (two N-tiles, tokens split between the
 *                        pair); read on every call.
 *   DG_DECODE_KG=1|2|4   K-blocks per ring stage (one TMA box each for weights
 *                        and tokens) of the FP8 M <= 128 kernel; read on every
 *                        call.
 *   DG_DECODE_PF=k       weight K-blocks the FP8 M <= 128 kernel keeps
 *                        requested into L2 ahead of its loads (rounded up to
 *                        a multiple of 8, default 64); read on every call.
 *   DG_WIDE_EPI=0|1      dense NT tile kernel with a 3-stage ring and
 *                        whole-tile output staging (default for K <= 1536);
 *                        read on every call.
 *   DG_SMALL_M_TILES=1   FP8 NT with M <= 128 on the 128 x 256 tile kernel,
 *                        every tile split along K over a cluster, instead of
 *                        the swap-AB decode kernel; read on every call. */

#ifdef __cplusplus
}
#endif
#endif /* DG_H */
