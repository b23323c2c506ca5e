/*
 * dg_oracle.h -- plain CPU reference ("oracle") for the FP8 fine-grained-scaled
 * GEMM family described on the DeepGEMM pages. TEST INFRASTRUCTURE ONLY: only
 * tests, the smoke check and the benchmark's CPU-baseline leg may load it. It
 * shares no code, header, table or helper with the CUDA library.
 *
 * Sources (page title, section):
 *   - "DeepGEMM" README summary (ja.news.hada.io topic 19459), section
 *     "GEMMインターフェースとレイアウト制約": D = C + A @ B.T with NT as the base
 *     layout; LHS scaling factors TMA-aligned and transposed; FP32 scales.
 *   - same page, section "DenseとGrouped GEMM": M-grouped contiguous layout
 *     (segments aligned to the M block), masked layout (only rows below the
 *     per-group count are computed), K-grouped TN for the MoE weight gradient.
 *   - "DeepSeek開源新突破：DeepGEMM庫揭秘" (picoinsstore.com), paragraph 2:
 *     two-level accumulation (promotion) because the FP8 tensor-core
 *     accumulator is imprecise.
 *   - E4M3 "FN" encoding: OCP 8-bit Floating Point Specification (OFP8) v1.0,
 *     section 5.3 (bias 7, no infinities, S.1111.111 is NaN, max 448).
 *
 * All GEMM arithmetic is FP64 on decoded bytes. Every function here is
 * "parity pinned" by CPU tests against closed forms, library routines and
 * invariants (see tests/test_oracle_*.py).
 */
#ifndef DG_ORACLE_H
#define DG_ORACLE_H
#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* E4M3 (FN) byte -> value, from the OFP8 definition. NaN for 0x7F/0xFF. */
double dgo_e4m3_decode(uint8_t code);

/* Nearest finite E4M3 value to y, ties to even mantissa, |y| > 448 saturates
 * to +-448, NaN -> 0x7F. Sign bit is copied from y (so -tiny -> 0x80). */
uint8_t dgo_e4m3_encode(float y);

/* bf16 bit pattern -> float (exact). */
float dgo_bf16_to_f32(uint16_t bits);

/* Quantisation modes (same numbering as the library ABI, re-declared here). */
enum { DGO_ROW_1x128 = 0, DGO_BLOCK_128x128 = 1, DGO_COL_128x1 = 2 };
/* Power-of-two (UE8M0) variants of ROW and BLOCK: the scale is rounded up to
 * the next power of two, s = 2^ceil(log2(max(amax, 1e-4f) / 448)), so that it
 * is exactly representable as a UE8M0 byte (the README summary's packed UE8M0
 * scales, "GEMMインターフェースとレイアウト制約") and no code saturates. Same
 * scale layouts as ROW / BLOCK. */
enum { DGO_ROW_1x128_POW2 = 3, DGO_BLOCK_128x128_POW2 = 4 };

/*
 * Quantise x[batch][rows][cols] (float if in_is_bf16 == 0, bf16 bits
 * otherwise) into E4M3 codes[batch][rows][cols] and FP32 scales:
 *   ROW_1x128    : one scale per (row, 128-column strip); cols % 128 == 0;
 *                  scales[b][cols/128][ld_scales] (transposed, "MN-major").
 *   BLOCK_128x128: one scale per 128x128 block; blocks at the bottom and
 *                  right edges cover only the rows and columns that exist
 *                  (their amax is taken over those elements);
 *                  scales[b][ceil(rows/128)][ceil(cols/128)].
 *   COL_128x1    : one scale per (128-row strip, column); rows % 128 == 0;
 *                  scales[b][rows/128][cols].
 * scale = max(amax, 1e-4f) / 448.0f and code = E4M3(x / scale), both IEEE
 * float divisions. Returns 0, or -1 on an invalid argument.
 */
int dgo_quantize(const void* x, int in_is_bf16, int batch, int rows, int cols,
                 int mode, uint8_t* codes, float* scales, int ld_scales);

/* ---- FP8 x FP4 (mixed precision) -------------------------------------------
 * Sources: README summary (ja.news.hada.io topic 19459), section on the
 * 2026-04 update (FP8xFP4 GEMM) and section "GEMMインターフェースとレイアウト
 * 制約" (SM100 scaling factors are packed UE8M0); "DeepGEMM技术解析" (mlqm.cn),
 * section 5.2 (FP8xFP4 -> BF16). The pages fix neither the FP4 encoding nor
 * its scale granularity; this oracle takes FP4 = E2M1 as defined by the OCP
 * Microscaling Formats (MX) Specification v1.0, section 5.3.3 (1 sign bit,
 * 2 exponent bits with bias 1, 1 mantissa bit, no Inf/NaN, max 6), with one
 * power-of-two scale per 32 consecutive K elements of a row (the MX block
 * size of that specification). */

/* E2M1 code (low 4 bits used) -> value. */
double dgo_e2m1_decode(uint8_t code);

/* Nearest E2M1 value to y, ties to the even code, |y| > 6 saturates to +-6.
 * Sign bit copied from y. */
uint8_t dgo_e2m1_encode(float y);

/*
 * FP4 quantiser: x[rows][cols] (float, or bf16 bits if in_is_bf16) with
 * cols % 32 == 0 -> codes[rows][cols/2] (element 2j in the low nibble of byte
 * j, element 2j+1 in the high nibble) and scales[rows][cols/32], one per
 * (row, 32-column strip): s = 2^ceil(log2 t) with t = max(amax, 1e-4f) / 6.0f
 * (IEEE float division), code = E2M1(x / s). Returns 0 or -1.
 */
int dgo_quantize_fp4(const void* x, int in_is_bf16, int rows, int cols,
                     uint8_t* codes, float* scales);

/*
 * FP8 x FP4 NT: R[i][n] = C[m][n] + sum_kb sfa[kb][m] *
 *                 sum_{c < 4} sfb[n][4 kb + c] * sum_{k in strip 4 kb + c}
 *                 dec8(A[m][k]) * dec4(B[n][k]),  m = rows[i]
 * A [M][K] E4M3, sfa [K/128][ld_sfa]; B [N][K/2] packed E2M1 (layout of
 * dgo_quantize_fp4), sfb [N][K/32]; C, R, rows as dgo_gemm_nt. K % 128 == 0.
 */
int dgo_gemm_fp8_fp4_nt(const uint8_t* A, const float* sfa, int ld_sfa,
                        const uint8_t* B, const float* sfb,
                        const void* C, int c_kind, double* R,
                        int M, int N, int K, const int* rows, int n_rows);

/* C operand kinds for the GEMMs below. */
enum { DGO_C_NONE = 0, DGO_C_BF16 = 1, DGO_C_F32 = 2 };

/*
 * Dense NT: R[i][n] = C[m][n] + sum_kb sfa[kb][m] * sfb[n/128][kb] *
 *                     sum_{k in kb} dec(A[m][k]) * dec(B[n][k]),  m = rows[i]
 * A [M][K], sfa [K/128][ld_sfa], B [N][K], sfb [ceil(N/128)][K/128],
 * C [M][N] (kind c_kind), R [n_rows][N] double. rows == NULL means all M rows
 * (n_rows must then equal M).
 */
int dgo_gemm_nt(const uint8_t* A, const float* sfa, int ld_sfa,
                const uint8_t* B, const float* sfb,
                const void* C, int c_kind, double* R,
                int M, int N, int K, const int* rows, int n_rows);

/*
 * M-grouped contiguous: A [Mt][K], sfa [K/128][ld_sfa], B [G][N][K],
 * sfb [G][ceil(N/128)][K/128], m_indices [Mt] (expert id, -1 = padding),
 * C [Mt][N] (nullable), R [n_rows][N]. Padding rows come back as NaN.
 */
int dgo_m_grouped_contiguous(const uint8_t* A, const float* sfa, int ld_sfa,
                             const uint8_t* B, const float* sfb,
                             const int32_t* m_indices, const void* C, int c_kind,
                             double* R, int Mt, int N, int K, int G,
                             const int* rows, int n_rows);

/*
 * M-grouped masked: A [G][max_m][K], sfa [G][K/128][ld_sfa], B [G][N][K],
 * sfb [G][ceil(N/128)][K/128], masked_m [G]; R [G][max_m][N] with rows
 * m >= masked_m[g] set to NaN (not computed). If row_stride > 1 only every
 * row_stride-th valid row (starting at row 0) is computed, the others NaN.
 */
int dgo_m_grouped_masked(const uint8_t* A, const float* sfa, int ld_sfa,
                         const uint8_t* B, const float* sfb,
                         const int32_t* masked_m, double* R,
                         int G, int max_m, int N, int K, int row_stride);

/*
 * K-grouped TN: A [sumK][M], B [sumK][N] (both M/N contiguous),
 * sfa [sumK/128][M], sfb [sumK/128][N], ks[G] (multiples of 128, may be 0).
 * R_g[m][n] = C_g[m][n] + sum_{kb in g} sfa[kb][m] * sfb[kb][n] *
 *             sum_{k in kb} dec(A[k][m]) * dec(B[k][n]).
 * C [G][M][N] float (nullable); R [G][n_rows][N] for the selected rows.
 */
int dgo_k_grouped_tn(const uint8_t* A, const float* sfa, const uint8_t* B,
                     const float* sfb, const int* ks, const float* C,
                     double* R, int G, int M, int N,
                     const int* rows, int n_rows);

/* 1 - 2*sum(D*R) / sum(D^2 + R^2) over pairs where R is not NaN; 0 if the
 * denominator is 0. */
double dgo_calc_diff(const double* D, const double* R, size_t n);

/* Threads the oracle's OpenMP loops use. */
int dgo_num_threads(void);

#ifdef __cplusplus
}
#endif
#endif
