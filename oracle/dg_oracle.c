/*
 * dg_oracle.c -- plain, slow, obviously correct CPU reference for the FP8
 * fine-grained-scaled GEMM family (dense NT, M-grouped contiguous, M-grouped
 * masked, K-grouped TN) and for the E4M3 quantiser that feeds it.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product library links, loads or
 * calls this file; the product fails loudly when its CUDA library is missing.
 *
 * Arithmetic: decoded E4M3 values and FP32 scales are widened to double and
 * summed in the order the definition states (per 128-wide K-block, the inner
 * product first, then scaled by sfa * sfb and added to the running total, then
 * C). OpenMP only splits independent output elements across threads; no
 * element's arithmetic is reordered.
 *
 * Citations: see dg_oracle.h. Every function is pinned by CPU tests.
 */
#include "dg_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- E4M3 (FN), OFP8 v1.0 section 5.3 ------------------------------------ */

double dgo_e4m3_decode(uint8_t code) {
  int s = (code >> 7) & 1;
  int e = (code >> 3) & 0xF;
  int m = code & 7;
  double v;
  if (e == 15 && m == 7) return NAN;          /* S.1111.111 */
  if (e == 0) v = ldexp((double)m, -9);        /* subnormal: m/8 * 2^(1-7) */
  else v = ldexp(1.0 + m / 8.0, e - 7);        /* normal, bias 7 */
  return s ? -v : v;
}

/* 256-entry decode table, filled once when the library is loaded. */
static double g_tab[256];

__attribute__((constructor)) static void build_table_at_load(void) {
  for (int c = 0; c < 256; ++c) g_tab[c] = dgo_e4m3_decode((uint8_t)c);
}

uint8_t dgo_e4m3_encode(float y) {
  if (isnan(y)) return 0x7F;
  uint8_t sign = signbit(y) ? 0x80 : 0x00;
  double a = fabs((double)y);
  if (a > 448.0) return (uint8_t)(sign | 0x7E);   /* satfinite */
  /* brute force: nearest of the 127 non-negative finite codes */
  int best = 0;
  double best_err = INFINITY;
  for (int c = 0; c <= 0x7E; ++c) {
    double err = fabs(a - g_tab[c]);
    if (err < best_err) { best = c; best_err = err; }
    else if (err == best_err && (c & 1) == 0 && (best & 1) == 1) best = c;  /* tie: even mantissa */
  }
  return (uint8_t)(sign | best);
}

float dgo_bf16_to_f32(uint16_t bits) {
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* ---- quantiser --------------------------------------------------------- */

static float load_x(const void* x, int in_is_bf16, size_t i) {
  if (in_is_bf16) return dgo_bf16_to_f32(((const uint16_t*)x)[i]);
  return ((const float*)x)[i];
}

static float scale_of(float amax) {
  /* IEEE single-precision division (SSE; compiled with -ffp-contract=off) */
  float a = amax > 1e-4f ? amax : 1e-4f;
  return a / 448.0f;
}

/* Power-of-two variant: the smallest power of two >= the FP32 scale above,
 * i.e. 2^ceil(log2 t). frexpf gives t = m * 2^ex with 0.5 <= m < 1, so t is
 * itself a power of two exactly when m == 0.5. */
static float pow2_scale_of(float amax) {
  float t = scale_of(amax);
  int ex = 0;
  float m = frexpf(t, &ex);
  return ldexpf(1.0f, m == 0.5f ? ex - 1 : ex);
}

int dgo_quantize(const void* x, int in_is_bf16, int batch, int rows, int cols,
                 int mode, uint8_t* codes, float* scales, int ld_scales) {
  if (batch < 0 || rows < 0 || cols < 0) return -1;
  int pow2 = mode == DGO_ROW_1x128_POW2 || mode == DGO_BLOCK_128x128_POW2;
  if (pow2) mode -= DGO_ROW_1x128_POW2;  /* same loops, power-of-two scales */
  if (mode == DGO_ROW_1x128) {
    if (cols % 128 != 0 || ld_scales < rows) return -1;
    int kbs = cols / 128;
    for (int b = 0; b < batch; ++b) {
      #pragma omp parallel for schedule(static)
      for (int r = 0; r < rows; ++r) {
        for (int kb = 0; kb < kbs; ++kb) {
          size_t base = ((size_t)b * rows + r) * cols + (size_t)kb * 128;
          float amax = 0.0f;
          for (int j = 0; j < 128; ++j) {
            float v = fabsf(load_x(x, in_is_bf16, base + j));
            if (v > amax) amax = v;
          }
          float s = pow2 ? pow2_scale_of(amax) : scale_of(amax);
          scales[((size_t)b * kbs + kb) * ld_scales + r] = s;
          for (int j = 0; j < 128; ++j) {
            float y = load_x(x, in_is_bf16, base + j) / s;
            codes[base + j] = dgo_e4m3_encode(y);
          }
        }
      }
    }
    return 0;
  }
  if (mode == DGO_BLOCK_128x128) {
    /* a block at the bottom or right edge holds the rows [r0, r1) and the
       columns [c0, c1) that exist */
    int kbs = (cols + 127) / 128, nbs = (rows + 127) / 128;
    for (int b = 0; b < batch; ++b) {
      #pragma omp parallel for collapse(2) schedule(static)
      for (int nb = 0; nb < nbs; ++nb) {
        for (int kb = 0; kb < kbs; ++kb) {
          int r0 = nb * 128, r1 = r0 + 128 < rows ? r0 + 128 : rows;
          int c0 = kb * 128, c1 = c0 + 128 < cols ? c0 + 128 : cols;
          float amax = 0.0f;
          for (int r = r0; r < r1; ++r)
            for (int c = c0; c < c1; ++c) {
              float v = fabsf(load_x(x, in_is_bf16, ((size_t)b * rows + r) * cols + c));
              if (v > amax) amax = v;
            }
          float s = pow2 ? pow2_scale_of(amax) : scale_of(amax);
          scales[((size_t)b * nbs + nb) * kbs + kb] = s;
          for (int r = r0; r < r1; ++r)
            for (int c = c0; c < c1; ++c) {
              size_t i = ((size_t)b * rows + r) * cols + c;
              codes[i] = dgo_e4m3_encode(load_x(x, in_is_bf16, i) / s);
            }
        }
      }
    }
    return 0;
  }
  if (mode == DGO_COL_128x1) {
    if (rows % 128 != 0) return -1;
    int rbs = rows / 128;
    for (int b = 0; b < batch; ++b) {
      #pragma omp parallel for collapse(2) schedule(static)
      for (int rb = 0; rb < rbs; ++rb) {
        for (int c = 0; c < cols; ++c) {
          float amax = 0.0f;
          for (int r = rb * 128; r < rb * 128 + 128; ++r) {
            float v = fabsf(load_x(x, in_is_bf16, ((size_t)b * rows + r) * cols + c));
            if (v > amax) amax = v;
          }
          float s = scale_of(amax);
          scales[((size_t)b * rbs + rb) * cols + c] = s;
          for (int r = rb * 128; r < rb * 128 + 128; ++r) {
            size_t i = ((size_t)b * rows + r) * cols + c;
            codes[i] = dgo_e4m3_encode(load_x(x, in_is_bf16, i) / s);
          }
        }
      }
    }
    return 0;
  }
  return -1;
}

/* ---- GEMMs ------------------------------------------------------------- */

static double load_c(const void* C, int c_kind, size_t i) {
  if (C == NULL || c_kind == DGO_C_NONE) return 0.0;
  if (c_kind == DGO_C_BF16) return (double)dgo_bf16_to_f32(((const uint16_t*)C)[i]);
  return (double)((const float*)C)[i];
}

/* One output row of D = C + A_row @ B.T with per-128 K-block promotion.
 * a_row: K codes; sfa_row(kb) = sfa_col[kb * ld]; B: [N][K]; sfb [nbN][KB]. */
static void nt_row(const uint8_t* a_row, const float* sfa_col, int ld_sfa,
                   const uint8_t* B, const float* sfb, int N, int K,
                   const void* C, int c_kind, size_t c_row_off, double* out) {
  int KB = K / 128;
  for (int n = 0; n < N; ++n) {
    const uint8_t* b_row = B + (size_t)n * K;
    double total = 0.0;
    for (int kb = 0; kb < KB; ++kb) {
      double inner = 0.0;
      for (int k = kb * 128; k < kb * 128 + 128; ++k)
        inner += g_tab[a_row[k]] * g_tab[b_row[k]];
      double scale = (double)sfa_col[(size_t)kb * ld_sfa] * (double)sfb[(size_t)(n / 128) * KB + kb];
      total += scale * inner;
    }
    out[n] = load_c(C, c_kind, c_row_off + n) + total;
  }
}

int dgo_gemm_nt(const uint8_t* A, const float* sfa, int ld_sfa,
                const uint8_t* B, const float* sfb,
                const void* C, int c_kind, double* R,
                int M, int N, int K, const int* rows, int n_rows) {
  if (K % 128 != 0 || ld_sfa < M) return -1;
  if (rows == NULL && n_rows != M) return -1;
  #pragma omp parallel for schedule(dynamic, 1)
  for (int i = 0; i < n_rows; ++i) {
    int m = rows ? rows[i] : i;
    nt_row(A + (size_t)m * K, sfa + m, ld_sfa, B, sfb, N, K, C, c_kind,
           (size_t)m * N, R + (size_t)i * N);
  }
  return 0;
}

/* ---- E2M1 (FP4), OCP MX v1.0 section 5.3.3 --------------------------------- */

double dgo_e2m1_decode(uint8_t code) {
  int s = (code >> 3) & 1;
  int e = (code >> 1) & 3;
  int m = code & 1;
  double v = e == 0 ? 0.5 * m                     /* subnormal: m/2 * 2^(1-1) */
                    : ldexp(1.0 + 0.5 * m, e - 1); /* normal, bias 1 */
  return s ? -v : v;
}

/* 16-entry decode table, filled once when the library is loaded. */
static double g_tab4[16];

__attribute__((constructor)) static void build_table4_at_load(void) {
  for (int c = 0; c < 16; ++c) g_tab4[c] = dgo_e2m1_decode((uint8_t)c);
}

uint8_t dgo_e2m1_encode(float y) {
  uint8_t sign = signbit(y) ? 0x8 : 0x0;
  double a = fabs((double)y);
  if (a > 6.0) return (uint8_t)(sign | 0x7);      /* satfinite */
  /* brute force: nearest of the 8 non-negative codes */
  int best = 0;
  double best_err = INFINITY;
  for (int c = 0; c <= 7; ++c) {
    double err = fabs(a - dgo_e2m1_decode((uint8_t)c));
    if (err < best_err) { best = c; best_err = err; }
    else if (err == best_err && (c & 1) == 0 && (best & 1) == 1) best = c;  /* tie: even code */
  }
  return (uint8_t)(sign | best);
}

/* s = 2^ceil(log2 t), t = max(amax, 1e-4f) / 6 (IEEE single division). */
static float fp4_scale_of(float amax) {
  float a = amax > 1e-4f ? amax : 1e-4f;
  float t = a / 6.0f;
  int ex = 0;
  float m = frexpf(t, &ex);
  return ldexpf(1.0f, m == 0.5f ? ex - 1 : ex);
}

int dgo_quantize_fp4(const void* x, int in_is_bf16, int rows, int cols,
                     uint8_t* codes, float* scales) {
  if (rows < 0 || cols < 0 || cols % 32 != 0) return -1;
  int strips = cols / 32;
  #pragma omp parallel for schedule(static)
  for (int r = 0; r < rows; ++r) {
    for (int c = 0; c < strips; ++c) {
      size_t base = (size_t)r * cols + (size_t)c * 32;
      float amax = 0.0f;
      for (int j = 0; j < 32; ++j) {
        float v = fabsf(load_x(x, in_is_bf16, base + j));
        if (v > amax) amax = v;
      }
      float s = fp4_scale_of(amax);
      scales[(size_t)r * strips + c] = s;
      for (int j = 0; j < 32; j += 2) {
        uint8_t lo = dgo_e2m1_encode(load_x(x, in_is_bf16, base + j) / s);
        uint8_t hi = dgo_e2m1_encode(load_x(x, in_is_bf16, base + j + 1) / s);
        codes[(base + j) / 2] = (uint8_t)(lo | (hi << 4));
      }
    }
  }
  return 0;
}

int dgo_gemm_fp8_fp4_nt(const uint8_t* A, const float* sfa, int ld_sfa,
                        const uint8_t* B, const float* sfb,
                        const void* C, int c_kind, double* R,
                        int M, int N, int K, const int* rows, int n_rows) {
  if (K % 128 != 0 || ld_sfa < M) return -1;
  if (rows == NULL && n_rows != M) return -1;
  int KB = K / 128, strips = K / 32;
  #pragma omp parallel for schedule(dynamic, 1)
  for (int i = 0; i < n_rows; ++i) {
    int m = rows ? rows[i] : i;
    const uint8_t* a = A + (size_t)m * K;
    for (int n = 0; n < N; ++n) {
      const uint8_t* b = B + (size_t)n * (K / 2);
      double total = 0.0;
      for (int kb = 0; kb < KB; ++kb) {
        double blk = 0.0;
        for (int c = 0; c < 4; ++c) {
          int strip = 4 * kb + c;
          double dot = 0.0;
          for (int k = 32 * strip; k < 32 * strip + 32; ++k) {
            uint8_t nib = (k & 1) ? (uint8_t)(b[k / 2] >> 4) : (uint8_t)(b[k / 2] & 0xF);
            dot += g_tab[a[k]] * g_tab4[nib];
          }
          blk += (double)sfb[(size_t)n * strips + strip] * dot;
        }
        total += (double)sfa[(size_t)kb * ld_sfa + m] * blk;
      }
      R[(size_t)i * N + n] = load_c(C, c_kind, (size_t)m * N + n) + total;
    }
  }
  return 0;
}

int dgo_m_grouped_contiguous(const uint8_t* A, const float* sfa, int ld_sfa,
                             const uint8_t* B, const float* sfb,
                             const int32_t* m_indices, const void* C, int c_kind,
                             double* R, int Mt, int N, int K, int G,
                             const int* rows, int n_rows) {
  if (K % 128 != 0 || ld_sfa < Mt) return -1;
  if (rows == NULL && n_rows != Mt) return -1;
  int KB = K / 128, nbN = (N + 127) / 128;
  #pragma omp parallel for schedule(dynamic, 1)
  for (int i = 0; i < n_rows; ++i) {
    int m = rows ? rows[i] : i;
    int g = m_indices[m];
    double* out = R + (size_t)i * N;
    if (g < 0 || g >= G) {
      for (int n = 0; n < N; ++n) out[n] = NAN;
      continue;
    }
    nt_row(A + (size_t)m * K, sfa + m, ld_sfa, B + (size_t)g * N * K,
           sfb + (size_t)g * nbN * KB, N, K, C, c_kind, (size_t)m * N, out);
  }
  return 0;
}

int dgo_m_grouped_masked(const uint8_t* A, const float* sfa, int ld_sfa,
                         const uint8_t* B, const float* sfb,
                         const int32_t* masked_m, double* R,
                         int G, int max_m, int N, int K, int row_stride) {
  if (K % 128 != 0 || ld_sfa < max_m || row_stride < 1) return -1;
  int KB = K / 128, nbN = (N + 127) / 128;
  #pragma omp parallel for collapse(2) schedule(dynamic, 1)
  for (int g = 0; g < G; ++g) {
    for (int m = 0; m < max_m; ++m) {
      double* out = R + ((size_t)g * max_m + m) * N;
      int valid = masked_m[g] < max_m ? masked_m[g] : max_m;
      if (m >= valid || (m % row_stride) != 0) {
        for (int n = 0; n < N; ++n) out[n] = NAN;
        continue;
      }
      nt_row(A + ((size_t)g * max_m + m) * K, sfa + (size_t)g * KB * ld_sfa + m,
             ld_sfa, B + (size_t)g * N * K, sfb + (size_t)g * nbN * KB, N, K,
             NULL, DGO_C_NONE, 0, out);
    }
  }
  return 0;
}

int dgo_k_grouped_tn(const uint8_t* A, const float* sfa, const uint8_t* B,
                     const float* sfb, const int* ks, const float* C,
                     double* R, int G, int M, int N,
                     const int* rows, int n_rows) {
  if (rows == NULL && n_rows != M) return -1;
  for (int g = 0; g < G; ++g)
    if (ks[g] < 0 || ks[g] % 128 != 0) return -1;
  long koff = 0;
  for (int g = 0; g < G; ++g) {
    int KB = ks[g] / 128;
    long kb0 = koff / 128;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < n_rows; ++i) {
      int m = rows ? rows[i] : i;
      double* out = R + ((size_t)g * n_rows + i) * N;
      double* inner = (double*)calloc((size_t)N, sizeof(double));
      double* total = (double*)calloc((size_t)N, sizeof(double));
      for (int kb = 0; kb < KB; ++kb) {
        /* inner[n] = sum_{k in kb} dec(A[k][m]) * dec(B[k][n]); the loop over
           n is outermost per k only to walk B rows contiguously -- each
           element still sums its k terms in increasing k order. */
        for (int n = 0; n < N; ++n) inner[n] = 0.0;
        for (int kk = 0; kk < 128; ++kk) {
          size_t k = (size_t)koff + (size_t)kb * 128 + kk;
          double a = g_tab[A[k * M + m]];
          const uint8_t* b_row = B + k * N;
          for (int n = 0; n < N; ++n) inner[n] += a * g_tab[b_row[n]];
        }
        double sa = (double)sfa[(size_t)(kb0 + kb) * M + m];
        const float* sb = sfb + (size_t)(kb0 + kb) * N;
        for (int n = 0; n < N; ++n) total[n] += (sa * (double)sb[n]) * inner[n];
      }
      for (int n = 0; n < N; ++n) {
        double c = C ? (double)C[((size_t)g * M + m) * N + n] : 0.0;
        out[n] = c + total[n];
      }
      free(inner);
      free(total);
    }
    koff += ks[g];
  }
  return 0;
}

double dgo_calc_diff(const double* D, const double* R, size_t n) {
  double num = 0.0, den = 0.0;
  for (size_t i = 0; i < n; ++i) {
    if (isnan(R[i])) continue;
    num += D[i] * R[i];
    den += D[i] * D[i] + R[i] * R[i];
  }
  if (den == 0.0) return 0.0;
  return 1.0 - 2.0 * num / den;
}

int dgo_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
