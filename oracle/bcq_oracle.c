/*
 * bcq_oracle.c -- plain, slow, obviously correct fp64 CPU oracle for the
 * multi-precision binary-coded-quantization (BCQ) matmul.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * CPU-baseline leg of bench.py may load this library.  It shares no code,
 * header, table or constant with the CUDA library under bit_gemv_bcq_b200/.
 *
 * What it computes (sources, by page title and section):
 *   - "AnyBCQ: Hardware Efficient Flexible Binary-Coded Quantization for
 *     Multi-Precision LLMs" (Paper-Notes page), section "研究背景与动机 /
 *     切入角度": weights are a linear combination of binary bit-planes,
 *     W_hat = sum_i alpha_i B_i, and p-bit inference uses p planes.
 *   - same page, "方法详解 / 训练策略": asymmetric, group-wise BCQ with g = 128
 *     (the asymmetric offset z is added once per (row, group)).
 *   - same page, "关键设计 / 直接bit-plane运算的CUDA内核": B_i in {-1,+1}, a
 *     p-bit call reads only planes 1..p.
 *   - "BiLoCo: Binary Low-Rank Corrections for Post-Training Quantization",
 *     section "核心思路：修正项只用 +1 和 −1": a +-1 vector times x is a signed
 *     sum of the entries of x.
 *
 * Readings taken where the pages are silent:
 *   bit value 1 -> +1 and 0 -> -1; bit j of 32-bit word w holds column 32w+j
 *   (LSB first); canonical planes are [p_H][N][K/32]; alpha for precision q is
 *   its own fp16 array [N][G][q]; one offset z[N][G] shared by all precisions;
 *   the LUT chunk is 8 consecutive columns, entry b holds
 *   sum_j (2*bit_j(b) - 1) * x[8c + j].
 *
 * Everything is accumulated in double.  fp16 inputs are exact in double.
 * Parallelism (OpenMP over output rows) does not change any result: every
 * output element is summed by one thread in a fixed order.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* IEEE binary16 -> double, written from the format definition:
 * sign (1 bit), exponent (5 bits, bias 15), fraction (10 bits). */
double bcq_oracle_half_to_double(uint16_t h) {
  const int sign = (h >> 15) & 1;
  const int expo = (h >> 10) & 0x1f;
  const int frac = h & 0x3ff;
  double v;
  if (expo == 0) {
    v = ldexp((double)frac, -24);                 /* subnormal: frac * 2^-24 */
  } else if (expo == 31) {
    v = frac ? NAN : INFINITY;
  } else {
    v = ldexp((double)(frac + 1024), expo - 25);  /* (1 + frac/1024) * 2^(e-15) */
  }
  return sign ? -v : v;
}

void bcq_oracle_halves_to_double(const uint16_t* h, double* out, size_t n) {
  for (size_t i = 0; i < n; ++i) out[i] = bcq_oracle_half_to_double(h[i]);
}

/* Bit k of a row of LSB-first packed 32-bit words. */
static int bit_at(const uint32_t* row_words, int k) {
  return (int)((row_words[k / 32] >> (k % 32)) & 1u);
}

/* sum_k (2*bit_k - 1) * x_k : the +-1 "signed sum" of x (BiLoCo page, section
 * "核心思路：修正项只用 +1 和 −1"). */
double bcq_oracle_signed_sum(const double* x, const uint32_t* bits, int n) {
  double acc = 0.0;
  for (int k = 0; k < n; ++k) {
    const double s = bit_at(bits, k) ? 1.0 : -1.0;
    acc += s * x[k];
  }
  return acc;
}

/* LUT of the 256 signed sums of every 8-column chunk of every row of x:
 *   lut[m][c][b] = sum_{j<8} (2*bit_j(b) - 1) * x[m][8c + j]
 * x is fp16 [M][K]; lut is double [M][K/8][256].  K must be a multiple of 8.
 * (AnyBCQ page, "直接bit-plane运算的CUDA内核": partial results of +-x are
 * cached in a lookup table, as in LUT-GEMM.) */
int bcq_oracle_lut(const uint16_t* x, int M, int K, double* lut) {
  if (!x || !lut || M < 0 || K < 0 || K % 8) return 1;
  const int C = K / 8;
  for (int m = 0; m < M; ++m)
    for (int c = 0; c < C; ++c)
      for (int b = 0; b < 256; ++b) {
        double acc = 0.0;
        for (int j = 0; j < 8; ++j) {
          const double xv = bcq_oracle_half_to_double(x[(size_t)m * K + 8 * c + j]);
          acc += (((b >> j) & 1) ? 1.0 : -1.0) * xv;
        }
        lut[((size_t)m * C + c) * 256 + b] = acc;
      }
  return 0;
}

/* Per-group sums of x: S[m][g] = sum_{k in group g} x[m][k].  They multiply
 * the offset z (the asymmetric term). */
int bcq_oracle_group_sums(const uint16_t* x, int M, int K, int group, double* S) {
  if (!x || !S || M < 0 || K < 0 || group <= 0 || K % group) return 1;
  const int G = K / group;
  for (int m = 0; m < M; ++m)
    for (int g = 0; g < G; ++g) {
      double acc = 0.0;
      for (int k = g * group; k < (g + 1) * group; ++k)
        acc += bcq_oracle_half_to_double(x[(size_t)m * K + k]);
      S[(size_t)m * G + g] = acc;
    }
  return 0;
}

/*
 * y[m][s] = sum_k x[m][k] * W_hat_{p_m}[n_s][k],   n_s = rows ? rows[s] : s
 *
 * W_hat_q[n][k] = sum_{i=1..q} alpha_q[n][g][i-1] * (2*bit(planes[i-1][n], k) - 1)
 *                 + z[n][g],                         g = k / group
 *
 * p_m = p for every m when p > 0; otherwise p_m = p_row[m].
 * alpha[q-1] -> fp16 [N][G][q] (needed for every q in use); z -> fp16 [N][G]
 * or NULL (offset 0).  planes -> [p_H][N][K/32] uint32.  y -> double
 * [M][n_out] where n_out = rows ? n_rows : N.
 * Returns 0 on success and a nonzero code for invalid arguments.
 */
int bcq_oracle_gemm(const uint16_t* x, const uint32_t* planes,
                    const uint16_t* const alpha[4], const uint16_t* z, int p,
                    const int32_t* p_row, int M, int N, int K, int p_H,
                    int group, const int32_t* rows, int n_rows, double* y) {
  if (!x || !planes || !alpha || !y) return 1;
  if (M < 0 || N < 0 || K < 0 || p_H < 1 || p_H > 4 || group <= 0) return 2;
  if (K % group || K % 32) return 2;
  if (p < 0 || p > p_H) return 3;
  if (p == 0 && !p_row) return 3;
  int used[5] = {0, 0, 0, 0, 0};
  for (int m = 0; m < M; ++m) {
    const int q = p > 0 ? p : p_row[m];
    if (q < 1 || q > p_H) return 3;
    used[q] = 1;
  }
  for (int q = 1; q <= 4; ++q)
    if (used[q] && !alpha[q - 1]) return 3;
  const int n_out = rows ? n_rows : N;
  if (rows)
    for (int s = 0; s < n_rows; ++s)
      if (rows[s] < 0 || rows[s] >= N) return 2;

  const int G = K / group;
  const int KW = K / 32;

  /* x converted once to double, [M][K]. */
  double* xd = (double*)malloc(sizeof(double) * ((size_t)M * K + 1));
  if (!xd) return 9;
  for (size_t i = 0; i < (size_t)M * K; ++i) xd[i] = bcq_oracle_half_to_double(x[i]);

  int status = 0;
#pragma omp parallel
  {
    /* One reconstructed weight row per precision in use. */
    double* w = (double*)malloc(sizeof(double) * ((size_t)4 * K + 1));
    if (!w) {
#pragma omp atomic write
      status = 9;
    } else {
#pragma omp for schedule(dynamic, 4)
      for (int s = 0; s < n_out; ++s) {
        const int n = rows ? rows[s] : s;
        for (int q = 1; q <= 4; ++q) {
          if (!used[q]) continue;
          double* wq = w + (size_t)(q - 1) * K;
          const uint16_t* aq = alpha[q - 1];
          for (int k = 0; k < K; ++k) {
            const int g = k / group;
            double v = z ? bcq_oracle_half_to_double(z[(size_t)n * G + g]) : 0.0;
            for (int i = 1; i <= q; ++i) {
              const uint32_t* row = planes + ((size_t)(i - 1) * N + n) * KW;
              const double a = bcq_oracle_half_to_double(aq[((size_t)n * G + g) * q + (i - 1)]);
              v += a * (bit_at(row, k) ? 1.0 : -1.0);
            }
            wq[k] = v;
          }
        }
        for (int m = 0; m < M; ++m) {
          const int q = p > 0 ? p : p_row[m];
          const double* wq = w + (size_t)(q - 1) * K;
          const double* xm = xd + (size_t)m * K;
          double acc = 0.0;
          for (int k = 0; k < K; ++k) acc += xm[k] * wq[k];
          y[(size_t)m * n_out + s] = acc;
        }
      }
      free(w);
    }
  }
  free(xd);
  return status;
}

/* Number of OpenMP threads the oracle runs with (for reporting). */
int bcq_oracle_num_threads(void) {
  int n = 1;
#pragma omp parallel
  {
#pragma omp single
    {
#ifdef _OPENMP
      n = omp_get_num_threads();
#endif
    }
  }
  return n;
}
