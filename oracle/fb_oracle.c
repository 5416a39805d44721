/*
 * fb_oracle.c -- plain, slow fp64 CPU oracle for attention with an additive
 * bias, as described in "FlashBias: Fast Computation of Attention with Bias"
 * (Wu, Guo, Ma, Sun, Wang, Matusik, Long; arXiv 2505.12044).
 *
 * THIS FILE IS TEST INFRASTRUCTURE. Only the test suite, the smoke check and
 * the CPU-baseline leg of the benchmark may load it. The product library
 * (libflashbias) never calls it, and it shares no code, header, table or
 * constant with the CUDA path.
 *
 * What it computes (FlashBias abstract: "an additive bias matrix to the
 * query-key scores"; the softmax form is the one the rebuttal writes for the
 * multiplicative analogue, reply to Reviewer BRmd, Q1 Eq. (1)):
 *
 *   s_ij  = scale * sum_c Q[i,c] K[j,c] + b_ij        for j in J(i)
 *   J(i)  = {0..N-1}, or {0..i} with the causal mask (top-left aligned)
 *   M_i   = max_j s_ij
 *   L_i   = sum_j exp(s_ij - M_i)
 *   O[i,:] = sum_j exp(s_ij - M_i) V[j,:] / L_i
 *   LSE_i = M_i + ln L_i
 *
 * This is the definition written out, row by row, two passes over the keys
 * (max, then sum). No tiling, no online rescaling, no fusion. A row with no
 * visible key (impossible for square causal attention) gets O = 0 and
 * LSE = -inf.
 *
 * The bias b_ij is built element by element from the definition of its kind:
 *   DENSE     b_ij given as an N x N matrix (the "FlashAttention w/ Bias"
 *             input, FlashBias Figure 1(c)).
 *   LOWRANK   b_ij = sum_r phi_q[i,r] phi_k[j,r] (FlashBias Figure 2; the
 *             factor tensors of shape heads x N x R, reply to Reviewer BRmd Q3).
 *   SANDWICH  b_ij = sum_{k=1}^{C/2} cos((i-j) / 10000^{2k/C}) (rebuttal,
 *             reply to Reviewer UJUf, Q1 (1)).
 *   ALIBI     b_ij = -m (i - j) (FlashBias Example 3.4, ALiBi; slope m given).
 *   TOEPLITZ  b_ij = table[i - j + N - 1]: a bias given by its values on the
 *             2N-1 offsets (how a materialised Sandwich or ALiBi bias is
 *             stored), for the dense comparison path.
 *   GRID      tokens on a g x g grid, token n = g*y + x; b_ij =
 *             table[(x_i - x_j + g - 1) * (2g - 1) + (y_i - y_j + g - 1)]: a
 *             bias given by its values on the 2-D offsets (Example 3.5,
 *             spatial distance), for the dense comparison path.
 *
 * Parity of every function here is pinned by the tests in tests/ against
 * closed forms, invariants, a library attention routine and a 50-digit
 * evaluation; none of those pins reuses this code.
 */
#include <math.h>
#ifdef _OPENMP
#include <omp.h>
#endif
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define FBO_BIAS_NONE 0
#define FBO_BIAS_DENSE 1
#define FBO_BIAS_LOWRANK 2
#define FBO_BIAS_SANDWICH 3
#define FBO_BIAS_ALIBI 4
#define FBO_BIAS_TOEPLITZ 5
#define FBO_BIAS_GRID 6

/* Per-head bias description. Pointers refer to fp64 host arrays. */
typedef struct {
  int kind;
  const double *dense; /* DENSE: [N, ld] row-major, b_ij = dense[i*ld + j] */
  int64_t ld;
  const double *phi_q; /* LOWRANK: [N, R] */
  const double *phi_k; /* LOWRANK: [N, R] */
  int R;
  int C;        /* SANDWICH: channel count C (even) */
  double slope; /* ALIBI: m */
  const double *table; /* TOEPLITZ: [2N-1]; GRID: [(2g-1) * (2g-1)] */
  int64_t n;           /* TOEPLITZ: N; GRID: g */
} fbo_bias;

/* b_ij straight from the definition of its kind. */
static double fbo_bias_at(const fbo_bias *b, int64_t i, int64_t j) {
  switch (b->kind) {
  case FBO_BIAS_NONE:
    return 0.0;
  case FBO_BIAS_DENSE:
    return b->dense[i * b->ld + j];
  case FBO_BIAS_LOWRANK: {
    double acc = 0.0;
    for (int r = 0; r < b->R; ++r)
      acc += b->phi_q[i * b->R + r] * b->phi_k[j * b->R + r];
    return acc;
  }
  case FBO_BIAS_SANDWICH: {
    /* Sandwich: sum over k = 1..C/2 of cos((i-j) / 10000^(2k/C)). */
    double acc = 0.0;
    const double delta = (double)(i - j);
    for (int k = 1; k <= b->C / 2; ++k)
      acc += cos(delta / pow(10000.0, 2.0 * k / (double)b->C));
    return acc;
  }
  case FBO_BIAS_ALIBI:
    return -b->slope * (double)(i - j);
  case FBO_BIAS_TOEPLITZ:
    return b->table[i - j + b->n - 1];
  case FBO_BIAS_GRID: {
    const int64_t g = b->n;
    const int64_t dx = i % g - j % g, dy = i / g - j / g;
    return b->table[(dx + g - 1) * (2 * g - 1) + (dy + g - 1)];
  }
  default:
    return NAN;
  }
}

/* Value of the bias of one head at (i, j); exported so that tests can read the
 * definition the oracle uses without a full attention call. */
double fbo_bias_value(const fbo_bias *b, int64_t i, int64_t j) {
  return fbo_bias_at(b, i, j);
}

/* Attention for one head, for the listed query rows.
 *   q [N, d], k [N, d], v [N, d]: fp64 row-major.
 *   rows[nrows]: query indices in [0, N); o [nrows, d], lse [nrows].
 * Returns 0, or -1 on a bad argument. */
int fbo_attention_rows(int64_t N, int d, const double *q, const double *k,
                       const double *v, const fbo_bias *bias, double scale,
                       int causal, const int64_t *rows, int64_t nrows,
                       double *o, double *lse) {
  if (N < 0 || d <= 0 || !q || !k || !v || !bias || !rows || !o || !lse)
    return -1;
  for (int64_t t = 0; t < nrows; ++t)
    if (rows[t] < 0 || rows[t] >= N)
      return -1;

#pragma omp parallel
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
#pragma omp for schedule(dynamic, 4)
    for (int64_t t = 0; t < nrows; ++t) {
      const int64_t i = rows[t];
      const int64_t jmax = causal ? i + 1 : N; /* keys 0..jmax-1 visible */
      double *orow = o + t * d;
      /* scores s_ij = scale * <q_i, k_j> + b_ij */
      for (int64_t j = 0; j < jmax; ++j) {
        double dot = 0.0;
        for (int c = 0; c < d; ++c)
          dot += q[i * d + c] * k[j * d + c];
        s[j] = scale * dot + fbo_bias_at(bias, i, j);
      }
      if (jmax == 0) {
        for (int c = 0; c < d; ++c)
          orow[c] = 0.0;
        lse[t] = -INFINITY;
        continue;
      }
      /* pass 1: row maximum */
      double m = -INFINITY;
      for (int64_t j = 0; j < jmax; ++j)
        if (s[j] > m)
          m = s[j];
      /* pass 2: normaliser and weighted sum of values */
      double l = 0.0;
      for (int c = 0; c < d; ++c)
        orow[c] = 0.0;
      for (int64_t j = 0; j < jmax; ++j) {
        const double p = exp(s[j] - m);
        l += p;
        for (int c = 0; c < d; ++c)
          orow[c] += p * v[j * d + c];
      }
      for (int c = 0; c < d; ++c)
        orow[c] /= l;
      lse[t] = m + log(l);
    }
    free(s);
  }
  return 0;
}

/* Dense bias of one head, [N, N], from its definition (used to hand the same
 * bias to the DENSE path and to check factorisations). */
int fbo_bias_dense(int64_t N, const fbo_bias *bias, double *out) {
  if (N < 0 || !bias || !out)
    return -1;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < N; ++i)
    for (int64_t j = 0; j < N; ++j)
      out[i * N + j] = fbo_bias_at(bias, i, j);
  return 0;
}

/* Exact Sandwich factors (rebuttal, reply to Reviewer UJUf, Q1 (2)):
 *   phi(i) = [cos(i w_1), sin(i w_1), ..., cos(i w_{C/2}), sin(i w_{C/2})],
 *   w_k = 10000^(-2k/C), k = 1..C/2;   phi_q = phi_k = phi.
 * out [N, C] fp64. The pages write the exponent's denominator as a lower-case
 * c in the factor formula and C in the bias formula; both are read as C. */
int fbo_sandwich_factors(int64_t N, int C, double *out) {
  if (N < 0 || C <= 0 || (C % 2) != 0 || !out)
    return -1;
  for (int64_t i = 0; i < N; ++i)
    for (int k = 1; k <= C / 2; ++k) {
      const double w = pow(10000.0, -2.0 * k / (double)C);
      out[i * C + 2 * (k - 1)] = cos((double)i * w);
      out[i * C + 2 * (k - 1) + 1] = sin((double)i * w);
    }
  return 0;
}

/* ALiBi slope of head h (0-based) of H heads: m_h = 2^(-8 (h+1) / H)
 * (FlashBias Example 3.4, ALiBi; the geometric slope sequence with ratio
 * 2^(-8/H) that starts at 2^(-8/H)). */
double fbo_alibi_slope(int h, int H) {
  return pow(2.0, -8.0 * (double)(h + 1) / (double)H);
}

/* Exact rank-2 ALiBi factors of one head (reply to Reviewer BRmd, Q2 (2):
 * Block x 2 factor tiles instead of a Block x Block bias):
 *   phi_q(i) = [-m i, 1],  phi_k(j) = [1, m j]  =>  phi_q(i).phi_k(j) = -m (i - j).
 * phi_q, phi_k: [N, 2] fp64. */
int fbo_alibi_factors(int64_t N, double m, double *phi_q, double *phi_k) {
  if (N < 0 || !phi_q || !phi_k)
    return -1;
  for (int64_t i = 0; i < N; ++i) {
    phi_q[2 * i] = -m * (double)i;
    phi_q[2 * i + 1] = 1.0;
    phi_k[2 * i] = 1.0;
    phi_k[2 * i + 1] = m * (double)i;
  }
  return 0;
}

/* Number of host threads the oracle's parallel loops use. */
int fbo_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
