/*
 * oracle.c -- plain fp64 CPU oracle for exact scaled-dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path
 * (the CUDA library and its binding) never calls it and shares no code,
 * header, table or helper with it.
 *
 * What it computes is the plain definition of attention, because the tiled
 * method reaches exactly that result (up to rounding order):
 *
 *   - standard attention: S = Q K^T, softmax over each row of S, O = P V,
 *     with S and P materialised as full N x N matrices
 *     ("FlashAttention分块计算优化Transformer显存效率", section 1.1, the
 *     three-step standard flow);
 *   - softmax(x)_i = exp(x_i) / sum_j exp(x_j)  (same page, section 3.1);
 *   - the 1/sqrt(d) factor multiplies the product Q K^T (same page, section
 *     1.1 code and section 3.2 code: "S_block = Q_block @ K_block.T / sqrt(d)");
 *     here it is the caller's `scale`;
 *   - the blockwise result equals the global softmax exactly
 *     ("图解Flash Attention运算原理", section 分块 Softmax 步骤, last sentence);
 *   - causal mode: key j is visible to query i iff j <= i (lower triangle,
 *     "FlashAttention分块计算优化Transformer显存效率", section 2.2);
 *   - what the backward keeps: per-row statistics only, recomputing P
 *     ("图解Flash Attention运算原理", 总结: Recomputation).  The stored
 *     statistic is LSE_i = m_i + ln Z_i (natural log, of the scaled logits).
 *
 * The gradient formulas are not on the pages; they are the analytic gradient
 * of the definition above for the loss L = sum(dO * O):
 *   dV = P^T dO,  dP = dO V^T,  D_i = sum_j P_ij dP_ij,
 *   dS = P * (dP - D),  dQ = scale dS K,  dK = scale dS^T Q.
 *
 * Layout: every tensor is a contiguous double array [B, H, N, d] (row-major);
 * LSE and D are [B, H, N].  Summation orders are the textbook ones (over the
 * contraction index, ascending).  Rows are independent, so OpenMP splits the
 * rows (or, for column sums, the columns) of one head across threads; no
 * value's arithmetic depends on the split.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_EINVAL -1
#define ORACLE_ENOMEM -2

static int bad_sizes(int B, int H, int N, int d) {
  return B <= 0 || H <= 0 || N <= 0 || d <= 0;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* Scores of one head: S[i][j] = scale * sum_c Q[i][c] K[j][c]; causal
 * entries above the diagonal are -inf.  Kt is K transposed ([d][N]) so that
 * the loop over j runs along contiguous memory; each S[i][j] still sums its
 * products in ascending c. */
static void head_scores(const double* Q, const double* Kt, int N, int d,
                        int causal, double scale, double* S) {
#pragma omp parallel for schedule(static)
  for (int i = 0; i < N; ++i) {
    double* s = S + (size_t)i * N;
    for (int j = 0; j < N; ++j) s[j] = 0.0;
    for (int c = 0; c < d; ++c) {
      const double q = Q[(size_t)i * d + c];
      const double* kt = Kt + (size_t)c * N;
      for (int j = 0; j < N; ++j) s[j] += q * kt[j];
    }
    for (int j = 0; j < N; ++j) s[j] = (causal && j > i) ? -INFINITY : s[j] * scale;
  }
}

static void transpose(const double* X, int N, int d, double* Xt) {
  for (int i = 0; i < N; ++i)
    for (int c = 0; c < d; ++c) Xt[(size_t)c * N + i] = X[(size_t)i * d + c];
}

/* Row softmax of a materialised score matrix, in place: S becomes P.
 * Also returns m_i (row max) and LSE_i = m_i + ln Z_i. */
static void head_softmax(double* S, int N, double* lse) {
#pragma omp parallel for schedule(static)
  for (int i = 0; i < N; ++i) {
    double* s = S + (size_t)i * N;
    double m = -INFINITY;
    for (int j = 0; j < N; ++j) m = s[j] > m ? s[j] : m;
    double z = 0.0;
    for (int j = 0; j < N; ++j) z += exp(s[j] - m);
    for (int j = 0; j < N; ++j) s[j] = exp(s[j] - m) / z;
    lse[i] = m + log(z);
  }
}

/* O = P V for one head: O[i][c] = sum_j P[i][j] V[j][c]. */
static void head_pv(const double* P, const double* V, int N, int d, double* O) {
#pragma omp parallel for schedule(static)
  for (int i = 0; i < N; ++i) {
    double* o = O + (size_t)i * d;
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    const double* p = P + (size_t)i * N;
    for (int j = 0; j < N; ++j) {
      const double pij = p[j];
      const double* v = V + (size_t)j * d;
      for (int c = 0; c < d; ++c) o[c] += pij * v[c];
    }
  }
}

/* Full forward: O [B,H,N,d] and LSE [B,H,N].  Materialises S (N x N). */
int oracle_forward(const double* Q, const double* K, const double* V, int B,
                   int H, int N, int d, int causal, double scale, double* O,
                   double* LSE) {
  if (!Q || !K || !V || !O || !LSE || bad_sizes(B, H, N, d)) return ORACLE_EINVAL;
  double* S = (double*)malloc(sizeof(double) * (size_t)N * N);
  double* Kt = (double*)malloc(sizeof(double) * (size_t)N * d);
  if (!S || !Kt) { free(S); free(Kt); return ORACLE_ENOMEM; }
  const size_t hs = (size_t)N * d;
  for (int bh = 0; bh < B * H; ++bh) {
    transpose(K + bh * hs, N, d, Kt);
    head_scores(Q + bh * hs, Kt, N, d, causal, scale, S);
    head_softmax(S, N, LSE + (size_t)bh * N);
    head_pv(S, V + bh * hs, N, d, O + bh * hs);
  }
  free(S);
  free(Kt);
  return ORACLE_OK;
}

/* The attention probabilities P of one head (b, h), N x N, for tests that
 * check row sums and the worked example. */
int oracle_probs(const double* Q, const double* K, int B, int H, int N, int d,
                 int causal, double scale, int bh, double* P) {
  if (!Q || !K || !P || bad_sizes(B, H, N, d) || bh < 0 || bh >= B * H) return ORACLE_EINVAL;
  double* Kt = (double*)malloc(sizeof(double) * (size_t)N * d);
  double* lse = (double*)malloc(sizeof(double) * (size_t)N);
  if (!Kt || !lse) { free(Kt); free(lse); return ORACLE_ENOMEM; }
  const size_t hs = (size_t)N * d;
  transpose(K + bh * hs, N, d, Kt);
  head_scores(Q + bh * hs, Kt, N, d, causal, scale, P);
  head_softmax(P, N, lse);
  free(Kt);
  free(lse);
  return ORACLE_OK;
}

/* One output row of the definition: row i of head bh.  Computes the score
 * row, its max, Z, and O_i = sum_j exp(s_j - m) V_j / Z.  `s` is scratch of N. */
static void one_row(const double* Qh, const double* Kh, const double* Vh,
                    int N, int d, int causal, double scale, int i, double* s,
                    double* o, double* lse) {
  const double* q = Qh + (size_t)i * d;
  double m = -INFINITY;
  for (int j = 0; j < N; ++j) {
    if (causal && j > i) { s[j] = -INFINITY; continue; }
    const double* k = Kh + (size_t)j * d;
    double acc = 0.0;
    for (int c = 0; c < d; ++c) acc += q[c] * k[c];
    s[j] = acc * scale;
    m = s[j] > m ? s[j] : m;
  }
  double z = 0.0;
  for (int j = 0; j < N; ++j) z += exp(s[j] - m);
  for (int c = 0; c < d; ++c) o[c] = 0.0;
  for (int j = 0; j < N; ++j) {
    const double p = exp(s[j] - m) / z;
    const double* v = Vh + (size_t)j * d;
    for (int c = 0; c < d; ++c) o[c] += p * v[c];
  }
  *lse = m + log(z);
}

/* Forward restricted to listed rows: rows[r] = bh * N + i.  O_rows is
 * [n_rows, d], LSE_rows is [n_rows].  Each row is computed on its own from
 * the definition, so any row of any size of problem can be checked. */
int oracle_forward_rows(const double* Q, const double* K, const double* V,
                        int B, int H, int N, int d, int causal, double scale,
                        int n_rows, const int64_t* rows, double* O_rows,
                        double* LSE_rows) {
  if (!Q || !K || !V || !rows || !O_rows || !LSE_rows || bad_sizes(B, H, N, d) || n_rows < 0)
    return ORACLE_EINVAL;
  for (int r = 0; r < n_rows; ++r)
    if (rows[r] < 0 || rows[r] >= (int64_t)B * H * N) return ORACLE_EINVAL;
  int err = 0;
#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)N);
    if (!s) {
#pragma omp atomic write
      err = 1;
    } else {
#pragma omp for schedule(dynamic)
      for (int r = 0; r < n_rows; ++r) {
        const int64_t bh = rows[r] / N;
        const int i = (int)(rows[r] % N);
        const size_t off = (size_t)bh * N * d;
        one_row(Q + off, K + off, V + off, N, d, causal, scale, i, s,
                O_rows + (size_t)r * d, LSE_rows + r);
      }
      free(s);
    }
  }
  return err ? ORACLE_ENOMEM : ORACLE_OK;
}

/* Full backward of one head from the definition (S, P, dP and dS are all
 * materialised).  D is the definitional D_i = sum_j P_ij dP_ij unless
 * O_for_D is given, in which case D_i = sum_c dO_ic O_for_D_ic (the
 * rowsum(dO * O) form, with the O the caller supplies). */
static int head_backward(const double* Qh, const double* Kh, const double* Vh,
                         const double* dOh, const double* OforD, int N, int d,
                         int causal, double scale, double* dQh, double* dKh,
                         double* dVh, double* Dh, double* D2h, double* Oh,
                         double* lseh) {
  double* P = (double*)malloc(sizeof(double) * (size_t)N * N);
  double* dS = (double*)malloc(sizeof(double) * (size_t)N * N);
  double* Xt = (double*)malloc(sizeof(double) * (size_t)N * d);
  if (!P || !dS || !Xt) { free(P); free(dS); free(Xt); return ORACLE_ENOMEM; }
  /* forward quantities */
  transpose(Kh, N, d, Xt);
  head_scores(Qh, Xt, N, d, causal, scale, P);
  head_softmax(P, N, lseh);
  head_pv(P, Vh, N, d, Oh);
  /* dP = dO V^T, the same contraction as the scores with (dO, V), no scale */
  transpose(Vh, N, d, Xt);
  head_scores(dOh, Xt, N, d, 0, 1.0, dS);
#pragma omp parallel for schedule(static)
  for (int i = 0; i < N; ++i) {
    const double* p = P + (size_t)i * N;
    const double* dp = dS + (size_t)i * N;
    double acc = 0.0;
    for (int j = 0; j < N; ++j) acc += p[j] * dp[j];
    Dh[i] = acc;
    double acc2 = 0.0;
    for (int c = 0; c < d; ++c) acc2 += dOh[(size_t)i * d + c] * Oh[(size_t)i * d + c];
    D2h[i] = acc2;
  }
  /* dS = P * (dP - D) */
#pragma omp parallel for schedule(static)
  for (int i = 0; i < N; ++i) {
    double Di = Dh[i];
    if (OforD) {
      Di = 0.0;
      for (int c = 0; c < d; ++c) Di += dOh[(size_t)i * d + c] * OforD[(size_t)i * d + c];
    }
    const double* p = P + (size_t)i * N;
    double* ds = dS + (size_t)i * N;
    for (int j = 0; j < N; ++j) ds[j] = p[j] * (ds[j] - Di);
  }
  /* dQ = scale dS K */
#pragma omp parallel for schedule(static)
  for (int i = 0; i < N; ++i) {
    double* g = dQh + (size_t)i * d;
    for (int c = 0; c < d; ++c) g[c] = 0.0;
    const double* ds = dS + (size_t)i * N;
    for (int j = 0; j < N; ++j) {
      const double w = ds[j];
      const double* k = Kh + (size_t)j * d;
      for (int c = 0; c < d; ++c) g[c] += w * k[c];
    }
    for (int c = 0; c < d; ++c) g[c] *= scale;
  }
  /* dK = scale dS^T Q and dV = P^T dO: column j sums over rows i */
#pragma omp parallel for schedule(static)
  for (int j = 0; j < N; ++j) {
    double* gk = dKh + (size_t)j * d;
    double* gv = dVh + (size_t)j * d;
    for (int c = 0; c < d; ++c) { gk[c] = 0.0; gv[c] = 0.0; }
    for (int i = 0; i < N; ++i) {
      const double ds = dS[(size_t)i * N + j];
      const double p = P[(size_t)i * N + j];
      const double* q = Qh + (size_t)i * d;
      const double* g = dOh + (size_t)i * d;
      for (int c = 0; c < d; ++c) { gk[c] += ds * q[c]; gv[c] += p * g[c]; }
    }
    for (int c = 0; c < d; ++c) gk[c] *= scale;
  }
  free(P);
  free(dS);
  free(Xt);
  return ORACLE_OK;
}

/* Full backward over all heads.  Outputs dQ, dK, dV [B,H,N,d]; D (the
 * definitional sum_j P dP, or the rowsum form over O_for_D when given),
 * D_rowsum = sum_c dO O with the oracle's own O, and the oracle's O and LSE. */
int oracle_backward(const double* Q, const double* K, const double* V,
                    const double* dO, const double* O_for_D, int B, int H,
                    int N, int d, int causal, double scale, double* dQ,
                    double* dK, double* dV, double* D, double* D_rowsum,
                    double* O, double* LSE) {
  if (!Q || !K || !V || !dO || !dQ || !dK || !dV || !D || !D_rowsum || !O || !LSE ||
      bad_sizes(B, H, N, d))
    return ORACLE_EINVAL;
  const size_t hs = (size_t)N * d;
  for (int bh = 0; bh < B * H; ++bh) {
    int rc = head_backward(Q + bh * hs, K + bh * hs, V + bh * hs, dO + bh * hs,
                           O_for_D ? O_for_D + bh * hs : NULL, N, d, causal, scale,
                           dQ + bh * hs, dK + bh * hs, dV + bh * hs, D + (size_t)bh * N,
                           D_rowsum + (size_t)bh * N, O + bh * hs, LSE + (size_t)bh * N);
    if (rc) return rc;
  }
  return ORACLE_OK;
}

/* Backward restricted to samples of one head bh: dQ for the listed query
 * rows, dK and dV for the listed key rows.  Every row's LSE and D is needed
 * (P_ij = exp(S_ij - LSE_i) and dS_ij = P_ij (dP_ij - D_i) for all i), so
 * those are computed for the whole head, row by row, without materialising
 * S; the sampled gradient rows then follow their definitions.  D is the
 * definitional sum_j P_ij dP_ij, or the rowsum form over O_for_D (a whole
 * [B,H,N,d] array) when that is given. */
int oracle_backward_sampled(const double* Q, const double* K, const double* V,
                            const double* dO, const double* O_for_D, int B,
                            int H, int N, int d, int causal, double scale,
                            int bh, int n_q, const int64_t* q_rows, int n_k,
                            const int64_t* k_rows, double* dQ_rows,
                            double* dK_rows, double* dV_rows, double* lse_out,
                            double* D_out) {
  if (!Q || !K || !V || !dO || bad_sizes(B, H, N, d) || bh < 0 || bh >= B * H ||
      n_q < 0 || n_k < 0 || (n_q && (!q_rows || !dQ_rows)) ||
      (n_k && (!k_rows || !dK_rows || !dV_rows)) || !lse_out || !D_out)
    return ORACLE_EINVAL;
  for (int r = 0; r < n_q; ++r) if (q_rows[r] < 0 || q_rows[r] >= N) return ORACLE_EINVAL;
  for (int r = 0; r < n_k; ++r) if (k_rows[r] < 0 || k_rows[r] >= N) return ORACLE_EINVAL;
  const size_t off = (size_t)bh * N * d;
  const double* Qh = Q + off; const double* Kh = K + off;
  const double* Vh = V + off; const double* dOh = dO + off;
  int err = 0;
  /* per-row statistics for the whole head */
#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)N);
    double* o = (double*)malloc(sizeof(double) * (size_t)d);
    if (!s || !o) {
#pragma omp atomic write
      err = 1;
    } else {
#pragma omp for schedule(dynamic, 16)
      for (int i = 0; i < N; ++i) {
        one_row(Qh, Kh, Vh, N, d, causal, scale, i, s, o, lse_out + i);
        double Di = 0.0;
        if (O_for_D) {
          for (int c = 0; c < d; ++c) Di += dOh[(size_t)i * d + c] * O_for_D[off + (size_t)i * d + c];
        } else {
          /* D_i = sum_j P_ij dP_ij with dP_ij = dO_i . V_j */
          for (int j = 0; j < N; ++j) {
            const double p = exp(s[j] - lse_out[i]);
            if (p == 0.0) continue;
            double dp = 0.0;
            for (int c = 0; c < d; ++c) dp += dOh[(size_t)i * d + c] * Vh[(size_t)j * d + c];
            Di += p * dp;
          }
        }
        D_out[i] = Di;
      }
    }
    free(s);
    free(o);
  }
  if (err) return ORACLE_ENOMEM;
  /* sampled dQ rows: dQ_i = scale sum_j P_ij (dP_ij - D_i) K_j */
#pragma omp parallel for schedule(dynamic)
  for (int r = 0; r < n_q; ++r) {
    const int i = (int)q_rows[r];
    double* g = dQ_rows + (size_t)r * d;
    for (int c = 0; c < d; ++c) g[c] = 0.0;
    for (int j = 0; j < N; ++j) {
      if (causal && j > i) continue;
      double sc = 0.0, dp = 0.0;
      for (int c = 0; c < d; ++c) sc += Qh[(size_t)i * d + c] * Kh[(size_t)j * d + c];
      for (int c = 0; c < d; ++c) dp += dOh[(size_t)i * d + c] * Vh[(size_t)j * d + c];
      const double p = exp(sc * scale - lse_out[i]);
      const double ds = p * (dp - D_out[i]);
      for (int c = 0; c < d; ++c) g[c] += ds * Kh[(size_t)j * d + c];
    }
    for (int c = 0; c < d; ++c) g[c] *= scale;
  }
  /* sampled dK, dV rows: sums over queries i of column j */
#pragma omp parallel for schedule(dynamic)
  for (int r = 0; r < n_k; ++r) {
    const int j = (int)k_rows[r];
    double* gk = dK_rows + (size_t)r * d;
    double* gv = dV_rows + (size_t)r * d;
    for (int c = 0; c < d; ++c) { gk[c] = 0.0; gv[c] = 0.0; }
    for (int i = 0; i < N; ++i) {
      if (causal && j > i) continue;
      double sc = 0.0, dp = 0.0;
      for (int c = 0; c < d; ++c) sc += Qh[(size_t)i * d + c] * Kh[(size_t)j * d + c];
      for (int c = 0; c < d; ++c) dp += dOh[(size_t)i * d + c] * Vh[(size_t)j * d + c];
      const double p = exp(sc * scale - lse_out[i]);
      const double ds = p * (dp - D_out[i]);
      for (int c = 0; c < d; ++c) {
        gk[c] += ds * Qh[(size_t)i * d + c];
        gv[c] += p * dOh[(size_t)i * d + c];
      }
    }
    for (int c = 0; c < d; ++c) gk[c] *= scale;
  }
  return ORACLE_OK;
}
