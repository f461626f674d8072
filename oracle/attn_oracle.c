/*
 * attn_oracle.c -- plain fp64 CPU oracle for exact scaled-dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * bench's CPU-baseline leg call this code.  The product path (the CUDA library)
 * never links, loads or calls it, and this file shares nothing with it.
 *
 * What it computes (no tiling, no fusion, no reordering beyond the definition):
 *
 *   Attention definition, "FlashAttention and long context: three ledgers"
 *   section "the problem with standard attention is not only FLOPs":
 *       O = softmax((Q K^T + M) / sqrt(d_h)) V
 *   and the three-step naive form of the FlashAttention-2 tutorial, 2.1.1:
 *       S = Q K^T * scale ; P = softmax(S) along keys ; O = P V.
 *   The scale is a caller argument (the pages use 1/sqrt(d_h)); the 0/-inf mask
 *   M is applied after scaling (same thing for such a mask).
 *
 *   Mask readings (the pages name "causal mask, padding mask or other bias"
 *   and leave the details open):
 *     causal : key j is visible to query i iff j <= i + (Lk - Lq)
 *              (bottom-right alignment; ordinary lower triangle when Lq == Lk)
 *     padding: key j is visible iff j < kv_len (per-sequence key length)
 *     sliding window (with causal, window W > 0): additionally
 *              j > i + (Lk - Lq) - W, i.e. each query sees its W latest keys
 *              (the local causal mask of the pages' mask discussion; W <= 0
 *              means no window)
 *     a row with no visible key has O = 0 and LSE = -inf.
 *
 *   LSE_i = m_i + ln(sum_j exp(S_ij - m_i)) over visible j: the per-row
 *   statistic that the same page says the backward keeps.
 *
 *   Backward (that page only says the backward recomputes score blocks from saved
 *   row statistics; the formulas are the calculus of the definition):
 *       dV = P^T dO ; dP = dO V^T ; D_i = sum_j P_ij dP_ij ;
 *       dS = P o (dP - D) ; dQ = scale dS K ; dK = scale dS^T Q.
 *
 *   Online softmax, for the equivalence pins only (never the parity reference):
 *     unnormalised form of the three-ledgers page ("the key is online softmax"):
 *       m' = max(m, max S_j); l' = e^{m-m'} l + sum_t e^{S_jt - m'};
 *       o' = e^{m-m'} o + sum_t e^{S_jt - m'} V_jt; O = o / l.
 *     normalised merge of the FlashAttention-2 tutorial, 2.1.3:
 *       m = max(m_a, m_b); l = e^{m_a-m} l_a + e^{m_b-m} l_b;
 *       O = (e^{m_a-m} l_a / l) O_a + (e^{m_b-m} l_b / l) O_b.
 *
 * Every row of S and P is materialised in full, in fp64.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static int g_threads = 0;

void oracle_set_threads(int n) { g_threads = n; }

int oracle_get_threads(void) {
#ifdef _OPENMP
  return g_threads > 0 ? g_threads : omp_get_max_threads();
#else
  return 1;
#endif
}

static int is_visible(int i, int j, int Lq, int Lk, int causal, int window, int kv_len) {
  if (j >= kv_len) return 0;
  if (causal && j > i + (Lk - Lq)) return 0;
  if (causal && window > 0 && j <= i + (Lk - Lq) - window) return 0;
  return 1;
}

/* One query row i of one head: fills s[0..Lk) (scaled, -inf where masked) and
 * p[0..Lk) (softmax), returns the number of visible keys; *lse receives LSE_i. */
static int row_probs(const double* Qh, const double* Kh, int i, int Lq, int Lk, int d,
                     double scale, int causal, int window, int kv_len, double* s, double* p,
                     double* lse) {
  const double* q = Qh + (size_t)i * d;
  double m = -INFINITY;
  int nvis = 0;
  for (int j = 0; j < Lk; ++j) {
    if (!is_visible(i, j, Lq, Lk, causal, window, kv_len)) {
      s[j] = -INFINITY;
      continue;
    }
    const double* k = Kh + (size_t)j * d;
    double acc = 0.0;
    for (int c = 0; c < d; ++c) acc += q[c] * k[c];
    s[j] = acc * scale;
    if (s[j] > m) m = s[j];
    ++nvis;
  }
  if (nvis == 0) {
    for (int j = 0; j < Lk; ++j) p[j] = 0.0;
    *lse = -INFINITY;
    return 0;
  }
  double l = 0.0;
  for (int j = 0; j < Lk; ++j) {
    p[j] = (s[j] == -INFINITY) ? 0.0 : exp(s[j] - m);
    l += p[j];
  }
  for (int j = 0; j < Lk; ++j) p[j] /= l;
  *lse = m + log(l);
  return nvis;
}

/* Forward for one (b, h) head.  Qh [Lq,d], Kh/Vh [Lk,d] row-major.
 * rows: the query rows to compute (NULL = all Lq rows, then n_rows = Lq).
 * O_rows [n_rows,d], lse_rows [n_rows]. */
void oracle_fwd_head(const double* Qh, const double* Kh, const double* Vh, int Lq, int Lk,
                     int d, double scale, int causal, int window, int kv_len, const int* rows,
                     int n_rows, double* O_rows, double* lse_rows) {
  if (rows == NULL) n_rows = Lq;
#pragma omp parallel num_threads(oracle_get_threads())
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
    double* p = (double*)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
#pragma omp for schedule(dynamic, 4)
    for (int r = 0; r < n_rows; ++r) {
      int i = rows ? rows[r] : r;
      double lse;
      row_probs(Qh, Kh, i, Lq, Lk, d, scale, causal, window, kv_len, s, p, &lse);
      double* o = O_rows + (size_t)r * d;
      for (int c = 0; c < d; ++c) o[c] = 0.0;
      for (int j = 0; j < Lk; ++j) {
        if (p[j] == 0.0) continue;
        const double* v = Vh + (size_t)j * d;
        for (int c = 0; c < d; ++c) o[c] += p[j] * v[c];
      }
      lse_rows[r] = lse;
    }
    free(s);
    free(p);
  }
}

/* Full probability matrix of one head, P [Lq,Lk] (for row-sum and tiny-case pins). */
void oracle_probs_head(const double* Qh, const double* Kh, int Lq, int Lk, int d, double scale,
                       int causal, int window, int kv_len, double* P, double* lse) {
  double* s = (double*)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
  for (int i = 0; i < Lq; ++i)
    row_probs(Qh, Kh, i, Lq, Lk, d, scale, causal, window, kv_len, s, P + (size_t)i * Lk, lse + i);
  free(s);
}

/* Backward for one (b, h) head, all rows.  dQh [Lq,d] is overwritten; dKh and
 * dVh [Lk,d] are ACCUMULATED into (+=) so grouped query heads sum naturally. */
void oracle_bwd_head(const double* Qh, const double* Kh, const double* Vh, const double* dOh,
                     int Lq, int Lk, int d, double scale, int causal, int window, int kv_len,
                     double* dQh, double* dKh, double* dVh) {
  int nt = oracle_get_threads();
  double* dK_part = (double*)calloc((size_t)nt * Lk * d + 1, sizeof(double));
  double* dV_part = (double*)calloc((size_t)nt * Lk * d + 1, sizeof(double));
#pragma omp parallel num_threads(nt)
  {
    int tid = 0;
#ifdef _OPENMP
    tid = omp_get_thread_num();
#endif
    double* myK = dK_part + (size_t)tid * Lk * d;
    double* myV = dV_part + (size_t)tid * Lk * d;
    double* s = (double*)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
    double* p = (double*)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
    double* dp = (double*)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
#pragma omp for schedule(dynamic, 4)
    for (int i = 0; i < Lq; ++i) {
      double lse;
      const double* q = Qh + (size_t)i * d;
      const double* g = dOh + (size_t)i * d;
      double* dq = dQh + (size_t)i * d;
      for (int c = 0; c < d; ++c) dq[c] = 0.0;
      if (row_probs(Qh, Kh, i, Lq, Lk, d, scale, causal, window, kv_len, s, p, &lse) == 0) continue;
      /* dP_ij = dO_i . V_j ; D_i = sum_j P_ij dP_ij */
      double D = 0.0;
      for (int j = 0; j < Lk; ++j) {
        if (p[j] == 0.0) { dp[j] = 0.0; continue; }
        const double* v = Vh + (size_t)j * d;
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += g[c] * v[c];
        dp[j] = acc;
        D += p[j] * acc;
      }
      for (int j = 0; j < Lk; ++j) {
        if (p[j] == 0.0) continue;
        double ds = p[j] * (dp[j] - D);
        const double* k = Kh + (size_t)j * d;
        double* dk = myK + (size_t)j * d;
        double* dv = myV + (size_t)j * d;
        for (int c = 0; c < d; ++c) {
          dq[c] += scale * ds * k[c];
          dk[c] += scale * ds * q[c];
          dv[c] += p[j] * g[c];
        }
      }
    }
    free(s);
    free(p);
    free(dp);
  }
  for (int t = 0; t < nt; ++t) {
    const double* a = dK_part + (size_t)t * Lk * d;
    const double* b = dV_part + (size_t)t * Lk * d;
    for (size_t e = 0; e < (size_t)Lk * d; ++e) {
      dKh[e] += a[e];
      dVh[e] += b[e];
    }
  }
  free(dK_part);
  free(dV_part);
}

/* Backward of one head evaluated only at sampled outputs: dQ at query rows
 * qrows[0..nq) (written) and dK, dV at key rows kcols[0..nk) (ACCUMULATED).
 * Every query row's P and D are still formed from the full row (as the
 * definition requires); only the outputs are restricted. */
void oracle_bwd_head_sampled(const double* Qh, const double* Kh, const double* Vh,
                             const double* dOh, int Lq, int Lk, int d, double scale, int causal,
                             int window,
                             int kv_len, const int* qrows, int nq, const int* kcols, int nk,
                             double* dQ_rows, double* dK_cols, double* dV_cols) {
  double* lse = (double*)malloc(sizeof(double) * (size_t)(Lq > 0 ? Lq : 1));
  double* D = (double*)malloc(sizeof(double) * (size_t)(Lq > 0 ? Lq : 1));
  int* has = (int*)malloc(sizeof(int) * (size_t)(Lq > 0 ? Lq : 1));
  /* pass 1: per-row LSE and D from full rows of P and dP */
#pragma omp parallel num_threads(oracle_get_threads())
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
    double* p = (double*)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
#pragma omp for schedule(dynamic, 8)
    for (int i = 0; i < Lq; ++i) {
      has[i] = row_probs(Qh, Kh, i, Lq, Lk, d, scale, causal, window, kv_len, s, p, &lse[i]) > 0;
      double acc_D = 0.0;
      const double* g = dOh + (size_t)i * d;
      for (int j = 0; j < Lk; ++j) {
        if (p[j] == 0.0) continue;
        const double* v = Vh + (size_t)j * d;
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += g[c] * v[c];
        acc_D += p[j] * acc;
      }
      D[i] = acc_D;
    }
    free(s);
    free(p);
  }
  /* dQ at sampled rows */
#pragma omp parallel for num_threads(oracle_get_threads()) schedule(dynamic, 1)
  for (int r = 0; r < nq; ++r) {
    int i = qrows[r];
    const double* q = Qh + (size_t)i * d;
    const double* g = dOh + (size_t)i * d;
    double* dq = dQ_rows + (size_t)r * d;
    for (int c = 0; c < d; ++c) dq[c] = 0.0;
    if (!has[i]) continue;
    for (int j = 0; j < Lk; ++j) {
      if (!is_visible(i, j, Lq, Lk, causal, window, kv_len)) continue;
      const double* k = Kh + (size_t)j * d;
      const double* v = Vh + (size_t)j * d;
      double sc = 0.0, dp = 0.0;
      for (int c = 0; c < d; ++c) { sc += q[c] * k[c]; dp += g[c] * v[c]; }
      double p = exp(sc * scale - lse[i]);
      double ds = p * (dp - D[i]);
      for (int c = 0; c < d; ++c) dq[c] += scale * ds * k[c];
    }
  }
  /* dK, dV at sampled key rows: sums over every query row that sees the key */
#pragma omp parallel for num_threads(oracle_get_threads()) schedule(dynamic, 1)
  for (int r = 0; r < nk; ++r) {
    int j = kcols[r];
    const double* k = Kh + (size_t)j * d;
    const double* v = Vh + (size_t)j * d;
    double* dk = dK_cols + (size_t)r * d;
    double* dv = dV_cols + (size_t)r * d;
    for (int i = 0; i < Lq; ++i) {
      if (!has[i] || !is_visible(i, j, Lq, Lk, causal, window, kv_len)) continue;
      const double* q = Qh + (size_t)i * d;
      const double* g = dOh + (size_t)i * d;
      double sc = 0.0, dp = 0.0;
      for (int c = 0; c < d; ++c) { sc += q[c] * k[c]; dp += g[c] * v[c]; }
      double p = exp(sc * scale - lse[i]);
      double ds = p * (dp - D[i]);
      for (int c = 0; c < d; ++c) {
        dk[c] += scale * ds * q[c];
        dv[c] += p * g[c];
      }
    }
  }
  free(lse);
  free(D);
  free(has);
}

/* Unnormalised online softmax over one score row s[0..n) (entries may be -inf)
 * and values V [n,d], scanning blocks that end (exclusive) at block_end[0..nb),
 * the last of which must be n.  Writes O = o / l and the final (m, l); the
 * running (m, l) after each block go to m_trace / l_trace when non-NULL. */
void oracle_online_row(const double* s, const double* V, int n, int d, const int* block_end,
                       int nb, double* O, double* m_out, double* l_out, double* m_trace,
                       double* l_trace) {
  double m = -INFINITY, l = 0.0;
  double* o = (double*)calloc((size_t)(d > 0 ? d : 1), sizeof(double));
  int start = 0;
  for (int b = 0; b < nb; ++b) {
    int end = block_end[b];
    double bmax = -INFINITY;
    for (int t = start; t < end; ++t)
      if (s[t] > bmax) bmax = s[t];
    double m_new = m > bmax ? m : bmax;
    if (m_new != -INFINITY) {
      double alpha = (m == -INFINITY) ? 0.0 : exp(m - m_new);
      l *= alpha;
      for (int c = 0; c < d; ++c) o[c] *= alpha;
      for (int t = start; t < end; ++t) {
        if (s[t] == -INFINITY) continue;
        double e = exp(s[t] - m_new);
        l += e;
        for (int c = 0; c < d; ++c) o[c] += e * V[(size_t)t * d + c];
      }
      m = m_new;
    }
    if (m_trace) m_trace[b] = m;
    if (l_trace) l_trace[b] = l;
    start = end;
  }
  for (int c = 0; c < d; ++c) O[c] = (l > 0.0) ? o[c] / l : 0.0;
  *m_out = m;
  *l_out = l;
  free(o);
}

/* Normalised merge of two partial results (m_a, l_a, O_a) and (m_b, l_b, O_b). */
void oracle_merge(double m_a, double l_a, const double* O_a, double m_b, double l_b,
                  const double* O_b, int d, double* m, double* l, double* O) {
  double mm = m_a > m_b ? m_a : m_b;
  if (mm == -INFINITY) {
    *m = -INFINITY;
    *l = 0.0;
    for (int c = 0; c < d; ++c) O[c] = 0.0;
    return;
  }
  double wa = (m_a == -INFINITY) ? 0.0 : exp(m_a - mm) * l_a;
  double wb = (m_b == -INFINITY) ? 0.0 : exp(m_b - mm) * l_b;
  double ll = wa + wb;
  for (int c = 0; c < d; ++c) O[c] = (wa / ll) * O_a[c] + (wb / ll) * O_b[c];
  *m = mm;
  *l = ll;
}
