/*
 * attention_oracle.c -- fp64 CPU oracle for exact scaled dot-product attention
 * and its gradient.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file; only the test-suite, the smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no code, header or constant with the CUDA
 * kernels.
 *
 * What it computes, and where that is defined:
 *   - Attention(Q,K,V) = softmax(scale * Q K^T) V, scale = 1/sqrt(d_k) by
 *     default ("第17讲 Tensor Core、HBM、SRAM 与 FlashAttention", §8.1, the
 *     scaled dot-product attention formula).
 *   - softmax(s_j) = e^{s_j} / sum_t e^{s_t}, evaluated with the row maximum
 *     subtracted for stability (same page, §8.3, first formula and the
 *     sentence on shifting by the row maximum).  The oracle does it in three
 *     passes over a row: max, sum of exponentials, normalise.
 *   - Causal attention (listed in §8.3 of the same page as a case a real
 *     kernel must handle; no formula is given).  Reading: key j is visible to
 *     query i iff j <= i (queries and keys share one length N).
 *   - lse_i = m_i + ln(l_i), the per-row log-sum-exp of the scaled scores.
 *     The page keeps (m, l); lse is the single statistic from which the
 *     backward recomputes P_ij = exp(s_ij - lse_i) ("CS336 Lecture 5 · GPUs,
 *     TPUs" notes, section "FlashAttention 解析", item ② on recomputation).
 *   - The backward is not written on any page (they only say it recomputes
 *     tile by tile).  Reading: the exact gradient of L = sum(O * dO) with
 *     respect to Q, K and V, by plain calculus on the definition:
 *        dV_j  = sum_i P_ij dO_i
 *        dP_ij = dO_i . V_j
 *        D_i   = sum_j P_ij dP_ij          (== dO_i . O_i)
 *        dS_ij = P_ij (dP_ij - D_i)
 *        dQ_i  = scale * sum_j dS_ij K_j
 *        dK_j  = scale * sum_i dS_ij Q_i
 *   - oracle_online_fwd: the online-softmax recurrence of §8.3 of the first
 *     page (running m, l, o; alpha = e^{m - m'}; p = e^{s - m'};
 *     l' = alpha l + sum p; o' = alpha o + p V_tile; O = o / l), written
 *     separately so a test can pin the three-pass definition against it.
 *   - oracle_gemm: the plain matrix product C = A B (the matrix multiply
 *     whose throughput curve the CS336 lecture opens with).
 *   - oracle_decode: the same attention for decode-shaped calls.  The first
 *     page's §9.2 splits inference into prefill (a whole prompt at once) and
 *     decode (one or a few new tokens per step); §9.3 says the KV cache keeps
 *     the keys and values of every earlier token so that decode reads them
 *     instead of recomputing them.  No formula is given; readings:
 *       * a head's cache has L rows, of which the first len_b are valid for
 *         batch b (all L when no lengths are given);
 *       * the Nq queries are the newest Nq positions, so under the causal
 *         mask query i sees keys j <= len_b - Nq + i (the mask's diagonal
 *         ends at the last valid key);
 *       * a query that sees no key gets O = 0 and lse = -inf.
 *
 * Layout: every tensor is [B, H, N, d] row-major (d contiguous), fp64; lse and
 * D are [B, H, N].  All loops are plain; OpenMP only splits independent rows
 * (or key columns) across threads.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef long long i64;

static int visible(int causal, i64 i, i64 j) { return !causal || j <= i; }

/* Scores of one query row against every visible key, and the three passes.
 * s[] receives scale * q.k_j for visible j; returns the number of visible keys
 * (keys 0..cnt-1 are exactly the visible ones). */
static i64 row_scores(const double *qi, const double *k, i64 N, i64 d,
                      double scale, int causal, i64 i, double *s) {
  i64 cnt = causal ? i + 1 : N;
  for (i64 j = 0; j < cnt; ++j) {
    const double *kj = k + j * d;
    double acc = 0.0;
    for (i64 c = 0; c < d; ++c) acc += qi[c] * kj[c];
    s[j] = scale * acc;
  }
  return cnt;
}

/* pass 1 (max) and pass 2 (sum of exp); returns l, writes m. */
static double row_max_sum(const double *s, i64 cnt, double *m_out) {
  double m = -INFINITY;
  for (i64 j = 0; j < cnt; ++j) if (s[j] > m) m = s[j];
  double l = 0.0;
  for (i64 j = 0; j < cnt; ++j) l += exp(s[j] - m);
  *m_out = m;
  return l;
}

/* Forward for one head: o [N,d], lse [N]. */
static void fwd_head(const double *q, const double *k, const double *v, i64 N,
                     i64 d, double scale, int causal, double *o, double *lse) {
#pragma omp parallel
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
#pragma omp for schedule(dynamic, 16)
    for (i64 i = 0; i < N; ++i) {
      i64 cnt = row_scores(q + i * d, k, N, d, scale, causal, i, s);
      double m;
      double l = row_max_sum(s, cnt, &m);
      double *oi = o + i * d;
      for (i64 c = 0; c < d; ++c) oi[c] = 0.0;
      /* pass 3: normalise and mix V */
      for (i64 j = 0; j < cnt; ++j) {
        double p = exp(s[j] - m) / l;
        const double *vj = v + j * d;
        for (i64 c = 0; c < d; ++c) oi[c] += p * vj[c];
      }
      lse[i] = m + log(l);
    }
    free(s);
  }
}

/* O and lse for all B*H heads. */
void oracle_fwd(const double *q, const double *k, const double *v, int B, int H,
                int N, int d, double scale, int causal, double *o, double *lse) {
  i64 hs = (i64)N * d;
  for (i64 bh = 0; bh < (i64)B * H; ++bh)
    fwd_head(q + bh * hs, k + bh * hs, v + bh * hs, N, d, scale, causal,
             o + bh * hs, lse + bh * (i64)N);
}

/* O and lse for selected rows of ONE head (pointers address that head). */
void oracle_fwd_rows(const double *q, const double *k, const double *v, int N,
                     int d, double scale, int causal, const int *rows,
                     int nrows, double *o_rows, double *lse_rows) {
#pragma omp parallel
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
#pragma omp for schedule(dynamic, 1)
    for (int r = 0; r < nrows; ++r) {
      i64 i = rows[r];
      i64 cnt = row_scores(q + i * d, k, N, d, scale, causal, i, s);
      double m;
      double l = row_max_sum(s, cnt, &m);
      double *oi = o_rows + (i64)r * d;
      for (i64 c = 0; c < d; ++c) oi[c] = 0.0;
      for (i64 j = 0; j < cnt; ++j) {
        double p = exp(s[j] - m) / l;
        for (i64 c = 0; c < d; ++c) oi[c] += p * v[j * d + c];
      }
      lse_rows[r] = m + log(l);
    }
    free(s);
  }
}

/* The probability matrix of one head, P [N,N] (zero where masked).  Small N
 * only: used to check that rows sum to one and the mask. */
void oracle_probs(const double *q, const double *k, int N, int d, double scale,
                  int causal, double *P) {
  double *s = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
  for (i64 i = 0; i < N; ++i) {
    i64 cnt = row_scores(q + i * d, k, N, d, scale, causal, i, s);
    double m;
    double l = row_max_sum(s, cnt, &m);
    for (i64 j = 0; j < N; ++j)
      P[i * N + j] = (j < cnt) ? exp(s[j] - m) / l : 0.0;
  }
  free(s);
}

/* Backward for one head.  Recomputes the forward from the definition (it
 * takes no statistic from anyone else), then applies the gradient formulas
 * in the header.  D_i is computed both ways; the largest disagreement between
 * sum_j P_ij dP_ij and dO_i . O_i is returned through *d_gap. */
static void bwd_head(const double *q, const double *k, const double *v,
                     const double *dO, i64 N, i64 d, double scale, int causal,
                     double *dq, double *dk, double *dv, double *D,
                     double *d_gap) {
  double *m_row = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
  double *l_row = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
  double gap = 0.0;
  /* Row statistics, D_i, and dQ_i: everything indexed by the query row. */
#pragma omp parallel reduction(max : gap)
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
    double *orow = (double *)malloc(sizeof(double) * (size_t)(d > 0 ? d : 1));
#pragma omp for schedule(dynamic, 16)
    for (i64 i = 0; i < N; ++i) {
      i64 cnt = row_scores(q + i * d, k, N, d, scale, causal, i, s);
      double m;
      double l = row_max_sum(s, cnt, &m);
      m_row[i] = m;
      l_row[i] = l;
      const double *doi = dO + i * d;
      for (i64 c = 0; c < d; ++c) orow[c] = 0.0;
      double d_pdp = 0.0;
      for (i64 j = 0; j < cnt; ++j) {
        double p = exp(s[j] - m) / l;
        double dp = 0.0;
        for (i64 c = 0; c < d; ++c) dp += doi[c] * v[j * d + c];
        d_pdp += p * dp;
        for (i64 c = 0; c < d; ++c) orow[c] += p * v[j * d + c];
      }
      double d_odo = 0.0;
      for (i64 c = 0; c < d; ++c) d_odo += doi[c] * orow[c];
      D[i] = d_pdp;
      double g = fabs(d_pdp - d_odo);
      if (g > gap) gap = g;
      double *dqi = dq + i * d;
      for (i64 c = 0; c < d; ++c) dqi[c] = 0.0;
      for (i64 j = 0; j < cnt; ++j) {
        double p = exp(s[j] - m) / l;
        double dp = 0.0;
        for (i64 c = 0; c < d; ++c) dp += doi[c] * v[j * d + c];
        double ds = p * (dp - d_pdp);
        for (i64 c = 0; c < d; ++c) dqi[c] += scale * ds * k[j * d + c];
      }
    }
    free(orow);
    free(s);
  }
  /* dK_j and dV_j: everything indexed by the key row. */
#pragma omp parallel for schedule(dynamic, 16)
  for (i64 j = 0; j < N; ++j) {
    double *dkj = dk + j * d, *dvj = dv + j * d;
    for (i64 c = 0; c < d; ++c) { dkj[c] = 0.0; dvj[c] = 0.0; }
    const double *kj = k + j * d, *vj = v + j * d;
    for (i64 i = causal ? j : 0; i < N; ++i) {
      if (!visible(causal, i, j)) continue;
      const double *qi = q + i * d, *doi = dO + i * d;
      double sc = 0.0, dp = 0.0;
      for (i64 c = 0; c < d; ++c) { sc += qi[c] * kj[c]; dp += doi[c] * vj[c]; }
      double p = exp(scale * sc - m_row[i]) / l_row[i];
      double ds = p * (dp - D[i]);
      for (i64 c = 0; c < d; ++c) {
        dvj[c] += p * doi[c];
        dkj[c] += scale * ds * qi[c];
      }
    }
  }
  free(m_row);
  free(l_row);
  if (d_gap && gap > *d_gap) *d_gap = gap;
}

/* dQ, dK, dV, D for all heads.  Returns the largest |sum_j P dP - dO.O|. */
double oracle_bwd(const double *q, const double *k, const double *v,
                  const double *dO, int B, int H, int N, int d, double scale,
                  int causal, double *dq, double *dk, double *dv, double *D) {
  i64 hs = (i64)N * d;
  double gap = 0.0;
  for (i64 bh = 0; bh < (i64)B * H; ++bh)
    bwd_head(q + bh * hs, k + bh * hs, v + bh * hs, dO + bh * hs, N, d, scale,
             causal, dq + bh * hs, dk + bh * hs, dv + bh * hs, D + bh * (i64)N,
             &gap);
  return gap;
}

/* The online-softmax recurrence of §8.3 of the first page, one head, with
 * keys consumed in tiles of `tile` columns:
 *   m' = max(m, max(s)); alpha = e^{m - m'}; p = e^{s - m'};
 *   l' = alpha l + sum_j p_j;  o' = alpha o + p V_tile;  O = o / l.
 * Returns O and lse = m + ln l.  Independent of fwd_head on purpose. */
void oracle_online_fwd(const double *q, const double *k, const double *v,
                       int N, int d, double scale, int causal, int tile,
                       double *o, double *lse) {
  if (tile < 1) tile = 1;
#pragma omp parallel
  {
    double *acc = (double *)malloc(sizeof(double) * (size_t)(d > 0 ? d : 1));
    double *sv = (double *)malloc(sizeof(double) * (size_t)tile);
#pragma omp for schedule(dynamic, 16)
    for (i64 i = 0; i < N; ++i) {
      const double *qi = q + i * d;
      double m = -INFINITY, l = 0.0;
      for (i64 c = 0; c < d; ++c) acc[c] = 0.0;
      for (i64 j0 = 0; j0 < N; j0 += tile) {
        i64 j1 = j0 + tile < N ? j0 + tile : N;
        double tmax = -INFINITY;
        int any = 0;
        for (i64 j = j0; j < j1; ++j) {
          if (!visible(causal, i, j)) { sv[j - j0] = -INFINITY; continue; }
          double dot = 0.0;
          for (i64 c = 0; c < d; ++c) dot += qi[c] * k[j * d + c];
          sv[j - j0] = scale * dot;
          if (sv[j - j0] > tmax) tmax = sv[j - j0];
          any = 1;
        }
        if (!any) continue; /* a tile with no visible key changes nothing */
        double mnew = m > tmax ? m : tmax;
        double alpha = exp(m - mnew); /* e^{-inf} = 0 on the first tile */
        double psum = 0.0;
        for (i64 c = 0; c < d; ++c) acc[c] *= alpha;
        for (i64 j = j0; j < j1; ++j) {
          if (!visible(causal, i, j)) continue;
          double p = exp(sv[j - j0] - mnew);
          psum += p;
          for (i64 c = 0; c < d; ++c) acc[c] += p * v[j * d + c];
        }
        l = alpha * l + psum;
        m = mnew;
      }
      for (i64 c = 0; c < d; ++c) o[i * d + c] = acc[c] / l;
      lse[i] = m + log(l);
    }
    free(sv);
    free(acc);
  }
}

/* Decode-shaped attention: q, o [B,H,Nq,d]; k, v [B,H,L,d]; lse [B,H,Nq];
 * lens [B] valid cache rows per batch (NULL: all L).  Three passes per query
 * row over its visible keys, as in fwd_head. */
void oracle_decode(const double *q, const double *k, const double *v,
                   const int *lens, int B, int H, int Nq, int L, int d,
                   double scale, int causal, double *o, double *lse) {
  const i64 rows = (i64)B * H * Nq;
#pragma omp parallel
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
#pragma omp for schedule(dynamic, 4)
    for (i64 r = 0; r < rows; ++r) {
      const i64 i = r % Nq, bh = r / Nq, b = bh / H;
      const i64 len = lens ? lens[b] : L;
      i64 cnt = causal ? len - Nq + i + 1 : len;
      if (cnt < 0) cnt = 0;
      const double *qi = q + r * d;
      const double *kh = k + bh * (i64)L * d, *vh = v + bh * (i64)L * d;
      double *oi = o + r * d;
      for (i64 c = 0; c < d; ++c) oi[c] = 0.0;
      if (cnt == 0) {
        lse[r] = -INFINITY;
        continue;
      }
      for (i64 j = 0; j < cnt; ++j) {
        double acc = 0.0;
        for (i64 c = 0; c < d; ++c) acc += qi[c] * kh[j * d + c];
        s[j] = scale * acc;
      }
      double m;
      double l = row_max_sum(s, cnt, &m);
      for (i64 j = 0; j < cnt; ++j) {
        double p = exp(s[j] - m) / l;
        for (i64 c = 0; c < d; ++c) oi[c] += p * vh[j * d + c];
      }
      lse[r] = m + log(l);
    }
    free(s);
  }
}

/* Plain matrix product C = A B in fp64: A [M,K], B [K,N], C [M,N], all
 * row-major.  The operation whose throughput-versus-size curve opens
 * "CS336 Lecture 5 · GPUs, TPUs" (notes, opening goal and "矩阵谜题"); its
 * cost, 2MKN, is "第17讲 Tensor Core、HBM、SRAM 与 FlashAttention" §5.3.
 * C_ij = sum_k A_ik B_kj, summed in k order. */
void oracle_gemm(const double *A, const double *B, double *C, int M, int N,
                 int K) {
#pragma omp parallel for schedule(static)
  for (i64 i = 0; i < M; ++i) {
    double *ci = C + i * N;
    for (i64 j = 0; j < N; ++j) ci[j] = 0.0;
    for (i64 k = 0; k < K; ++k) {
      const double a = A[i * K + k];
      const double *bk = B + k * N;
      for (i64 j = 0; j < N; ++j) ci[j] += a * bk[j];
    }
  }
}

/* Scalar loss L = sum(O * dO) of the forward, for finite differences. */
double oracle_loss(const double *q, const double *k, const double *v,
                   const double *dO, int N, int d, double scale, int causal) {
  double *o = (double *)malloc(sizeof(double) * (size_t)N * d);
  double *lse = (double *)malloc(sizeof(double) * (size_t)N);
  fwd_head(q, k, v, N, d, scale, causal, o, lse);
  double L = 0.0;
  for (i64 t = 0; t < (i64)N * d; ++t) L += o[t] * dO[t];
  free(o);
  free(lse);
  return L;
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
