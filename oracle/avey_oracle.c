/*
 * avey_oracle.c -- plain fp64 CPU oracle for the Avey-B ranker and
 * neural-processor layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark load this library.  It shares no code with
 * the CUDA library (no headers, helpers or tables), and the CUDA library never
 * calls it.
 *
 * Every function is a direct transcription of a definition, with naive loops
 * and no blocking, fusion or reordering.  Pages cited (by title / section):
 *   [AB-notes]  "Avey-B: 把无注意力架构改造成双向编码器" (papernotes.org,
 *               ICLR 2026 note), 方法详解: 整体框架 (ranker, enricher, fuser),
 *               关键设计 2 (static / dynamic layers), 关键设计 3 (eq. 6),
 *               关键设计 4 (eq. 8, neural compression).
 *   [AB-sum]    "Avey-B" (paperlayer.ai summary of arXiv 2602.15814v1),
 *               §3 Background, §4 Avey-B, App. A, App. B, App. H.
 *   [coreui]    "Avey-B架构：无注意力机制的高效双向编码器解析", §1, §3.1
 *               (L2 normalisation before the similarity, eps about 1e-8).
 *
 * Readings where the pages are silent:
 *   - pad rows of the last split are zero vectors; N(0) = 0 through the
 *     floor max(||x||, 1e-12), so a pad row has cosine 0 with every row;
 *   - the candidate set is every other split of the same sequence
 *     (bidirectional), self excluded; ties order by lower split index;
 *   - X_cat = [X_t ; w_1 X_c1 ; ... ; w_k X_ck] in rank order, the target
 *     block unweighted; missing candidates (n-1 < k) contribute zero blocks;
 *   - contextualizer activation is the identity and has no bias;
 *   - optional prenorm: the enricher input row is divided by
 *     sqrt(mean(x^2) + 1e-6) (gain-free RMS norm); the residual is unchanged.
 *
 * Parallelism: OpenMP over independent output rows only; every individual
 * value is computed by one thread in the order written.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define NORM_FLOOR 1e-12

void avey_orc_coupled_causal_mix(const double *V, const double *zt, int S, int mt, long long ld,
                                 double *c, long long ldc);

int avey_orc_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void avey_orc_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* Row L2 normalisation N(x) = x / max(||x||_2, 1e-12).
 * [AB-notes] 关键设计 2 (N(Z) N(Z)^T is a cosine similarity); [coreui] §1. */
static void l2_normalize_row(const double *x, int d, double *out) {
  double ss = 0.0;
  for (int q = 0; q < d; ++q) ss += x[q] * x[q];
  double nrm = sqrt(ss);
  if (nrm < NORM_FLOOR) nrm = NORM_FLOOR;
  for (int q = 0; q < d; ++q) out[q] = x[q] / nrm;
}

static double dot(const double *a, const double *b, int d) {
  double s = 0.0;
#pragma omp simd reduction(+ : s)
  for (int q = 0; q < d; ++q) s += a[q] * b[q];
  return s;
}

/* Padded split view: row j of split c of sequence b, or NULL for a pad row.
 * [AB-notes] 整体框架: the sequence is cut into S-token splits and zero-padded
 * when N is not a multiple of S. */
static const double *split_row(const double *x, int N, int d, int S, int b, int c, int j) {
  long long tok = (long long)c * S + j;
  if (tok >= N) return NULL;
  return x + ((long long)b * N + tok) * d;
}

/* N(X) for every row of X [B, N, d] (out has the same shape). */
void avey_orc_normalize(const double *x, long long rows, int d, double *out) {
#pragma omp parallel for schedule(static)
  for (long long r = 0; r < rows; ++r) l2_normalize_row(x + r * d, d, out + r * d);
}

/* MaxSim relevance of candidate split c for target split t:
 *   score(t, c) = sum_{i in t} max_{j in c} cos(x_i, x_j),
 * computed on the shallow (input) embeddings.  [AB-sum] §3 Background and
 * App. H (ranker retrieves on the initial embeddings); [AB-notes] 整体框架.
 * xn holds N(X) [B, N, d]; a pad row has cosine 0 with everything. */
static double maxsim(const double *xn, int N, int d, int S, int b, int t, int c) {
  double total = 0.0;
  for (int i = 0; i < S; ++i) {
    const double *xi = split_row(xn, N, d, S, b, t, i);
    double best = -INFINITY;
    for (int j = 0; j < S; ++j) {
      const double *xj = split_row(xn, N, d, S, b, c, j);
      double cs = (xi && xj) ? dot(xi, xj, d) : 0.0;
      if (cs > best) best = cs;
    }
    total += best;
  }
  return total;
}

/* Scores of every split c of sequence sel_b[s] against target sel_t[s]:
 * scores[s, c] for c in 0..n-1 (the diagonal c == t is included). */
void avey_orc_maxsim_rows(const double *xn, int B, int N, int d, int S, const int *sel_b,
                          const int *sel_t, int n_sel, double *scores) {
  (void)B;
  int n = (N + S - 1) / S;
#pragma omp parallel for collapse(2) schedule(dynamic, 4)
  for (int s = 0; s < n_sel; ++s)
    for (int c = 0; c < n; ++c)
      scores[(long long)s * n + c] = maxsim(xn, N, d, S, sel_b[s], sel_t[s], c);
}

typedef struct {
  double score;
  int idx;
} cand_t;

/* Order: higher score first, then lower split index. */
static int cand_cmp(const void *pa, const void *pb) {
  const cand_t *a = (const cand_t *)pa, *b = (const cand_t *)pb;
  if (a->score > b->score) return -1;
  if (a->score < b->score) return 1;
  return (a->idx > b->idx) - (a->idx < b->idx);
}

/* Top-k selection and normalisation for one target split t.
 * The k best candidates c != t (bidirectional: no causal mask, [AB-sum] §4);
 * weights w_r = s_r / s_1, the best selected score, so the top-1 weight is 1
 * ([AB-notes] 整体框架: "divide by the largest of them"; [AB-sum] §3).
 * Returns the number of real candidates k' = min(k, n-1); positions >= k' get
 * idx -1 and weight 0. */
int avey_orc_topk_row_dir(const double *scores, int n, int t, int k, int causal, int *idx,
                          double *w);

int avey_orc_topk_row(const double *scores, int n, int t, int k, int *idx, double *w) {
  return avey_orc_topk_row_dir(scores, n, t, k, 0, idx, w);
}

/* As above; with causal != 0 the candidates are only the preceding splits
 * c < t (the unidirectional ranker of the original Avey, and the ablation
 * setting of [AB-sum] App. B "Ranker direction"). */
int avey_orc_topk_row_dir(const double *scores, int n, int t, int k, int causal, int *idx,
                          double *w) {
  cand_t *cand = (cand_t *)malloc(sizeof(cand_t) * (size_t)(n > 0 ? n : 1));
  int m = 0;
  for (int c = 0; c < n; ++c)
    if (c != t && (!causal || c < t)) {
      cand[m].score = scores[c];
      cand[m].idx = c;
      ++m;
    }
  qsort(cand, (size_t)m, sizeof(cand_t), cand_cmp);
  int kk = k < m ? k : m;
  double s1 = kk > 0 ? cand[0].score : 1.0;
  if (!(s1 > 1e-30)) s1 = 1e-30; /* guard: unreachable with these mixtures */
  for (int r = 0; r < k; ++r) {
    if (r < kk) {
      idx[r] = cand[r].idx;
      w[r] = cand[r].score / s1;
    } else {
      idx[r] = -1;
      w[r] = 0.0;
    }
  }
  free(cand);
  return kk;
}

/* Neural compression with residual, for target split t of sequence b:
 *   X_cat = [X_t ; w_1 X_c1 ; ... ; w_k X_ck]          ((k+1)S x d)
 *   out   = P X_cat + X_t,  P in R^{S x (k+1)S}
 * [AB-notes] 关键设计 4 (eq. 8 and the residual to the split's own tokens);
 * [AB-sum] §4.3, App. H (residual).  x is the raw embedding X [B, N, d]. */
void avey_orc_compress_split(const double *x, int N, int d, int S, int k, int b, int t,
                             const int *idx, const double *w, const double *P, double *out) {
  int KS = (k + 1) * S;
  for (int i = 0; i < S; ++i) {
    double *o = out + (long long)i * d;
    const double *xt_i = split_row(x, N, d, S, b, t, i);
    for (int q = 0; q < d; ++q) o[q] = xt_i ? xt_i[q] : 0.0; /* residual X_t */
    for (int r = 0; r <= k; ++r) {
      int c = (r == 0) ? t : idx[r - 1];
      double wr = (r == 0) ? 1.0 : w[r - 1];
      if (c < 0) continue; /* missing candidate: zero block */
      for (int j = 0; j < S; ++j) {
        const double *xc_j = split_row(x, N, d, S, b, c, j);
        if (!xc_j) continue;
        double coef = P[(long long)i * KS + (long long)r * S + j] * wr;
        for (int q = 0; q < d; ++q) o[q] += coef * xc_j[q];
      }
    }
  }
}

/* Static contextualizer c = V Z_t over the tokens of one split (identity
 * activation, no bias).  [AB-notes] 关键设计 2, c_static. */
void avey_orc_static_mix(const double *V, const double *zt, int S, int mt, long long ld,
                         double *c, long long ldc) {
  /* c[i, f] = sum_j V[i, j] zt[j, f], summed over j in order (j outer so
   * that the f loop walks contiguous rows) */
  for (int i = 0; i < S; ++i) {
    double *ci = c + (long long)i * ldc;
    for (int f = 0; f < mt; ++f) ci[f] = 0.0;
    for (int j = 0; j < S; ++j) {
      double v = V[(long long)i * S + j];
      const double *zj = zt + (long long)j * ld;
      for (int f = 0; f < mt; ++f) ci[f] += v * zj[f];
    }
  }
}

/* Dynamic weights of one split:
 *   G_ij = N(z_i) . N(z_j)               (cosine similarity)
 *   Gt_ij = G_ij / (sum_j G_ij + eps)     (eq. 6, row normalisation)
 * [AB-notes] 关键设计 2 (S = N(Z)N(Z)^T) and 关键设计 3 (eq. 6);
 * [coreui] §3.1 (eps about 1e-8). */
void avey_orc_dynamic_weights(const double *zt, int S, int mt, long long ld, double eps,
                              double *Gt) {
  double *u = (double *)malloc(sizeof(double) * (size_t)S * (size_t)mt);
  for (int i = 0; i < S; ++i) l2_normalize_row(zt + (long long)i * ld, mt, u + (long long)i * mt);
  for (int i = 0; i < S; ++i) {
    double rowsum = 0.0;
    for (int j = 0; j < S; ++j) {
      double g = dot(u + (long long)i * mt, u + (long long)j * mt, mt);
      Gt[(long long)i * S + j] = g;
      rowsum += g;
    }
    for (int j = 0; j < S; ++j) Gt[(long long)i * S + j] /= (rowsum + eps);
  }
  free(u);
}

/* Dynamic contextualizer c = Gt Z_t (identity activation, no bias). */
void avey_orc_dynamic_mix(const double *zt, int S, int mt, long long ld, double eps, double *c,
                          long long ldc) {
  double *Gt = (double *)malloc(sizeof(double) * (size_t)S * (size_t)S);
  avey_orc_dynamic_weights(zt, S, mt, ld, eps, Gt);
  avey_orc_static_mix(Gt, zt, S, mt, ld, c, ldc); /* same product, with Gt as the map */
  free(Gt);
}

/* One neural-processor layer applied in place to n_splits independent splits
 * x [n_splits, S, d]:
 *   enricher  Z = relu(X U + b)^2                 ([AB-notes] 整体框架;
 *                                                   [AB-sum] App. A: ReLU^2)
 *   head/tail Z_h = Z[:, :m_h], Z_t = Z[:, m_h:]   ([AB-notes] 整体框架)
 *   context   c = V Z_t (static) or Gt Z_t (dynamic)
 *   fuser     X' = X + [Z_h || c] O               ([AB-notes] 整体框架)
 * kind: 0 static, 1 dynamic, 2 coupled causal (original Avey, see
 * avey_orc_coupled_causal_mix).
 * U is [d, m], bU [m], V [S, S] (static and coupled), O [m, d]. */
void avey_orc_layer(double *x, int n_splits, int S, int d, int m, int m_h, int kind, int prenorm,
                    double eps, const double *U, const double *bU, const double *V,
                    const double *O) {
  int mt = m - m_h;
#pragma omp parallel for schedule(dynamic, 1)
  for (int sp = 0; sp < n_splits; ++sp) {
    double *xs = x + (long long)sp * S * d;
    double *xin = (double *)malloc(sizeof(double) * (size_t)S * (size_t)d);
    double *Z = (double *)malloc(sizeof(double) * (size_t)S * (size_t)m);
    double *c = (double *)malloc(sizeof(double) * (size_t)S * (size_t)mt);
    double *acc = (double *)malloc(sizeof(double) * (size_t)d);
    for (int i = 0; i < S; ++i) {
      double scale = 1.0;
      if (prenorm) {
        double ms = 0.0;
        for (int q = 0; q < d; ++q) ms += xs[(long long)i * d + q] * xs[(long long)i * d + q];
        scale = 1.0 / sqrt(ms / d + 1e-6);
      }
      for (int q = 0; q < d; ++q) xin[(long long)i * d + q] = xs[(long long)i * d + q] * scale;
    }
    /* a[i, f] = b[f] + sum_q xin[i, q] U[q, f], summed over q in order (q
     * outer so that the f loop walks contiguous rows of U); Z = relu(a)^2 */
    for (int i = 0; i < S; ++i) {
      double *zi = Z + (long long)i * m;
      for (int f = 0; f < m; ++f) zi[f] = bU[f];
      for (int q = 0; q < d; ++q) {
        double xv = xin[(long long)i * d + q];
        const double *uq = U + (long long)q * m;
        for (int f = 0; f < m; ++f) zi[f] += xv * uq[f];
      }
      for (int f = 0; f < m; ++f) {
        double r = zi[f] > 0.0 ? zi[f] : 0.0;
        zi[f] = r * r;
      }
    }
    if (kind == 0)
      avey_orc_static_mix(V, Z + m_h, S, mt, m, c, mt);
    else if (kind == 1)
      avey_orc_dynamic_mix(Z + m_h, S, mt, m, eps, c, mt);
    else
      avey_orc_coupled_causal_mix(V, Z + m_h, S, mt, m, c, mt);
    /* X'[i, q] = X[i, q] + sum_f [Z_h || c][i, f] O[f, q], the sum over f in
     * order (f outer so that the q loop walks contiguous rows of O) */
    for (int i = 0; i < S; ++i) {
      for (int q = 0; q < d; ++q) acc[q] = 0.0;
      for (int f = 0; f < m; ++f) {
        double v = f < m_h ? Z[(long long)i * m + f] : c[(long long)i * mt + (f - m_h)];
        const double *of = O + (long long)f * d;
        for (int q = 0; q < d; ++q) acc[q] += v * of[q];
      }
      for (int q = 0; q < d; ++q) xs[(long long)i * d + q] += acc[q];
    }
    free(acc);
    free(xin);
    free(Z);
    free(c);
  }
}

/* Uncompressed context of target split t of sequence b (the tensor that the
 * compressor of [AB-notes] 关键设计 4 maps from (k+1)S tokens to S, and that
 * the neural processor sees in full without it, [AB-sum] §4.3):
 *   X_cat = [X_t ; w_1 X_c1 ; ... ; w_k X_ck]          ((k+1)S x d)
 * in rank order, the target block unweighted; a missing candidate (-1) and the
 * pad rows of a ragged last split are zero rows. */
void avey_orc_context_split(const double *x, int N, int d, int S, int k, int b, int t,
                            const int *idx, const double *w, double *out) {
  for (int r = 0; r <= k; ++r) {
    int c = (r == 0) ? t : idx[r - 1];
    double wr = (r == 0) ? 1.0 : w[r - 1];
    for (int j = 0; j < S; ++j) {
      double *o = out + ((long long)r * S + j) * d;
      const double *xc_j = c < 0 ? 0 : split_row(x, N, d, S, b, c, j);
      for (int q = 0; q < d; ++q) o[q] = xc_j ? wr * xc_j[q] : 0.0;
    }
  }
}

void avey_orc_context_rows(const double *x, int N, int d, int S, int k, const int *sel_b,
                           const int *sel_t, int n_sel, const int *idx, const double *w,
                           double *out) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int s = 0; s < n_sel; ++s)
    avey_orc_context_split(x, N, d, S, k, sel_b[s], sel_t[s], idx + (long long)s * k,
                           w + (long long)s * k, out + (long long)s * (k + 1) * S * d);
}

/* Compression of several target splits (independent; one split per thread). */
void avey_orc_compress_rows(const double *x, int N, int d, int S, int k, const int *sel_b,
                            const int *sel_t, int n_sel, const int *idx, const double *w,
                            const double *P, double *out) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int s = 0; s < n_sel; ++s)
    avey_orc_compress_split(x, N, d, S, k, sel_b[s], sel_t[s], idx + (long long)s * k,
                            w + (long long)s * k, P, out + (long long)s * S * d);
}

/* Coupled contextualizer of the original Avey ([AB-notes] 关键设计 2: the
 * learned static matrix V multiplied element-wise with the input-dependent
 * cosine matrix N(Z_t)N(Z_t)^T, the result combining the embeddings), with the
 * autoregressive (causal) mask of the original Avey ([AB-sum] §3, §4: Avey-B
 * removes that mask):
 *   M_ij = V_ij * N(z_i).N(z_j) for j <= i, 0 for j > i;   c = M Z_t.
 * Identity activation, no bias, no row normalisation. */
void avey_orc_coupled_causal_mix(const double *V, const double *zt, int S, int mt, long long ld,
                                 double *c, long long ldc) {
  double *u = (double *)malloc(sizeof(double) * (size_t)S * (size_t)mt);
  double *M = (double *)malloc(sizeof(double) * (size_t)S * (size_t)S);
  for (int i = 0; i < S; ++i) l2_normalize_row(zt + (long long)i * ld, mt, u + (long long)i * mt);
  for (int i = 0; i < S; ++i)
    for (int j = 0; j < S; ++j)
      M[(long long)i * S + j] =
          j <= i ? V[(long long)i * S + j] * dot(u + (long long)i * mt, u + (long long)j * mt, mt) : 0.0;
  avey_orc_static_mix(M, zt, S, mt, ld, c, ldc); /* same product, with M as the map */
  free(u);
  free(M);
}
