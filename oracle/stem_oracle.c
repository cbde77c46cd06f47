/*
 * CPU oracle for Stem block-sparse causal prefill.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load or call this library. The product path (the CUDA
 * library) never links, loads or calls it, and it shares no code with it.
 *
 * It restates, in plain double-precision loops, what the method computes, as
 * described for "Stem: Rethinking Causal Information Flow in Sparse Attention"
 * (arXiv 2603.06274). Page tags used below, all titled with that name:
 *   [es] gist.science/es, "Resumen tecnico"        (sections 1-5)
 *   [it] gist.science/it, "Sommario tecnico"       (sections 1-5)
 *   [nl] gist.science/nl, "Technische samenvatting" (Methodologie, Implementatie)
 *   [fr] gist.science/fr, "Resume technique"        (sections 1-5)
 *   [zh] shd-paper.top index page, English abstract and "key design" paragraph
 *
 * The pages describe three stages (block downsampling; a position-dependent
 * budget; top-k by the output-aware metric and exact attention over the kept
 * blocks): [es] section 2 "Implementacion", [it] section 2.C, [nl]
 * "Implementatie", [fr] section 2.C. Where the pages leave a step open, the
 * parameterised reading used here is:
 *   budget   k(i) = min(i+1, max(k_min, ceil(rho(i)*(i+1)))),
 *            rho(i) = rho_min + (1-rho_min)*exp(-i/tau), i = query-block index;
 *            or the pages' linear form ([es] 2.A, [it] 2.A, [nl] TPD, [fr] 2.A)
 *            k(i) = min(i+1, max(k_min, ceil(k_start*(1 - (1-mu)*i/(nb-1)))));
 *            for i >= 1 at least 2 blocks (sink and diagonal); k(0) = 1;
 *   pooling  arithmetic mean of Q rows and of K rows per block; mean of the
 *            per-row L2 norms of V per block (or their maximum: the "maximised
 *            magnitudes of V" of [nl] Implementatie step 1);
 *   metric   m_ij = softmax_{j<=i}(qbar_i . kbar_j / sqrt(D)) * n_j;
 *            or the pages' additive form ([es] 2.B, [it] 2.B, [nl] OAM, [fr] 2.B)
 *            M_ij = qbar_i . kbar_j / sqrt(D) + beta * max(0, log(n_j^2));
 *   keep     block 0, block i, and the k(i)-2 best other blocks j in [1, i-1]
 *            by (m descending, j ascending);
 *   attend   exact softmax attention of each query token over all tokens of
 *            the kept blocks, token-causal inside the diagonal block.
 *
 * Layouts: Q [B,Hq,S,D], K and V [B,Hkv,S,D], contiguous. Query head h reads
 * key/value head h / (Hq/Hkv). S need not be a multiple of block: there are
 * nb = ceil(S/block) blocks and the last one holds the S - (nb-1)*block
 * remaining tokens (pooled over those rows only). dtype 0 = bfloat16 (raw 16-bit patterns),
 * dtype 1 = float32. Every value is widened to double before any arithmetic.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int stem_oracle_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Exact widening of one stored element to double. */
static double elem(const void* base, int dtype, int64_t idx) {
  if (dtype == 1) return (double)((const float*)base)[idx];
  uint32_t bits = (uint32_t)((const uint16_t*)base)[idx] << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

/*
 * Token Position-Decay budget ([es] 2.A, [it] 2.A, [nl] TPD, [fr] 2.A: a budget
 * that is large for early query positions and shrinks with position; [zh] key
 * design: the decay is usually exponential). The exponential-ratio form above
 * is the reading used. Returns sum_i k(i); writes k[nb] and the prefix sums
 * off[nb+1] (off[0] = 0).
 */
int64_t stem_oracle_budget(int nb, double rho_min, double tau, int k_min,
                           int32_t* k_out, int64_t* off_out) {
  int64_t total = 0;
  for (int i = 0; i < nb; ++i) {
    double rho = rho_min + (1.0 - rho_min) * exp(-(double)i / tau);
    double want = ceil(rho * (double)(i + 1));
    double kk = want > (double)k_min ? want : (double)k_min;
    if (kk > (double)(i + 1)) kk = (double)(i + 1);
    int k = (int)kk;
    if (i == 0) {
      k = 1; /* only the block itself exists */
    } else if (k < 2) {
      k = 2; /* the sink and the diagonal are always kept */
    }
    if (off_out) off_out[i] = total;
    if (k_out) k_out[i] = k;
    total += k;
  }
  if (off_out) off_out[nb] = total;
  return total;
}

/*
 * Token Position-Decay budget, linear form ([es] 2.A: a high budget k_start for
 * the first tokens that decays linearly to k_end = mu * k_start for the last
 * ones, by linear interpolation; [it] 2.A and [nl] TPD: mu in (0, 1]; [fr] 2.A).
 * Reading: positions are query blocks, k_start is in blocks, the interpolation
 * runs from block 0 (k_start) to block nb-1 (k_end), and the interpolated
 * budget is rounded up, floored by k_min and capped by the i+1 causal blocks as
 * in the exponential form. Returns sum_i k(i); writes k[nb] and off[nb+1].
 */
int64_t stem_oracle_budget_linear(int nb, double k_start, double mu, int k_min,
                                  int32_t* k_out, int64_t* off_out) {
  int64_t total = 0;
  for (int i = 0; i < nb; ++i) {
    /* fraction of the way from the first block to the last */
    double t = nb > 1 ? (double)i / (double)(nb - 1) : 0.0;
    double k_lin = k_start * (1.0 - (1.0 - mu) * t);
    double want = ceil(k_lin);
    double kk = want > (double)k_min ? want : (double)k_min;
    if (kk > (double)(i + 1)) kk = (double)(i + 1);
    int k = (int)kk;
    if (i == 0) {
      k = 1;
    } else if (k < 2) {
      k = 2;
    }
    if (off_out) off_out[i] = total;
    if (k_out) k_out[i] = k;
    total += k;
  }
  if (off_out) off_out[nb] = total;
  return total;
}

/*
 * Block downsampling ([es] 2 "Implementacion" step 1: block-level Q, K and V
 * magnitude; [it] 2.C step 1; [nl] Implementatie step 1; [fr] 2.C step 1).
 * qbar [B,Hq,nb,D], kbar [B,Hkv,nb,D]: mean over the block's rows.
 * vnorm [B,Hkv,nb]: vmax == 0: mean over the block's rows of the row's
 * Euclidean norm; vmax == 1: the largest row norm of the block ([nl]
 * Implementatie step 1: maximised magnitudes of V).
 */
void stem_oracle_pool(const void* q, const void* k, const void* v, int dtype, int B,
                      int Hq, int Hkv, int S, int D, int block, int vmax, double* qbar,
                      double* kbar, double* vnorm) {
  const int nb = (S + block - 1) / block;
  const int64_t nq = (int64_t)B * Hq * nb;
  const int64_t nk = (int64_t)B * Hkv * nb;
#pragma omp parallel for schedule(static)
  for (int64_t u = 0; u < nq; ++u) {
    const int64_t bh = u / nb, i = u % nb;
    const int64_t row0 = bh * S + i * block;
    const int n = S - i * block < block ? (int)(S - i * block) : block; /* rows of block i */
    for (int d = 0; d < D; ++d) {
      double acc = 0.0;
      for (int r = 0; r < n; ++r) acc += elem(q, dtype, (row0 + r) * D + d);
      qbar[u * D + d] = acc / n;
    }
  }
#pragma omp parallel for schedule(static)
  for (int64_t u = 0; u < nk; ++u) {
    const int64_t bh = u / nb, i = u % nb;
    const int64_t row0 = bh * S + i * block;
    const int n = S - i * block < block ? (int)(S - i * block) : block;
    for (int d = 0; d < D; ++d) {
      double acc = 0.0;
      for (int r = 0; r < n; ++r) acc += elem(k, dtype, (row0 + r) * D + d);
      kbar[u * D + d] = acc / n;
    }
    double nacc = 0.0, nmax = 0.0;
    for (int r = 0; r < n; ++r) {
      double sq = 0.0;
      for (int d = 0; d < D; ++d) {
        double x = elem(v, dtype, (row0 + r) * D + d);
        sq += x * x;
      }
      const double norm = sqrt(sq);
      nacc += norm;
      if (norm > nmax) nmax = norm;
    }
    vnorm[u] = vmax ? nmax : nacc / n;
  }
}

/*
 * Output-Aware Metric on pooled blocks ([es] 2.B, [it] 2.B, [nl] OAM, [fr] 2.B:
 * routing relevance combined with value magnitude, since a block whose values
 * are near zero contributes little to the output; [zh] English abstract:
 * prioritises blocks by approximate output magnitude). Reading used: the
 * pooled attention probability times the pooled value norm,
 *   s_ij = qbar_i . kbar_j / sqrt(D),  p_ij = exp(s_ij - max_j s) / sum_j exp(...),
 *   m_ij = p_ij * n_j,   for j = 0..i.
 * Output packed by row: m[(b*Hq+h)*T + i*(i+1)/2 + j], T = nb*(nb+1)/2.
 */
void stem_oracle_metric(const double* qbar, const double* kbar, const double* vnorm,
                        int B, int Hq, int Hkv, int nb, int D, double* m) {
  const int G = Hq / Hkv;
  const int64_t T = (int64_t)nb * (nb + 1) / 2;
  const double scale = 1.0 / sqrt((double)D);
  const int64_t rows = (int64_t)B * Hq * nb;
#pragma omp parallel for schedule(dynamic, 16)
  for (int64_t u = 0; u < rows; ++u) {
    const int64_t bh = u / nb;
    const int i = (int)(u % nb);
    const int64_t b = bh / Hq, h = bh % Hq;
    const int64_t bg = b * Hkv + h / G;
    const double* qi = qbar + u * D;
    double* mrow = m + bh * T + (int64_t)i * (i + 1) / 2;
    double mx = -INFINITY;
    for (int j = 0; j <= i; ++j) {
      const double* kj = kbar + (bg * nb + j) * D;
      double dot = 0.0;
      for (int d = 0; d < D; ++d) dot += qi[d] * kj[d];
      mrow[j] = dot * scale; /* s_ij, kept here until normalised */
      if (mrow[j] > mx) mx = mrow[j];
    }
    double z = 0.0;
    for (int j = 0; j <= i; ++j) z += exp(mrow[j] - mx);
    for (int j = 0; j <= i; ++j) {
      double p = exp(mrow[j] - mx) / z;
      mrow[j] = p * vnorm[bg * nb + j];
    }
  }
}

/*
 * Output-Aware Metric, the pages' additive form ([es] 2.B, [it] 2.B, [nl] OAM,
 * [fr] 2.B): routing score plus a weighted, clamped log energy of the value,
 *   M_ij = qbar_i . kbar_j / sqrt(D) + beta * max(0, log(n_j^2)),   j = 0..i,
 * with n_j the block's V magnitude (pooled as above) standing for ||V_j||.
 * clamp == 0 drops the max(0, .). beta == 0 gives M = s (the magnitude term is
 * taken as 0 even where n_j = 0). Same packed layout as stem_oracle_metric.
 */
void stem_oracle_metric_additive(const double* qbar, const double* kbar,
                                 const double* vnorm, int B, int Hq, int Hkv, int nb,
                                 int D, double beta, int clamp, double* m) {
  const int G = Hq / Hkv;
  const int64_t T = (int64_t)nb * (nb + 1) / 2;
  const double scale = 1.0 / sqrt((double)D);
  const int64_t rows = (int64_t)B * Hq * nb;
#pragma omp parallel for schedule(dynamic, 16)
  for (int64_t u = 0; u < rows; ++u) {
    const int64_t bh = u / nb;
    const int i = (int)(u % nb);
    const int64_t b = bh / Hq, h = bh % Hq;
    const int64_t bg = b * Hkv + h / G;
    const double* qi = qbar + u * D;
    double* mrow = m + bh * T + (int64_t)i * (i + 1) / 2;
    for (int j = 0; j <= i; ++j) {
      const double* kj = kbar + (bg * nb + j) * D;
      double dot = 0.0;
      for (int d = 0; d < D; ++d) dot += qi[d] * kj[d];
      const double n = vnorm[bg * nb + j];
      double energy = log(n * n);
      if (clamp && energy < 0.0) energy = 0.0;
      mrow[j] = dot * scale + (beta == 0.0 ? 0.0 : beta * energy);
    }
  }
}

typedef struct {
  double m;
  int j;
} cand_t;

/* Larger metric first; equal metrics: lower block index first. */
static int cand_cmp(const void* pa, const void* pb) {
  const cand_t* a = (const cand_t*)pa;
  const cand_t* b = (const cand_t*)pb;
  if (a->m > b->m) return -1;
  if (a->m < b->m) return 1;
  return (a->j > b->j) - (a->j < b->j);
}

static int int_cmp(const void* pa, const void* pb) {
  int a = *(const int*)pa, b = *(const int*)pb;
  return (a > b) - (a < b);
}

/*
 * Top-k block selection with the position-dependent budget ([es] 2
 * "Implementacion" steps 2-3; [it] 2.C step 2; [nl] Implementatie steps 2-3;
 * [fr] 2.C steps 2-3), keeping the initial block that every later token depends
 * on ([es] 1 and 2.A; [fr] 2.A; [zh] abstract: initial tokens are retained)
 * and the query block itself. Rows are written in ascending block order:
 *   sel_idx[(b*Hq+h)*cap + off[i] + t], t < k[i];  sel_cnt[(b*Hq+h)*nb + i] = k[i].
 */
void stem_oracle_select(const double* m, const int32_t* k, const int64_t* off, int B,
                        int Hq, int nb, int64_t cap, int32_t* sel_idx, int32_t* sel_cnt) {
  const int64_t T = (int64_t)nb * (nb + 1) / 2;
  const int64_t rows = (int64_t)B * Hq * nb;
#pragma omp parallel for schedule(dynamic, 16)
  for (int64_t u = 0; u < rows; ++u) {
    const int64_t bh = u / nb;
    const int i = (int)(u % nb);
    const double* mrow = m + bh * T + (int64_t)i * (i + 1) / 2;
    int32_t* dst = sel_idx + bh * cap + off[i];
    const int ki = k[i];
    sel_cnt[u] = ki;
    if (i == 0) {
      dst[0] = 0;
      continue;
    }
    int* chosen = (int*)malloc(sizeof(int) * (size_t)ki);
    int n = 0;
    chosen[n++] = 0;
    chosen[n++] = i;
    const int ncand = i - 1; /* blocks 1 .. i-1 */
    if (ncand > 0 && ki > 2) {
      cand_t* c = (cand_t*)malloc(sizeof(cand_t) * (size_t)ncand);
      for (int j = 1; j < i; ++j) {
        c[j - 1].m = mrow[j];
        c[j - 1].j = j;
      }
      qsort(c, (size_t)ncand, sizeof(cand_t), cand_cmp);
      for (int t = 0; t < ki - 2; ++t) chosen[n++] = c[t].j;
      free(c);
    }
    qsort(chosen, (size_t)n, sizeof(int), int_cmp);
    for (int t = 0; t < n; ++t) dst[t] = chosen[t];
    free(chosen);
  }
}

/*
 * Exact attention over the kept blocks ([es] 2 "Implementacion" step 3: exact
 * softmax and aggregation only over the selected blocks; [it] 2.C step 3;
 * [nl] Implementatie step 3; [fr] 2.C step 3). For query token r of block i:
 * keys are every token of every kept block j < i, plus tokens i*block .. r of
 * the diagonal block; logits Q[r].K[c] / sqrt(D); output sum_c softmax_c * V[c].
 *
 * Computes the listed query blocks only: rows[t] = (b*Hq + h)*nb + i,
 * nb = ceil(S/block). out_rows [nrows, block, D] (double); rows of a partial
 * last block past token S-1 are left 0.
 */
void stem_oracle_attention(const void* q, const void* k, const void* v, int dtype, int B,
                           int Hq, int Hkv, int S, int D, int block,
                           const int32_t* sel_idx, const int32_t* sel_cnt,
                           const int64_t* off, int64_t cap, const int64_t* rows,
                           int64_t nrows, double* out_rows) {
  const int nb = (S + block - 1) / block;
  const int G = Hq / Hkv;
  const double scale = 1.0 / sqrt((double)D);
  (void)B;
#pragma omp parallel
  {
    /* per-thread scratch: logits for every key a query token may see */
    double* logit = (double*)malloc(sizeof(double) * (size_t)S);
    double* qrow = (double*)malloc(sizeof(double) * (size_t)D);
    int64_t* keyrow = (int64_t*)malloc(sizeof(int64_t) * (size_t)S);
#pragma omp for schedule(dynamic, 1)
    for (int64_t t = 0; t < nrows; ++t) {
      const int64_t u = rows[t];
      const int64_t bh = u / nb;
      const int i = (int)(u % nb);
      const int64_t b = bh / Hq, h = bh % Hq;
      const int64_t kvbase = (b * Hkv + h / G) * (int64_t)S; /* row index of token 0 */
      const int32_t* list = sel_idx + bh * cap + off[i];
      const int cnt = sel_cnt[u];
      double* ob = out_rows + t * block * (int64_t)D;
      for (int64_t e = 0; e < (int64_t)block * D; ++e) ob[e] = 0.0;
      for (int r = 0; r < block && (int64_t)i * block + r < S; ++r) {
        const int64_t qtok = (int64_t)i * block + r;
        for (int d = 0; d < D; ++d) qrow[d] = elem(q, dtype, (bh * S + qtok) * D + d);
        int nkeys = 0;
        double mx = -INFINITY;
        for (int e = 0; e < cnt; ++e) {
          const int j = list[e];
          /* token-causal on the diagonal; a partial last block has S - j*block tokens */
          int last = (j == i) ? r : block - 1;
          if ((int64_t)j * block + last > S - 1) last = (int)(S - 1 - (int64_t)j * block);
          for (int c = 0; c <= last; ++c) {
            const int64_t krow = kvbase + (int64_t)j * block + c;
            double dot = 0.0;
            for (int d = 0; d < D; ++d) dot += qrow[d] * elem(k, dtype, krow * D + d);
            logit[nkeys] = dot * scale;
            keyrow[nkeys] = krow;
            if (logit[nkeys] > mx) mx = logit[nkeys];
            ++nkeys;
          }
        }
        double z = 0.0;
        for (int c = 0; c < nkeys; ++c) {
          logit[c] = exp(logit[c] - mx);
          z += logit[c];
        }
        double* o = out_rows + (t * block + r) * (int64_t)D;
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        for (int c = 0; c < nkeys; ++c) {
          const double w = logit[c] / z;
          for (int d = 0; d < D; ++d) o[d] += w * elem(v, dtype, keyrow[c] * D + d);
        }
      }
    }
    free(logit);
    free(qrow);
    free(keyrow);
  }
}

/*
 * Block scores by anti-diagonal sampling ([fr] 2.C step 1: the per-block
 * metrics are computed with anti-diagonal sampling for efficiency). The pages
 * give no formula; the reading used here:
 *   - tokens are grouped into runs of `stride` (sigma) consecutive tokens; a
 *     group of query tokens u and a group of key tokens w span a sigma x sigma
 *     sub-tile of the token logit matrix Q K^T / sqrt(D);
 *   - that sub-tile is sampled along its anti-diagonal (query token
 *     u*sigma + t with key token w*sigma + sigma-1-t, t = 0..sigma-1), and the
 *     mean of the sigma samples stands for it:
 *       a_uw = (1/sigma) sum_t Q[u*sigma+t] . K[w*sigma+sigma-1-t] / sqrt(D);
 *   - each query group takes a softmax over the key groups it may see
 *     causally (w <= u);
 *   - the block probability p_ij is the mass that the query groups of block i
 *     put on the key groups of block j, averaged over the query groups of
 *     block i (block / sigma of them; fewer in a partial last block):
 *       p_ij = (1/n_i) sum_{u in i} sum_{w in j} softmax_w(a_u.),  j = 0..i.
 *     Each row of p sums to 1 over j <= i, like the pooled probability.
 * Requires S % stride == 0 and block % stride == 0 (the caller checks).
 * Computes the listed query blocks only: ids[t] = (b*Hq + h)*nb + i;
 * p_out [nids, nb] (double), entries j > i left 0.
 */
void stem_oracle_antidiag(const void* q, const void* k, int dtype, int B, int Hq, int Hkv,
                          int S, int D, int block, int stride, const int64_t* ids,
                          int64_t nids, double* p_out) {
  const int nb = (S + block - 1) / block;
  const int G = Hq / Hkv;
  const int R = block / stride;   /* query (or key) groups per block */
  const int nred = S / stride;    /* groups per head */
  const double scale = 1.0 / ((double)stride * sqrt((double)D));
  (void)B;
#pragma omp parallel
  {
    double* a = (double*)malloc(sizeof(double) * (size_t)(nred > 0 ? nred : 1));
#pragma omp for schedule(dynamic, 1)
    for (int64_t t = 0; t < nids; ++t) {
      const int64_t id = ids[t];
      const int64_t bh = id / nb;
      const int i = (int)(id % nb);
      const int64_t b = bh / Hq, h = bh % Hq;
      const int64_t qbase = bh * (int64_t)S;                    /* token 0 of this head */
      const int64_t kbase = (b * Hkv + h / G) * (int64_t)S;
      double* prow = p_out + t * (int64_t)nb;
      for (int j = 0; j < nb; ++j) prow[j] = 0.0;
      const int u0 = i * R;
      const int n_i = nred - u0 < R ? nred - u0 : R;             /* query groups of block i */
      for (int u = u0; u < u0 + n_i; ++u) {
        double mx = -INFINITY;
        for (int w = 0; w <= u; ++w) {
          double acc = 0.0;
          for (int s = 0; s < stride; ++s) {
            const int64_t qtok = qbase + (int64_t)u * stride + s;
            const int64_t ktok = kbase + (int64_t)w * stride + (stride - 1 - s);
            for (int d = 0; d < D; ++d)
              acc += elem(q, dtype, qtok * D + d) * elem(k, dtype, ktok * D + d);
          }
          a[w] = acc * scale;
          if (a[w] > mx) mx = a[w];
        }
        double z = 0.0;
        for (int w = 0; w <= u; ++w) z += exp(a[w] - mx);
        for (int w = 0; w <= u; ++w) prow[w / R] += exp(a[w] - mx) / z / n_i;
      }
    }
    free(a);
  }
}
