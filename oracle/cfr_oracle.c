/*
 * cfr_oracle.c -- plain, slow fp64 CPU oracle for paged decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg may load this file's library.  It shares no code,
 * header, table or helper with the CUDA library: it decodes the stored bytes
 * itself, resolves page indices itself and evaluates the attention definition
 * directly in double precision.
 *
 * What it computes, per (sequence b, query head h):
 *
 *   o = softmax(q K^T * sigma + bias) V
 *
 * the scaled dot-product attention definition given on the RustAttention page
 * (section "Mathematical Framework Covered": Softmax(QK^T / sqrt(d_k) + Mask) V)
 * for one query row, over the n = seq_lens[b] cached tokens j = 0..n-1 (the
 * decode query attends to every cached token; no further mask).  The softmax
 * is evaluated with the max subtracted (RustAttention page, "Numerically
 * Stable Softmax").  K and V are first materialised in full from the pages
 * (the full-KV baseline of the CFR-Atlas page, "core contract":
 * folded attention == full-KV baseline attention).
 *
 *   - token j lives on logical page p = j / P at row t = j % P;
 *   - its physical slot is page_table[b][p] inside the pool of its format
 *     page_fmt[b][p] (uniform_fmt when page_fmt is NULL);
 *   - the row of kv head g is at byte ((slot * Hkv + g) * P + t) * row_bytes;
 *   - values: F32 as stored, BF16 widened from its 16 bits, I8 code * scale,
 *     I4 nibble code * scale, with scale = scales[fmt][slot][g][0 for K, 1 for V]
 *     (ARGUS page, "Why It Works: Storage vs. Computation": pages are stored
 *     compressed and restored to full precision before attention);
 *   - sigma = softmax_scale, or 1/sqrt(d) when softmax_scale is 0;
 *   - bias_j = -slope_h * (n - 1 - j) with ALiBi slopes, else 0
 *     (CFR-Atlas page, "RoPE/ALiBi positional policy");
 *   - kv head g = head_map[h], or h / (Hq / Hkv) when head_map is NULL
 *     (CFR-Atlas page, "MHA/MQA/GQA head mapping").
 *
 * Modes: 0 evaluates the definition directly.  1 folds blocks of `arg` tokens
 * one at a time into a running (max, normaliser, accumulator) -- the folded
 * online-softmax pass of the CFR-Atlas page ("exact folded online-softmax
 * attention pass") and the page-by-page online softmax of the ARGUS page
 * ("Fused Triton Attention Kernel").  2 splits the pages into `arg`
 * contiguous ranges, evaluates each range directly and merges the partial
 * results by their log-sum-exp (the split-K decoding of the CMF page, "attention
 * uses split-K flash-decoding").
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_F32 0
#define ORC_BF16 1
#define ORC_I8 2
#define ORC_I4 3
#define ORC_NFMT 4

#define ORC_OK 0
#define ORC_BAD_ARG 1
#define ORC_BAD_PAGE 2
#define ORC_NO_MEMORY 3
#define ORC_EMPTY 4

typedef struct {
  int32_t batch, num_q_heads, num_kv_heads, head_dim, page_tokens, max_pages;
  int32_t q_fmt, uniform_fmt;
  const void *q;                       /* [B][Hq][d] f32 or bf16 bits */
  const void *k_pool[ORC_NFMT];
  const void *v_pool[ORC_NFMT];
  const float *scales[ORC_NFMT];       /* [slots][Hkv][2] for I8/I4 */
  int64_t pool_pages[ORC_NFMT];
  const int32_t *page_table;           /* [B][max_pages] */
  const uint8_t *page_fmt;             /* [B][max_pages] or NULL */
  const int32_t *seq_lens;             /* [B] */
  const int32_t *head_map;             /* [Hq] or NULL */
  const float *alibi_slopes;           /* [Hq] or NULL */
  double softmax_scale;                /* 0 => 1/sqrt(d) */
} orc_problem;

/* ---- decoding of one stored element ------------------------------------ */

static double orc_from_f32(const unsigned char *p) {
  float f;
  memcpy(&f, p, sizeof f);
  return (double)f;
}

static double orc_from_bf16(const unsigned char *p) {
  /* bf16 is the upper half of an IEEE binary32 */
  uint16_t h;
  memcpy(&h, p, sizeof h);
  uint32_t w = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &w, sizeof f);
  return (double)f;
}

static int orc_i8_code(unsigned char byte) {
  return byte < 128 ? (int)byte : (int)byte - 256;
}

static int orc_i4_code(unsigned char byte, int high) {
  int nib = high ? (byte >> 4) : (byte & 15);
  return nib < 8 ? nib : nib - 16;
}

static long orc_row_bytes(int fmt, int d) {
  switch (fmt) {
    case ORC_F32: return 4L * d;
    case ORC_BF16: return 2L * d;
    case ORC_I8: return (long)d;
    case ORC_I4: return (long)d / 2;
  }
  return -1;
}

/* element i of a stored row, times the block scale for quantised formats */
static double orc_element(int fmt, const unsigned char *row, int i, double scale) {
  switch (fmt) {
    case ORC_F32: return orc_from_f32(row + 4L * i);
    case ORC_BF16: return orc_from_bf16(row + 2L * i);
    case ORC_I8: return (double)orc_i8_code(row[i]) * scale;
    case ORC_I4: return (double)orc_i4_code(row[i / 2], i % 2) * scale;
  }
  return NAN;
}

static double orc_query(const orc_problem *pr, int b, int h, int i) {
  long idx = ((long)b * pr->num_q_heads + h) * pr->head_dim + i;
  const unsigned char *base = (const unsigned char *)pr->q;
  if (pr->q_fmt == ORC_F32) return orc_from_f32(base + 4L * idx);
  return orc_from_bf16(base + 2L * idx);
}

static int orc_kv_head(const orc_problem *pr, int h) {
  if (pr->head_map) return pr->head_map[h];
  return h / (pr->num_q_heads / pr->num_kv_heads);
}

/* ---- materialising the full K and V of (b, g) -------------------------- */

/*
 * Writes K[j][i], V[j][i] (double, [n][d]) for the tokens of sequence b and kv
 * head g, and keep[j] = 1 for tokens whose page resolved.  A page with an
 * out-of-range slot, an unknown format or a missing pool is an error unless
 * skip_invalid is set, in which case its tokens get keep = 0.
 */
static int orc_materialise(const orc_problem *pr, int b, int g, int n, int skip_invalid,
                           double *K, double *V, unsigned char *keep) {
  const int d = pr->head_dim, P = pr->page_tokens, Hkv = pr->num_kv_heads;
  for (int j = 0; j < n; ++j) {
    const int p = j / P, t = j % P;
    const long cell = (long)b * pr->max_pages + p;
    const int fmt = pr->page_fmt ? (int)pr->page_fmt[cell] : pr->uniform_fmt;
    const long slot = pr->page_table[cell];
    int ok = fmt >= 0 && fmt < ORC_NFMT && pr->k_pool[fmt] && pr->v_pool[fmt] &&
             slot >= 0 && slot < pr->pool_pages[fmt] &&
             ((fmt != ORC_I8 && fmt != ORC_I4) || pr->scales[fmt]);
    if (!ok) {
      if (!skip_invalid) return ORC_BAD_PAGE;
      keep[j] = 0;
      for (int i = 0; i < d; ++i) K[(long)j * d + i] = V[(long)j * d + i] = 0.0;
      continue;
    }
    keep[j] = 1;
    const long rb = orc_row_bytes(fmt, d);
    const long off = ((slot * Hkv + g) * (long)P + t) * rb;
    const unsigned char *krow = (const unsigned char *)pr->k_pool[fmt] + off;
    const unsigned char *vrow = (const unsigned char *)pr->v_pool[fmt] + off;
    double ks = 1.0, vs = 1.0;
    if (fmt == ORC_I8 || fmt == ORC_I4) {
      const float *sc = pr->scales[fmt] + (slot * Hkv + g) * 2;
      ks = (double)sc[0];
      vs = (double)sc[1];
    }
    for (int i = 0; i < d; ++i) {
      K[(long)j * d + i] = orc_element(fmt, krow, i, ks);
      V[(long)j * d + i] = orc_element(fmt, vrow, i, vs);
    }
  }
  return ORC_OK;
}

/* ---- the attention definition over a token range ----------------------- */

static double orc_sigma(const orc_problem *pr) {
  return pr->softmax_scale != 0.0 ? pr->softmax_scale : 1.0 / sqrt((double)pr->head_dim);
}

/* score of token j for query head h of sequence b with n tokens */
static double orc_score(const orc_problem *pr, const double *qv, const double *K, int j,
                        int h, int n) {
  const int d = pr->head_dim;
  double dot = 0.0;
  for (int i = 0; i < d; ++i) dot += qv[i] * K[(long)j * d + i];
  double s = orc_sigma(pr) * dot;
  if (pr->alibi_slopes) s += -(double)pr->alibi_slopes[h] * (double)(n - 1 - j);
  return s;
}

/*
 * Softmax partial over tokens [j0, j1): m = max score, l = sum exp(s - m),
 * a[i] = sum exp(s - m) V[j][i].  With no kept token: m = -inf, l = 0, a = 0.
 */
static void orc_partial(const orc_problem *pr, const double *qv, const double *K, const double *V,
                        const unsigned char *keep, int h, int n, int j0, int j1,
                        double *m, double *l, double *a) {
  const int d = pr->head_dim;
  double mx = -INFINITY;
  for (int j = j0; j < j1; ++j)
    if (keep[j]) {
      double s = orc_score(pr, qv, K, j, h, n);
      if (s > mx) mx = s;
    }
  double sum = 0.0;
  for (int i = 0; i < d; ++i) a[i] = 0.0;
  if (mx != -INFINITY) {
    for (int j = j0; j < j1; ++j) {
      if (!keep[j]) continue;
      double w = exp(orc_score(pr, qv, K, j, h, n) - mx);
      sum += w;
      for (int i = 0; i < d; ++i) a[i] += w * V[(long)j * d + i];
    }
  }
  *m = mx;
  *l = sum;
}

/* fold partial (m2, l2, a2) into the running (m, l, a) */
static void orc_combine(int d, double *m, double *l, double *a, double m2, double l2,
                        const double *a2) {
  if (m2 == -INFINITY) return;
  if (*m == -INFINITY) {
    *m = m2;
    *l = l2;
    for (int i = 0; i < d; ++i) a[i] = a2[i];
    return;
  }
  double mn = *m > m2 ? *m : m2;
  double c1 = exp(*m - mn), c2 = exp(m2 - mn);
  *l = *l * c1 + l2 * c2;
  for (int i = 0; i < d; ++i) a[i] = a[i] * c1 + a2[i] * c2;
  *m = mn;
}

/* one (b, h): out[d] and lse; K/V/keep already materialised for kv head of h */
static int orc_one(const orc_problem *pr, int b, int h, int n, const double *K, const double *V,
                   const unsigned char *keep, int mode, long arg, double *out, double *lse) {
  const int d = pr->head_dim, P = pr->page_tokens;
  double *qv = (double *)malloc(sizeof(double) * d);
  double *a = (double *)malloc(sizeof(double) * d);
  double *a2 = (double *)malloc(sizeof(double) * d);
  if (!qv || !a || !a2) {
    free(qv); free(a); free(a2);
    return ORC_NO_MEMORY;
  }
  for (int i = 0; i < d; ++i) qv[i] = orc_query(pr, b, h, i);
  double m = -INFINITY, l = 0.0;
  for (int i = 0; i < d; ++i) a[i] = 0.0;
  if (mode == 0) {
    orc_partial(pr, qv, K, V, keep, h, n, 0, n, &m, &l, a);
  } else if (mode == 1) {
    long blk = arg > 0 ? arg : n;
    for (long j0 = 0; j0 < n; j0 += blk) {
      long j1 = j0 + blk < n ? j0 + blk : n;
      double m2, l2;
      orc_partial(pr, qv, K, V, keep, h, n, (int)j0, (int)j1, &m2, &l2, a2);
      orc_combine(d, &m, &l, a, m2, l2, a2);
    }
  } else {
    /* split the NP pages into `arg` contiguous ranges of ceil(NP/arg) pages */
    long np = (n + P - 1) / P;
    long S = arg > 0 ? arg : 1;
    long per = (np + S - 1) / S;
    if (per < 1) per = 1;
    /* partials first, then the log-sum-exp merge of all of them */
    double *pm = (double *)malloc(sizeof(double) * S);
    double *pl = (double *)malloc(sizeof(double) * S);
    double *pa = (double *)malloc(sizeof(double) * S * d);
    if (!pm || !pl || !pa) {
      free(pm); free(pl); free(pa); free(qv); free(a); free(a2);
      return ORC_NO_MEMORY;
    }
    for (long s = 0; s < S; ++s) {
      long j0 = s * per * P, j1 = (s + 1) * per * P;
      if (j0 > n) j0 = n;
      if (j1 > n) j1 = n;
      orc_partial(pr, qv, K, V, keep, h, n, (int)j0, (int)j1, &pm[s], &pl[s], pa + s * d);
    }
    double M = -INFINITY;
    for (long s = 0; s < S; ++s)
      if (pl[s] > 0.0 && pm[s] > M) M = pm[s];
    if (M != -INFINITY) {
      for (long s = 0; s < S; ++s) {
        if (!(pl[s] > 0.0)) continue;
        double w = exp(pm[s] - M);
        l += pl[s] * w;
        for (int i = 0; i < d; ++i) a[i] += pa[s * d + i] * w;
      }
      m = M;
    }
    free(pm); free(pl); free(pa);
  }
  if (l > 0.0) {
    for (int i = 0; i < d; ++i) out[i] = a[i] / l;
    *lse = m + log(l);
  } else {
    for (int i = 0; i < d; ++i) out[i] = 0.0;
    *lse = -INFINITY;
  }
  free(qv); free(a); free(a2);
  return ORC_OK;
}

static int orc_check(const orc_problem *pr) {
  if (!pr || pr->batch < 0 || pr->num_q_heads <= 0 || pr->num_kv_heads <= 0 ||
      pr->head_dim <= 0 || pr->page_tokens <= 0 || pr->max_pages < 0 || !pr->q ||
      !pr->page_table || !pr->seq_lens)
    return ORC_BAD_ARG;
  if (!pr->head_map && pr->num_q_heads % pr->num_kv_heads) return ORC_BAD_ARG;
  if (pr->head_dim % 2) return ORC_BAD_ARG;
  return ORC_OK;
}

/* one run of selections [k0, k1) that share (b, kv head g) */
static int orc_run(const orc_problem *pr, const int32_t *sel_h, int64_t k0, int64_t k1, int b,
                   int g, int mode, int64_t arg, int skip_invalid, int nthreads, double *out,
                   double *lse) {
  const int d = pr->head_dim;
  const int n = pr->seq_lens[b];
  if (n <= 0) {
    for (int64_t kk = k0; kk < k1; ++kk) {
      for (int i = 0; i < d; ++i) out[kk * d + i] = 0.0;
      lse[kk] = -INFINITY;
    }
    return ORC_EMPTY;
  }
  double *K = (double *)malloc(sizeof(double) * (size_t)n * d);
  double *V = (double *)malloc(sizeof(double) * (size_t)n * d);
  unsigned char *keep = (unsigned char *)malloc((size_t)n);
  int rc = (!K || !V || !keep) ? ORC_NO_MEMORY
                               : orc_materialise(pr, b, g, n, skip_invalid, K, V, keep);
  int err = ORC_OK;
  if (!rc) {
#pragma omp parallel for num_threads(nthreads > 0 ? nthreads : 1) schedule(dynamic, 1)
    for (int64_t kk = k0; kk < k1; ++kk) {
      const int h = sel_h ? sel_h[kk] : (int)(kk % pr->num_q_heads);
      int r = orc_one(pr, b, h, n, K, V, keep, mode, arg, out + kk * d, lse + kk);
      if (r) {
#pragma omp critical
        err = r;
      }
    }
  }
  free(K); free(V); free(keep);
  return rc ? rc : err;
}

/*
 * Attention output for the selected (sel_b[k], sel_h[k]) pairs, k < n_sel, in
 * that order (all pairs b-major when sel_b is NULL: n_sel must be B*Hq).
 * out: [n_sel][d], lse: [n_sel] natural-log log-sum-exp of the scores.
 * Consecutive selections with the same (b, kv head) form a run that shares one
 * materialisation of K and V.  Runs execute concurrently on `nthreads` OpenMP
 * threads when there are enough of them and their K/V fit in `mem_limit`
 * bytes together; otherwise runs execute one at a time with their heads in
 * parallel.  Returns ORC_EMPTY (after writing 0 / -inf) when a selected
 * sequence has no token, ORC_BAD_PAGE when a page does not resolve (unless
 * skip_invalid).
 */
int cfr_oracle_attend(const orc_problem *pr, const int32_t *sel_b, const int32_t *sel_h,
                      int64_t n_sel, int mode, int64_t arg, int skip_invalid, int nthreads,
                      int64_t mem_limit, double *out, double *lse) {
  int rc = orc_check(pr);
  if (rc) return rc;
  if (!sel_b && n_sel != (int64_t)pr->batch * pr->num_q_heads) return ORC_BAD_ARG;
  /* split the selection into runs */
  int64_t *run_start = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n_sel + 1));
  int *run_b = (int *)malloc(sizeof(int) * (size_t)(n_sel + 1));
  int *run_g = (int *)malloc(sizeof(int) * (size_t)(n_sel + 1));
  if (!run_start || !run_b || !run_g) {
    free(run_start); free(run_b); free(run_g);
    return ORC_NO_MEMORY;
  }
  int64_t nrun = 0, biggest = 0;
  for (int64_t k = 0; k < n_sel; ++k) {
    const int b = sel_b ? sel_b[k] : (int)(k / pr->num_q_heads);
    const int h = sel_h ? sel_h[k] : (int)(k % pr->num_q_heads);
    if (b < 0 || b >= pr->batch || h < 0 || h >= pr->num_q_heads) { rc = ORC_BAD_ARG; break; }
    const int g = orc_kv_head(pr, h);
    if (g < 0 || g >= pr->num_kv_heads) { rc = ORC_BAD_ARG; break; }
    if (pr->seq_lens[b] > (long)pr->max_pages * pr->page_tokens) { rc = ORC_BAD_ARG; break; }
    if (nrun == 0 || run_b[nrun - 1] != b || run_g[nrun - 1] != g) {
      run_start[nrun] = k;
      run_b[nrun] = b;
      run_g[nrun] = g;
      ++nrun;
      int64_t need = (int64_t)(pr->seq_lens[b] > 0 ? pr->seq_lens[b] : 0) * pr->head_dim * 17;
      if (need > biggest) biggest = need;
    }
  }
  run_start[nrun] = n_sel;
  int status = ORC_OK;
  if (!rc) {
    int nt = nthreads > 0 ? nthreads : 1;
    int across = nrun >= nt && nt > 1 && (mem_limit <= 0 || biggest * nt <= mem_limit);
    if (across) {
#pragma omp parallel for num_threads(nt) schedule(dynamic, 1)
      for (int64_t r = 0; r < nrun; ++r) {
        int e = orc_run(pr, sel_h, run_start[r], run_start[r + 1], run_b[r], run_g[r], mode, arg,
                        skip_invalid, 1, out, lse);
        if (e) {
#pragma omp critical
          {
            if (e != ORC_EMPTY || status == ORC_OK) status = e;
          }
        }
      }
    } else {
      for (int64_t r = 0; r < nrun; ++r) {
        int e = orc_run(pr, sel_h, run_start[r], run_start[r + 1], run_b[r], run_g[r], mode, arg,
                        skip_invalid, nt, out, lse);
        if (e && (e != ORC_EMPTY || status == ORC_OK)) status = e;
        if (e && e != ORC_EMPTY) break;
      }
    }
  }
  free(run_start); free(run_b); free(run_g);
  return rc ? rc : status;
}

/*
 * Log-sum-exp merge of split partials (the merge step of split-K decoding):
 * for each (b, h) over splits s in [split_off[b], split_off[b+1]):
 *   M = max m_s over splits with l_s > 0,  w_s = 2^(m_s - M),
 *   L = sum l_s w_s,  out = sum a_s w_s / L,  lse = (M + log2 L) * ln 2.
 * Partial maxima m are base-2 (scores times log2(e)).  With no non-empty split:
 * out = 0, lse = -inf.
 * part_acc: [S][Hq][d], part_m, part_l: [S][Hq]; out: [B][Hq][d]; lse: [B][Hq].
 */
int cfr_oracle_merge(const float *part_acc, const float *part_m, const float *part_l,
                     const int32_t *split_off, int32_t batch, int32_t num_q_heads,
                     int32_t head_dim, double *out, double *lse) {
  if (!part_acc || !part_m || !part_l || !split_off || batch < 0 || num_q_heads <= 0 ||
      head_dim <= 0 || !out || !lse)
    return ORC_BAD_ARG;
  for (int b = 0; b < batch; ++b) {
    for (int h = 0; h < num_q_heads; ++h) {
      double M = -INFINITY;
      for (int s = split_off[b]; s < split_off[b + 1]; ++s) {
        long c = (long)s * num_q_heads + h;
        if (part_l[c] > 0.0f && (double)part_m[c] > M) M = (double)part_m[c];
      }
      double L = 0.0;
      double *o = out + ((long)b * num_q_heads + h) * head_dim;
      for (int i = 0; i < head_dim; ++i) o[i] = 0.0;
      if (M == -INFINITY) {
        lse[(long)b * num_q_heads + h] = -INFINITY;
        continue;
      }
      for (int s = split_off[b]; s < split_off[b + 1]; ++s) {
        long c = (long)s * num_q_heads + h;
        if (!(part_l[c] > 0.0f)) continue;
        double w = exp2((double)part_m[c] - M);
        L += (double)part_l[c] * w;
        for (int i = 0; i < head_dim; ++i) o[i] += (double)part_acc[c * head_dim + i] * w;
      }
      for (int i = 0; i < head_dim; ++i) o[i] /= L;
      lse[(long)b * num_q_heads + h] = (M + log2(L)) * log(2.0);
    }
  }
  return ORC_OK;
}

/*
 * Bytes of K plus V that a full-KV baseline keeps resident for `tokens` tokens
 * of one head, and that one scratch page of `page_tokens` tokens holds, in
 * storage format fmt (the byte accounting of the CFR-Atlas page's benchmark
 * run: baseline_kv_bytes and cfr_scratch_bytes).
 */
int64_t cfr_oracle_kv_bytes(int32_t fmt, int64_t tokens, int32_t head_dim) {
  long rb = orc_row_bytes(fmt, head_dim);
  if (rb < 0 || tokens < 0) return -1;
  return 2 * tokens * rb;
}
