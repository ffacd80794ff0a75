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
 *     I4 nibble code * scale, FP8 E4M3 value * scale, with
 *     scale = scales[fmt][slot][g][0 for K, 1 for V]
 *     (ARGUS page, "Visual Architecture": the FP8, INT8 and INT4 tiers of the
 *     compression cascade; "Why It Works: Storage vs. Computation": pages are
 *     stored compressed and restored to full precision before attention);
 *   - sigma = softmax_scale, or 1/sqrt(d) when softmax_scale is 0;
 *   - bias_j = -slope_h * (n - 1 - j) with ALiBi slopes, else 0
 *     (CFR-Atlas page, "RoPE/ALiBi positional policy");
 *   - kv head g = head_map[h], or h / (Hq / Hkv) when head_map is NULL
 *     (CFR-Atlas page, "MHA/MQA/GQA head mapping").
 *
 * Token subsets: with window_tokens > 0 the softmax runs over the tokens
 * j < sink_tokens and j >= n - window_tokens only (the attention sinks kept by
 * the ARGUS page, "sink_tokens: keep initial attention sinks", and the recent
 * window of the CFR-Atlas page's KeepRecent policy; exactness holds on the
 * chosen set); ALiBi distances stay n - 1 - j.
 *
 * Several queries per sequence (num_queries = Q > 1): the queries are the
 * last Q tokens of the sequence, at positions n - Q + i (i = 0..Q-1), with q
 * laid out [B][Q][Hq][d]; query i attends causally to the tokens j <= n - Q + i
 * (the causal mask of the RustAttention page, "Mathematical Framework
 * Covered", applied to the query rows of a speculative or chunked-prefill
 * step over the paged cache), with ALiBi distance n - Q + i - j.  Query i of
 * sequence b is therefore the single-query definition over the first
 * n - Q + i + 1 tokens.  Outputs are [B][Q][Hq][d] and [B][Q][Hq].
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
#define ORC_FP8 4
#define ORC_NFMT 5

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
  const float *scales[ORC_NFMT];       /* [slots][Hkv][2] for I8/I4/FP8 */
  int64_t pool_pages[ORC_NFMT];
  const int32_t *page_table;           /* [B][max_pages] */
  const uint8_t *page_fmt;             /* [B][max_pages] or NULL */
  const int32_t *seq_lens;             /* [B] */
  const int32_t *head_map;             /* [Hq] or NULL */
  const float *alibi_slopes;           /* [Hq] or NULL */
  double softmax_scale;                /* 0 => 1/sqrt(d) */
  int32_t sink_tokens, window_tokens;  /* window_tokens > 0: attend to [0, sink) and [n-window, n) only */
  int32_t num_queries;                 /* Q >= 1 query tokens per sequence (0 is read as 1) */
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

/*
 * FP8 E4M3 (the OCP 8-bit floating-point format without infinities): sign bit,
 * 4 exponent bits with bias 7, 3 mantissa bits.  Exponent field 0 holds the
 * subnormals m * 2^-9; fields 1..15 hold (1 + m/8) * 2^(e-7), except e = 15,
 * m = 7, which is NaN.  Largest finite magnitude: 448.
 */
static double orc_e4m3_value(unsigned char byte) {
  const int e = (byte >> 3) & 15, m = byte & 7;
  double mag;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) mag = ldexp((double)m, -9);
  else mag = ldexp(1.0 + m / 8.0, e - 7);
  return (byte & 0x80) ? -mag : mag;
}

static int orc_quantised(int fmt) { return fmt == ORC_I8 || fmt == ORC_I4 || fmt == ORC_FP8; }

static long orc_row_bytes(int fmt, int d) {
  switch (fmt) {
    case ORC_F32: return 4L * d;
    case ORC_BF16: return 2L * d;
    case ORC_I8: return (long)d;
    case ORC_I4: return (long)d / 2;
    case ORC_FP8: return (long)d;
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
    case ORC_FP8: return orc_e4m3_value(row[i]) * scale;
  }
  return NAN;
}

static int orc_nq(const orc_problem *pr) { return pr->num_queries > 1 ? pr->num_queries : 1; }

/* element i of query row (b, query qi, head h) */
static double orc_query(const orc_problem *pr, int b, int qi, int h, int i) {
  long idx = (((long)b * orc_nq(pr) + qi) * pr->num_q_heads + h) * pr->head_dim + i;
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
             (!orc_quantised(fmt) || pr->scales[fmt]);
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
    if (orc_quantised(fmt)) {
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

/*
 * one (b, query row vh): out[d] and lse.  vh = qi * Hq + h selects query qi of
 * head h; that query sees the first n - Q + qi + 1 of the n materialised tokens
 * (all n with one query).  K/V/keep are materialised for the kv head of h.
 */
static int orc_one(const orc_problem *pr, int b, int vh, int n_all, const double *K,
                   const double *V, const unsigned char *keep, int mode, long arg, double *out,
                   double *lse) {
  const int d = pr->head_dim, P = pr->page_tokens;
  const int h = vh % pr->num_q_heads, qi = vh / pr->num_q_heads;
  const int n = n_all - orc_nq(pr) + qi + 1;
  if (n <= 0) {
    for (int i = 0; i < d; ++i) out[i] = 0.0;
    *lse = -INFINITY;
    return ORC_EMPTY;
  }
  double *qv = (double *)malloc(sizeof(double) * d);
  double *a = (double *)malloc(sizeof(double) * d);
  double *a2 = (double *)malloc(sizeof(double) * d);
  if (!qv || !a || !a2) {
    free(qv); free(a); free(a2);
    return ORC_NO_MEMORY;
  }
  for (int i = 0; i < d; ++i) qv[i] = orc_query(pr, b, qi, h, i);
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
  if (pr->sink_tokens < 0 || pr->window_tokens < 0) return ORC_BAD_ARG;
  if (pr->num_queries < 0 || (orc_nq(pr) > 1 && pr->window_tokens > 0)) return ORC_BAD_ARG;
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
  if (!rc && pr->window_tokens > 0) {
    /* only the sink tokens and the recent window take part */
    for (int j = 0; j < n; ++j)
      if (!(j < pr->sink_tokens || j >= n - pr->window_tokens)) keep[j] = 0;
  }
  int err = ORC_OK;
  if (!rc) {
#pragma omp parallel for num_threads(nthreads > 0 ? nthreads : 1) schedule(dynamic, 1)
    for (int64_t kk = k0; kk < k1; ++kk) {
      const int64_t rows = (int64_t)orc_nq(pr) * pr->num_q_heads;
      const int vh = sel_h ? sel_h[kk] : (int)(kk % rows);
      int r = orc_one(pr, b, vh, n, K, V, keep, mode, arg, out + kk * d, lse + kk);
      if (r) {
#pragma omp critical
        err = (err == ORC_OK || err == ORC_EMPTY) ? r : err;
      }
    }
  }
  free(K); free(V); free(keep);
  return rc ? rc : err;
}

/*
 * Attention output for the selected (sel_b[k], sel_h[k]) pairs, k < n_sel, in
 * that order (all pairs b-major when sel_b is NULL: n_sel must be B*Q*Hq).
 * sel_h is a query row vh = qi * Hq + h (just h with one query).
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
  const int64_t rows = (int64_t)orc_nq(pr) * pr->num_q_heads;  /* query rows per sequence */
  if (!sel_b && n_sel != (int64_t)pr->batch * rows) return ORC_BAD_ARG;
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
    const int b = sel_b ? sel_b[k] : (int)(k / rows);
    const int vh = sel_h ? sel_h[k] : (int)(k % rows);
    if (b < 0 || b >= pr->batch || vh < 0 || vh >= rows) { rc = ORC_BAD_ARG; break; }
    const int g = orc_kv_head(pr, vh % pr->num_q_heads);
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

/* ---- page demotion and KV append ----------------------------------------
 *
 * The compression cascade of the ARGUS page ("Visual Architecture": hot pages
 * in full precision, cold pages re-encoded FP8 -> INT8 -> INT4) re-encodes a
 * whole page of one storage format into another.  The reading followed here,
 * per (page, kv head, K-or-V) block of P rows x d, over its `valid` first rows:
 *
 *   x      = the stored value as fp32 (F32 as is, BF16 widened, quantised
 *            formats code * scale rounded to fp32);
 *   amax   = max |x| over the valid rows (fp32);
 *   scale  = amax / Q in fp32, Q = 127 (I8), 7 (I4), 448 (FP8);
 *   I8/I4  code = clamp(round_half_even(x / scale), -Q, Q), the division in fp32;
 *   FP8    code = E4M3 nearest to x / scale (ties to even, saturating at 448);
 *   BF16   x rounded to bfloat16 (nearest, ties to even);
 *   F32    x.
 * With amax = 0 the scale is 0 and every code is 0; a NaN value gets integer
 * code 0 and the FP8 NaN code 0x7F.  Rows at or past `valid`
 * are written as zero bytes.  Every decision that turns a float into a code is
 * taken in fp32, the precision in which the values are stored.
 */

#define ORC_DEV_PAGE_ID 0x1u
#define ORC_DEV_PAGE_FMT 0x2u
#define ORC_DEV_SEQ_LEN 0x4u

static float orc_value_f32(int fmt, const unsigned char *row, int i, float scale) {
  switch (fmt) {
    case ORC_F32: {
      float f;
      memcpy(&f, row + 4L * i, sizeof f);
      return f;
    }
    case ORC_BF16: return (float)orc_from_bf16(row + 2L * i);
    case ORC_I8: return (float)orc_i8_code(row[i]) * scale;
    case ORC_I4: return (float)orc_i4_code(row[i / 2], i % 2) * scale;
    case ORC_FP8: return (float)orc_e4m3_value(row[i]) * scale;
  }
  return NAN;
}

/* bfloat16 nearest to x (ties to even); NaN becomes the quiet NaN 0x7FC0 */
static uint16_t orc_bf16_bits(float x) {
  uint32_t w;
  memcpy(&w, &x, sizeof w);
  if (isnan(x)) return 0x7FC0;
  /* keep the upper 16 bits, adding half an ulp of bf16 minus one unless the kept part is odd */
  uint32_t lsb = (w >> 16) & 1u;
  w += 0x7FFFu + lsb;
  return (uint16_t)(w >> 16);
}

/* E4M3 code nearest to x (ties to even mantissa), magnitudes above 448 saturate to 448 */
static unsigned char orc_e4m3_code(float x) {
  if (isnan(x)) return 0x7F;
  const unsigned char sign = signbit(x) ? 0x80 : 0x00;
  double a = fabs((double)x);
  if (a >= 448.0) return sign | 0x7E;
  if (a < ldexp(1.0, -6)) {
    /* subnormal range: multiples of 2^-9; 8 * 2^-9 is the smallest normal, code 0x08 */
    int m = (int)rint(ldexp(a, 9));
    return sign | (unsigned char)m;
  }
  int k;
  (void)frexp(a, &k);            /* a = f * 2^k, f in [0.5, 1) */
  int e = k - 1;                 /* a in [2^e, 2^(e+1)) */
  int r = (int)rint(ldexp(a, 3 - e));  /* in [8, 16] */
  if (r == 16) {
    r = 8;
    ++e;
  }
  int code = ((e + 7) << 3) | (r - 8);
  if (code > 0x7E) code = 0x7E;
  return sign | (unsigned char)code;
}

static int orc_qmax(int fmt) { return fmt == ORC_I8 ? 127 : fmt == ORC_I4 ? 7 : 448; }

/* re-encodes one block: src rows [P][rb_src] -> dst rows [P][rb_dst] */
static void orc_demote_block(int src_fmt, const unsigned char *src, float src_scale, int dst_fmt,
                             unsigned char *dst, float *dst_scale, int P, int d, int valid) {
  const long rs = orc_row_bytes(src_fmt, d), rd = orc_row_bytes(dst_fmt, d);
  memset(dst, 0, (size_t)(rd * P));
  float scale = 0.0f;
  if (orc_quantised(dst_fmt)) {
    float amax = 0.0f;
    for (int t = 0; t < valid; ++t)
      for (int i = 0; i < d; ++i) {
        float a = fabsf(orc_value_f32(src_fmt, src + t * rs, i, src_scale));
        if (a > amax) amax = a;
      }
    scale = amax / (float)orc_qmax(dst_fmt);
    *dst_scale = scale;
  }
  for (int t = 0; t < valid; ++t) {
    unsigned char *row = dst + t * rd;
    for (int i = 0; i < d; ++i) {
      const float x = orc_value_f32(src_fmt, src + t * rs, i, src_scale);
      if (dst_fmt == ORC_F32) {
        memcpy(row + 4L * i, &x, sizeof x);
      } else if (dst_fmt == ORC_BF16) {
        uint16_t hbits = orc_bf16_bits(x);
        memcpy(row + 2L * i, &hbits, sizeof hbits);
      } else if (dst_fmt == ORC_FP8) {
        row[i] = scale > 0.0f ? orc_e4m3_code(x / scale) : 0;
      } else {
        const int q = orc_qmax(dst_fmt);
        int c = 0;
        if (scale > 0.0f) {
          float r = rintf(x / scale);
          c = isnan(r) ? 0 : r > (float)q ? q : r < (float)-q ? -q : (int)r;
        }
        if (dst_fmt == ORC_I8) {
          row[i] = (unsigned char)(c & 0xFF);
        } else {
          const unsigned char nib = (unsigned char)(c & 15);
          row[i / 2] |= (i % 2) ? (unsigned char)(nib << 4) : nib;
        }
      }
    }
  }
}

/*
 * Demotes num_pages pages: page k is read from slot src_slots[k] of the source
 * pool (format src_fmt) and written to slot dst_slots[k] of the destination
 * pool (format dst_fmt), every kv head, K and V, over its valid_tokens[k] first
 * rows (all P when valid_tokens is NULL).  Pools are
 * [slots][Hkv][P][row_bytes]; scales [slots][Hkv][2] (K, V).  A page whose
 * slot is out of range (ORC_DEV_PAGE_ID) or whose valid count is outside
 * [1, P] (ORC_DEV_SEQ_LEN) is skipped and the bit is OR-ed into *err.
 */
int cfr_oracle_demote(int32_t num_kv_heads, int32_t head_dim, int32_t page_tokens,
                      int32_t src_fmt, const uint8_t *src_k, const uint8_t *src_v,
                      const float *src_scales, int64_t src_pages, int32_t dst_fmt,
                      uint8_t *dst_k, uint8_t *dst_v, float *dst_scales, int64_t dst_pages,
                      const int32_t *src_slots, const int32_t *dst_slots,
                      const int32_t *valid_tokens, int32_t num_pages, uint32_t *err) {
  if (num_kv_heads <= 0 || head_dim <= 0 || head_dim % 2 || page_tokens <= 0 || num_pages < 0 ||
      src_fmt < 0 || src_fmt >= ORC_NFMT || dst_fmt < 0 || dst_fmt >= ORC_NFMT ||
      !src_k || !src_v || !dst_k || !dst_v || !src_slots || !dst_slots || !err ||
      (orc_quantised(src_fmt) && !src_scales) || (orc_quantised(dst_fmt) && !dst_scales))
    return ORC_BAD_ARG;
  const int d = head_dim, P = page_tokens, H = num_kv_heads;
  const long rs = orc_row_bytes(src_fmt, d), rd = orc_row_bytes(dst_fmt, d);
  for (int k = 0; k < num_pages; ++k) {
    const int64_t s = src_slots[k], t = dst_slots[k];
    const int valid = valid_tokens ? valid_tokens[k] : P;
    if (s < 0 || s >= src_pages || t < 0 || t >= dst_pages) {
      *err |= ORC_DEV_PAGE_ID;
      continue;
    }
    if (valid < 1 || valid > P) {
      *err |= ORC_DEV_SEQ_LEN;
      continue;
    }
    for (int g = 0; g < H; ++g) {
      const long src_off = (s * H + g) * (long)P * rs, dst_off = (t * H + g) * (long)P * rd;
      const float ks = orc_quantised(src_fmt) ? src_scales[(s * H + g) * 2 + 0] : 1.0f;
      const float vs = orc_quantised(src_fmt) ? src_scales[(s * H + g) * 2 + 1] : 1.0f;
      float kd = 0.0f, vd = 0.0f;
      orc_demote_block(src_fmt, src_k + src_off, ks, dst_fmt, dst_k + dst_off, &kd, P, d, valid);
      orc_demote_block(src_fmt, src_v + src_off, vs, dst_fmt, dst_v + dst_off, &vd, P, d, valid);
      if (orc_quantised(dst_fmt)) {
        dst_scales[(t * H + g) * 2 + 0] = kd;
        dst_scales[(t * H + g) * 2 + 1] = vd;
      }
    }
  }
  return ORC_OK;
}

/*
 * Appends one token to every sequence b with positions[b] >= 0: the new K and
 * V rows k_new[b][g][:], v_new[b][g][:] (fp32 or bf16 by new_fmt) become token
 * j = positions[b] of the sequence, i.e. row j % P of logical page j / P,
 * whose slot and format come from the page table as in the decode.  The page
 * must be an F32 or BF16 page (new tokens enter the full-precision hot tier,
 * ARGUS page, "The One-Minute Explanation": recent tokens stay in high
 * precision); values are widened to F32 or rounded to BF16 (nearest, ties to
 * even).  Faults are skipped and reported in *err: j beyond max_pages * P
 * (ORC_DEV_SEQ_LEN), a quantised or unknown page format or a missing pool
 * (ORC_DEV_PAGE_FMT), a slot outside its pool (ORC_DEV_PAGE_ID).
 */
int cfr_oracle_append(int32_t num_kv_heads, int32_t head_dim, int32_t page_tokens,
                      uint8_t *const *k_pool, uint8_t *const *v_pool, const int64_t *pool_pages,
                      const int32_t *page_table, int32_t max_pages, const uint8_t *page_fmt,
                      int32_t uniform_fmt, const int32_t *positions, int32_t batch,
                      int32_t new_fmt, const void *k_new, const void *v_new, uint32_t *err) {
  if (num_kv_heads <= 0 || head_dim <= 0 || page_tokens <= 0 || max_pages < 0 || batch < 0 ||
      !k_pool || !v_pool || !pool_pages || !page_table || !positions || !k_new || !v_new ||
      !err || (new_fmt != ORC_F32 && new_fmt != ORC_BF16))
    return ORC_BAD_ARG;
  const int d = head_dim, P = page_tokens, H = num_kv_heads;
  for (int b = 0; b < batch; ++b) {
    const long j = positions[b];
    if (j < 0) continue;
    if (j >= (long)max_pages * P) {
      *err |= ORC_DEV_SEQ_LEN;
      continue;
    }
    const long cell = (long)b * max_pages + j / P;
    const int fmt = page_fmt ? (int)page_fmt[cell] : uniform_fmt;
    if ((fmt != ORC_F32 && fmt != ORC_BF16) || !k_pool[fmt] || !v_pool[fmt]) {
      *err |= ORC_DEV_PAGE_FMT;
      continue;
    }
    const long slot = page_table[cell];
    if (slot < 0 || slot >= pool_pages[fmt]) {
      *err |= ORC_DEV_PAGE_ID;
      continue;
    }
    const long rb = orc_row_bytes(fmt, d);
    for (int g = 0; g < H; ++g) {
      unsigned char *kr = k_pool[fmt] + ((slot * H + g) * (long)P + j % P) * rb;
      unsigned char *vr = v_pool[fmt] + ((slot * H + g) * (long)P + j % P) * rb;
      for (int i = 0; i < d; ++i) {
        const long e = ((long)b * H + g) * d + i;
        float kx, vx;
        if (new_fmt == ORC_F32) {
          kx = ((const float *)k_new)[e];
          vx = ((const float *)v_new)[e];
        } else {
          kx = (float)orc_from_bf16((const unsigned char *)k_new + 2 * e);
          vx = (float)orc_from_bf16((const unsigned char *)v_new + 2 * e);
        }
        if (fmt == ORC_F32) {
          memcpy(kr + 4L * i, &kx, sizeof kx);
          memcpy(vr + 4L * i, &vx, sizeof vx);
        } else {
          uint16_t kb = orc_bf16_bits(kx), vb = orc_bf16_bits(vx);
          memcpy(kr + 2L * i, &kb, sizeof kb);
          memcpy(vr + 2L * i, &vb, sizeof vb);
        }
      }
    }
  }
  return ORC_OK;
}

/* the E4M3 code of x and the decoded value of a code, exposed for pinning */
int32_t cfr_oracle_e4m3_code(float x) { return orc_e4m3_code(x); }
double cfr_oracle_e4m3_value(int32_t code) { return orc_e4m3_value((unsigned char)code); }
int32_t cfr_oracle_bf16_bits(float x) { return orc_bf16_bits(x); }
