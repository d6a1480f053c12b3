/*
 * Oracle for scaled-dot-product attention: plain, slow, fp64, materialised.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file; only the tests, the smoke check and the bench's CPU
 * baseline leg use it.  It shares no code with the CUDA library.
 *
 * What it computes (the plain definition the fused kernels reach up to
 * rounding order):
 *
 *   For batch b, query head hq, query row i (0 <= i < L):
 *     g  = Hq / Hkv, hk = floor(hq / g)          grouped-query mapping: each KV
 *                                                head serves g consecutive query
 *                                                heads (mlx issue #3826, routing
 *                                                analysis: "gqa_factor" heads per
 *                                                KV head)
 *     p  = i + (S - L)                            queries sit at the end of the KV
 *                                                sequence (mlx PR #3552,
 *                                                "Implementation": qL_off = kL - qL)
 *     s_j = scale * sum_d Q[b,hq,i,d] * K[b,hk,j,d]
 *     visible(j) = key_lo <= j < key_hi
 *                  and (not causal or j <= p)
 *                  and (W == 0 or p - j < W)      sliding window of the last W key
 *                                                positions including the query's own
 *                                                (mlx PR #3552, "Summary" and the
 *                                                left-edge rule row - col >= W masked)
 *     m   = max over visible j of s_j
 *     w_j = exp(s_j - m) for visible j, else 0
 *     l   = sum_j w_j
 *     O[b,hq,i,:] = sum_j w_j V[b,hk,j,:] / l
 *     LSE[b,hq,i] = m + log(l)
 *
 *   A row with no visible key (possible only when a key sub-range is asked
 *   for) gets O = 0 and LSE = -inf: the weight such a partial result carries
 *   in a log-sum-exp merge is zero.
 *
 *   Query offset: p = i + q_offset when the caller gives one, for a query
 *   block that does not end at the last key (chunked prefill, or keys held
 *   in a rotating window cache, addressed relative to the cache: mlx PR
 *   #3552, "Implementation", K-relative coordinates).  Without one,
 *   q_offset = S - L as above.
 *
 *   Sinks: when sinks is non-NULL, head hq has a sink logit sigma_hq that
 *   joins the softmax normalisation as one more score without a value row
 *   (the `sinks` argument of mlx PR #4185 "API" and mlx PR #3552 "Public
 *   API"; the pages name it without defining it, this is the plain reading):
 *     m'  = max(m, sigma),  l = sum_j exp(s_j - m') + exp(sigma - m'),
 *     O   = sum_j exp(s_j - m') V_j / l,  LSE = m' + log(l).
 *
 *   The key sub-range [key_lo, key_hi) exists so that a test can check one
 *   split of a split-KV pass (mlx issue #3826: split over S with a
 *   log-sum-exp merge) against the same definition restricted to its keys.
 *   The full problem is key_lo = 0, key_hi = S.
 *
 * Rows: when `rows` is non-NULL only the query rows rows[0..nrows) are
 * computed (for every b and hq), and the output is laid out
 * [B][Hq][nrows][Dv]; otherwise nrows must equal L and all rows are computed.
 *
 * Layouts: q [B][Hq][L][Dqk], k [B][Hkv][S][Dqk], v [B][Hkv][S][Dv], all
 * dense row-major fp64.  lse may be NULL.
 *
 * Mutants: when compiled with -DORACLE_MUTANT=n (n >= 1) one deliberate
 * mistake is planted, so that the tests can show that their pins catch it.
 * The normal build never defines ORACLE_MUTANT.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

typedef struct {
  const double *q, *k, *v;
  double *out, *lse;
  int64_t B, Hq, Hkv, L, S, Dqk, Dv;
  double scale;
  int causal;
  int64_t window;
  int64_t key_lo, key_hi;
  const int64_t *rows;
  int64_t nrows;
  int64_t q_offset;
  const double *sinks;
  int64_t total;      /* B * Hq * nrows work items */
  int64_t next;       /* next unclaimed work item */
  pthread_mutex_t mu;
} oracle_ctx;

static int key_visible(const oracle_ctx *c, int64_t j, int64_t p) {
  if (j < c->key_lo || j >= c->key_hi) return 0;
#if ORACLE_MUTANT == 1
  /* planted: causal bound off by one (the diagonal key is hidden) */
  if (c->causal && j >= p) return 0;
#else
  if (c->causal && j > p) return 0;
#endif
#if ORACLE_MUTANT == 2
  /* planted: window one key too wide */
  if (c->window > 0 && p - j > c->window) return 0;
#else
  if (c->window > 0 && p - j >= c->window) return 0;
#endif
  return 1;
}

/* One (b, hq, row) item.  `scores` is scratch of S doubles. */
static void oracle_row(const oracle_ctx *c, int64_t item, double *scores) {
  const int64_t r = item % c->nrows;
  const int64_t hq = (item / c->nrows) % c->Hq;
  const int64_t b = item / (c->nrows * c->Hq);
  const int64_t g = c->Hq / c->Hkv;
#if ORACLE_MUTANT == 3
  /* planted: strided instead of grouped KV-head mapping */
  const int64_t hk = hq % c->Hkv;
#else
  const int64_t hk = hq / g;
#endif
  const int64_t i = c->rows ? c->rows[r] : r;
#if ORACLE_MUTANT == 4
  /* planted: causal alignment to the start of the keys instead of the end */
  const int64_t p = i;
#else
  const int64_t p = i + c->q_offset;
#endif
  const double *qi = c->q + ((b * c->Hq + hq) * c->L + i) * c->Dqk;
  const double *kh = c->k + (b * c->Hkv + hk) * c->S * c->Dqk;
  const double *vh = c->v + (b * c->Hkv + hk) * c->S * c->Dv;
  double *o = c->out + ((b * c->Hq + hq) * c->nrows + r) * c->Dv;

  double m = -INFINITY;
  int any = 0;
  for (int64_t j = 0; j < c->S; ++j) {
    if (!key_visible(c, j, p)) continue;
    const double *kj = kh + j * c->Dqk;
    double dot = 0.0;
    for (int64_t d = 0; d < c->Dqk; ++d) dot += qi[d] * kj[d];
#if ORACLE_MUTANT == 5
    scores[j] = dot; /* planted: scale dropped */
#else
    scores[j] = c->scale * dot;
#endif
    if (!any || scores[j] > m) m = scores[j];
    any = 1;
  }

  for (int64_t d = 0; d < c->Dv; ++d) o[d] = 0.0;
  const int has_sink = c->sinks != NULL;
  const double sink = has_sink ? c->sinks[hq] : -INFINITY;
  if (!any) {
    if (c->lse) c->lse[(b * c->Hq + hq) * c->nrows + r] = has_sink ? sink : -INFINITY;
    return;
  }
  if (has_sink && sink > m) m = sink;

  double l = has_sink ? exp(sink - m) : 0.0;
  for (int64_t j = 0; j < c->S; ++j) {
    if (!key_visible(c, j, p)) continue;
    const double w = exp(scores[j] - m);
    l += w;
    const double *vj = vh + j * c->Dv;
#if ORACLE_MUTANT == 6
    /* planted: V rows indexed in reverse (a transposed operand index) */
    vj = vh + (c->S - 1 - j) * c->Dv;
#endif
    for (int64_t d = 0; d < c->Dv; ++d) o[d] += w * vj[d];
  }
#if ORACLE_MUTANT == 7
  (void)l; /* planted: missing normalisation */
#else
  for (int64_t d = 0; d < c->Dv; ++d) o[d] /= l;
#endif
  if (c->lse) c->lse[(b * c->Hq + hq) * c->nrows + r] = m + log(l);
}

static void *oracle_worker(void *arg) {
  oracle_ctx *c = (oracle_ctx *)arg;
  double *scores = (double *)malloc((size_t)(c->S > 0 ? c->S : 1) * sizeof(double));
  if (!scores) return (void *)1;
  for (;;) {
    int64_t start, stop;
    pthread_mutex_lock(&c->mu);
    start = c->next;
    stop = start + 4;
    if (stop > c->total) stop = c->total;
    c->next = stop;
    pthread_mutex_unlock(&c->mu);
    if (start >= c->total) break;
    for (int64_t it = start; it < stop; ++it) oracle_row(c, it, scores);
  }
  free(scores);
  return NULL;
}

/*
 * Returns 0 on success, a negative number for invalid arguments, -100 if a
 * thread or buffer could not be created.  nthreads <= 0 means one thread.
 */
int oracle_sdpa2_f64(const double *q, const double *k, const double *v,
                     double *out, double *lse,
                     int64_t B, int64_t Hq, int64_t Hkv, int64_t L, int64_t S,
                     int64_t Dqk, int64_t Dv, double scale, int causal,
                     int64_t window, int64_t key_lo, int64_t key_hi,
                     const int64_t *rows, int64_t nrows, int nthreads,
                     int has_q_offset, int64_t q_offset, const double *sinks) {
  if (!q || !k || !v || !out) return -1;
  if (B < 1 || Hq < 1 || Hkv < 1 || L < 1 || S < 1 || Dqk < 1 || Dv < 1) return -2;
  if (Hq % Hkv != 0) return -3;
  if (window < 0) return -4;
  if (key_lo < 0 || key_hi > S || key_lo > key_hi) return -5;
  if (rows) {
    for (int64_t r = 0; r < nrows; ++r)
      if (rows[r] < 0 || rows[r] >= L) return -6;
  } else if (nrows != L) {
    return -7;
  }
  oracle_ctx c;
  memset(&c, 0, sizeof(c));
  c.q = q; c.k = k; c.v = v; c.out = out; c.lse = lse;
  c.B = B; c.Hq = Hq; c.Hkv = Hkv; c.L = L; c.S = S; c.Dqk = Dqk; c.Dv = Dv;
  c.scale = scale; c.causal = causal; c.window = window;
  c.key_lo = key_lo; c.key_hi = key_hi;
  c.rows = rows; c.nrows = nrows;
  c.q_offset = has_q_offset ? q_offset : S - L;
  c.sinks = sinks;
  c.total = B * Hq * nrows;
  c.next = 0;
  pthread_mutex_init(&c.mu, NULL);
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  pthread_t tid[256];
  int started = 0, failed = 0;
  for (int t = 1; t < nthreads; ++t) {
    if (pthread_create(&tid[started], NULL, oracle_worker, &c) != 0) break;
    ++started;
  }
  if (oracle_worker(&c) != NULL) failed = 1;
  for (int t = 0; t < started; ++t) {
    void *ret = NULL;
    pthread_join(tid[t], &ret);
    if (ret != NULL) failed = 1;
  }
  pthread_mutex_destroy(&c.mu);
  return failed ? -100 : 0;
}

int oracle_sdpa_f64(const double *q, const double *k, const double *v,
                    double *out, double *lse,
                    int64_t B, int64_t Hq, int64_t Hkv, int64_t L, int64_t S,
                    int64_t Dqk, int64_t Dv, double scale, int causal,
                    int64_t window, int64_t key_lo, int64_t key_hi,
                    const int64_t *rows, int64_t nrows, int nthreads) {
  return oracle_sdpa2_f64(q, k, v, out, lse, B, Hq, Hkv, L, S, Dqk, Dv, scale, causal, window,
                          key_lo, key_hi, rows, nrows, nthreads, 0, 0, NULL);
}

int oracle_mutant_id(void) { return ORACLE_MUTANT; }
