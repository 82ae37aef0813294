/*
 * ORACLE — TEST INFRASTRUCTURE ONLY.  Not part of the product path; only the
 * tests, the smoke check and the benchmark's CPU-baseline leg may load it.
 * It shares no code, header or constant with the CUDA library.
 *
 * The reference model of prefix-sliding attention, in float64 on the CPU:
 * attention of one query over an explicit list of history rows (position,
 * key, value), with every row that the visibility rule excludes masked to
 * minus infinity before the softmax.  The list may be the whole history or any
 * superset of the visible rows: masked rows get softmax weight exactly 0.
 *
 * Sources:
 *  - "Formal verification of a sliding-window KV cache in Lean4" (pnsm.cn
 *    blog), section 2.1: the reference implementation keeps the full K/V
 *    history and applies a window mask (logits of positions older than
 *    t-W+1 set to minus infinity) plus a causal mask, then softmax(q K^T /
 *    sqrt(d)) V.
 *  - "Prefix Sliding" digest (longzhangge.com PaperDaily), section 03: the
 *    query at step t sees the pinned prefix [1,P] and the recent window
 *    [max(P+1, t-W+1), t]; written here 0-indexed as [0,P) and
 *    [max(P, t-W+1), t].
 * Readings where the pages are silent: a query inside the prefix (t < P)
 * sees [0, t] (plain causal); the softmax scale is supplied by the caller.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>

/* Visibility of history position p for the query at position t. */
int oracle_is_visible(int64_t P, int64_t W, int64_t t, int64_t p) {
  if (p < 0 || p > t) return 0;   /* causal mask: nothing after the query */
  if (t < P) return 1;            /* query inside the pinned prompt: causal only */
  if (p < P) return 1;            /* the pinned prefix is never masked */
  int64_t lo = t - W + 1;         /* window mask: positions below t-W+1 */
  if (lo < P) lo = P;             /* the window starts after the prefix */
  return p >= lo;
}

/* mask[i] = visibility of position p0+i, for i in [0, n). */
void oracle_visible_mask(int64_t P, int64_t W, int64_t t, int64_t p0, int64_t n,
                         uint8_t* mask) {
  for (int64_t i = 0; i < n; ++i) mask[i] = (uint8_t)oracle_is_visible(P, W, t, p0 + i);
}

/*
 * out[h][:] = sum_r softmax_r(z_hr) v_r, with
 *   z_hr = scale * <q_h, k_r>  if row r is visible, minus infinity otherwise,
 * for the G query heads h that share this key/value head.
 * q: [G][d]; hpos: [nh]; hk, hv: [nh][d]; out: [G][d]; z: scratch [nh].
 * Returns the number of visible rows (0 means the output is undefined/NaN).
 */
int64_t oracle_attend(int64_t P, int64_t W, int64_t t, double scale, int G, int d,
                      const double* q, int64_t nh, const int64_t* hpos,
                      const double* hk, const double* hv, double* out, double* z) {
  int64_t nvis = 0;
  for (int64_t r = 0; r < nh; ++r) nvis += oracle_is_visible(P, W, t, hpos[r]);
  for (int h = 0; h < G; ++h) {
    const double* qh = q + (size_t)h * d;
    double* oh = out + (size_t)h * d;
    double m = -INFINITY;
    for (int64_t r = 0; r < nh; ++r) {
      if (oracle_is_visible(P, W, t, hpos[r])) {
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += qh[c] * hk[(size_t)r * d + c];
        z[r] = scale * dot;
        if (z[r] > m) m = z[r];
      } else {
        z[r] = -INFINITY;
      }
    }
    double den = 0.0;
    for (int c = 0; c < d; ++c) oh[c] = 0.0;
    for (int64_t r = 0; r < nh; ++r) {
      if (z[r] == -INFINITY) continue;  /* exp(-inf - m) = 0: contributes nothing */
      double w = exp(z[r] - m);
      den += w;
      for (int c = 0; c < d; ++c) oh[c] += w * hv[(size_t)r * d + c];
    }
    for (int c = 0; c < d; ++c) oh[c] /= den;
  }
  return nvis;
}

/* One independent attention problem (one query position, one key/value head). */
typedef struct {
  int64_t P, W, t;
  double scale;
  int32_t G, d;
  const double* q;
  int64_t nh;
  const int64_t* hpos;
  const double* hk;
  const double* hv;
  double* out;
  int64_t nvis; /* written back */
} oracle_problem;

typedef struct {
  oracle_problem* probs;
  int64_t nprob;
  int64_t next;
  pthread_mutex_t lock;
} pool_t;

static void* pool_worker(void* arg) {
  pool_t* pool = (pool_t*)arg;
  double* z = NULL;
  int64_t zcap = 0;
  for (;;) {
    pthread_mutex_lock(&pool->lock);
    int64_t i = pool->next++;
    pthread_mutex_unlock(&pool->lock);
    if (i >= pool->nprob) break;
    oracle_problem* p = &pool->probs[i];
    if (p->nh > zcap) {
      free(z);
      zcap = p->nh;
      z = (double*)malloc(sizeof(double) * (size_t)(zcap > 0 ? zcap : 1));
    }
    p->nvis = oracle_attend(p->P, p->W, p->t, p->scale, p->G, p->d, p->q, p->nh, p->hpos,
                            p->hk, p->hv, p->out, z);
  }
  free(z);
  return NULL;
}

/* Solve nprob independent problems on nthreads host threads. */
void oracle_attend_many(oracle_problem* probs, int64_t nprob, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  pool_t pool;
  pool.probs = probs;
  pool.nprob = nprob;
  pool.next = 0;
  pthread_mutex_init(&pool.lock, NULL);
  pthread_t th[256];
  for (int i = 1; i < nthreads; ++i) pthread_create(&th[i], NULL, pool_worker, &pool);
  pool_worker(&pool);
  for (int i = 1; i < nthreads; ++i) pthread_join(th[i], NULL);
  pthread_mutex_destroy(&pool.lock);
}
