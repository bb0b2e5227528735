/*
 * fp64 CPU oracle for batched single-token decode attention over a paged KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this library.  It shares no code, header, table or
 * constant with the CUDA path; the two meet only at the seeded inputs.
 *
 * What it computes (the plain definition, nothing more):
 *   Attention(Q, K, V) = softmax(Q K^T / sqrt(d)) V, with Q a single decode token
 *   and K, V the request's accumulated cache, including its own just-appended
 *   token.  Sources: the PAT review (section 三, 核心公式: the attention formula and
 *   "Q is a single token in decode") and the short-term-memory page (技术原理:
 *   K_t, V_t are appended to the cache, then the token attends over K_1..K_t).
 *
 * Readings where the pages are silent (the plainest reading in each case):
 *   - GQA: query head h reads kv head h / G with G = Hq / Hkv (contiguous groups).
 *   - The 1/sqrt(d) scale multiplies the fp64 dot products (d = head_dim).
 *   - lse is the natural log of the sum of exp(scaled logits).
 *   - Paging: token t of request b sits in page block_table[b][t / P], slot t % P,
 *     and a pool page is laid out [Hkv][P][D].
 *
 * Every bf16 input is widened exactly (bits << 16 -> float -> double); all
 * arithmetic is double.  Each (request, head) is computed on its own, over its
 * full un-shared KV: no tree, no split, no merge.
 *
 * oracle_merge is the log-sum-exp combine of attention results over disjoint
 * key sets (the PAT review's Merge stage, section 三, Pack-Forward-merge 范式
 * item 3: an online-softmax combine of each query's partial results).  The tests
 * pin it by the identity merge(split) == unsplit.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf16_to_f64(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/*
 * Attention of one query row over n dense keys.
 * q[D], K[n][D], V[n][D] row-major doubles; out[D]; *lse.
 * n == 0 gives out = 0 and lse = -inf.
 */
void oracle_attend_dense(int D, double scale, const double *q, const double *K, const double *V, int64_t n,
                         double *out, double *lse) {
  for (int d = 0; d < D; ++d) out[d] = 0.0;
  if (n <= 0) {
    *lse = -INFINITY;
    return;
  }
  double *score = (double *)malloc(sizeof(double) * (size_t)n);
  double m = -INFINITY;
  for (int64_t t = 0; t < n; ++t) {
    double s = 0.0;
    for (int d = 0; d < D; ++d) s += q[d] * K[t * D + d];
    score[t] = scale * s;
    if (score[t] > m) m = score[t];
  }
  double l = 0.0;
  for (int64_t t = 0; t < n; ++t) {
    double w = exp(score[t] - m);
    l += w;
    for (int d = 0; d < D; ++d) out[d] += w * V[t * D + d];
  }
  for (int d = 0; d < D; ++d) out[d] /= l;
  *lse = m + log(l);
  free(score);
}

/*
 * Log-sum-exp merge of n_parts attention results of one query row over disjoint
 * key sets: LSE = log sum_j exp(lse_j); out = sum_j exp(lse_j - LSE) o_j.
 * Parts with lse = -inf (no keys) contribute nothing.
 */
void oracle_merge(int D, int n_parts, const double *o, const double *lse, double *out, double *lse_out) {
  double m = -INFINITY;
  for (int j = 0; j < n_parts; ++j)
    if (lse[j] > m) m = lse[j];
  for (int d = 0; d < D; ++d) out[d] = 0.0;
  if (m == -INFINITY) {
    *lse_out = -INFINITY;
    return;
  }
  double z = 0.0;
  for (int j = 0; j < n_parts; ++j)
    if (lse[j] != -INFINITY) z += exp(lse[j] - m);
  double L = m + log(z);
  for (int j = 0; j < n_parts; ++j) {
    if (lse[j] == -INFINITY) continue;
    double w = exp(lse[j] - L);
    for (int d = 0; d < D; ++d) out[d] += w * o[(size_t)j * D + d];
  }
  *lse_out = L;
}

typedef struct {
  int B, Hq, Hkv, D, P, max_pages;
  double scale;
  const uint16_t *q, *k_pool, *v_pool;
  const int32_t *block_table, *kv_lens;
  const int32_t *queries; /* which requests to compute (indices into 0..B-1) */
  int n_queries;
  double *out, *lse;      /* [n_queries][Hq][D], [n_queries][Hq] */
  int64_t next;           /* shared work counter over (query, head) */
  pthread_mutex_t mu;
} paged_job;

static void attend_one(paged_job *j, int qi, int h) {
  const int b = j->queries[qi];
  const int D = j->D, P = j->P, Hkv = j->Hkv;
  const int G = j->Hq / j->Hkv;
  const int g = h / G;
  const int64_t n = j->kv_lens[b];
  double *qd = (double *)malloc(sizeof(double) * D);
  double *score = (double *)malloc(sizeof(double) * (size_t)n);
  double *out = j->out + ((size_t)qi * j->Hq + h) * D;
  for (int d = 0; d < D; ++d) qd[d] = bf16_to_f64(j->q[((size_t)b * j->Hq + h) * D + d]);
  /* token t of request b: slot t % P of page block_table[b][t / P], kv head g */
#define ORACLE_ROW(pool, t)                                                                  \
  ((pool) + ((((size_t)j->block_table[(size_t)b * j->max_pages + (t) / P] * Hkv + g) * P + \
              (size_t)((t) % P)) * D))
  double m = -INFINITY;
  for (int64_t t = 0; t < n; ++t) {
    const uint16_t *krow = ORACLE_ROW(j->k_pool, t);
    double s = 0.0;
    for (int d = 0; d < D; ++d) s += qd[d] * bf16_to_f64(krow[d]);
    score[t] = j->scale * s;
    if (score[t] > m) m = score[t];
  }
  double l = 0.0;
  for (int d = 0; d < D; ++d) out[d] = 0.0;
  for (int64_t t = 0; t < n; ++t) {
    const uint16_t *vrow = ORACLE_ROW(j->v_pool, t);
    const double w = exp(score[t] - m);
    l += w;
    for (int d = 0; d < D; ++d) out[d] += w * bf16_to_f64(vrow[d]);
  }
#undef ORACLE_ROW
  for (int d = 0; d < D; ++d) out[d] /= l;
  j->lse[(size_t)qi * j->Hq + h] = m + log(l);
  free(qd);
  free(score);
}

static void *paged_worker(void *arg) {
  paged_job *j = (paged_job *)arg;
  const int64_t total = (int64_t)j->n_queries * j->Hq;
  for (;;) {
    pthread_mutex_lock(&j->mu);
    int64_t w = j->next++;
    pthread_mutex_unlock(&j->mu);
    if (w >= total) break;
    attend_one(j, (int)(w / j->Hq), (int)(w % j->Hq));
  }
  return 0;
}

/*
 * Paged decode attention for a set of requests.
 *   q           bf16 bits [B][Hq][D]
 *   k_pool      bf16 bits [num_pages][Hkv][P][D]  (v_pool alike)
 *   block_table int32 [B][max_pages]; kv_lens int32 [B]
 *   queries     indices of the requests to compute (NULL = all B, in order)
 *   out         double [n][Hq][D]; lse double [n][Hq]
 *   scale       <= 0 selects 1/sqrt(D)
 * Returns 0, or -1 on invalid arguments (bad page id, kv_len out of range,
 * Hq not a multiple of Hkv).
 */
int oracle_attend_paged(int B, int Hq, int Hkv, int D, int P, double scale, const uint16_t *q,
                        const uint16_t *k_pool, const uint16_t *v_pool, int64_t num_pages,
                        const int32_t *block_table, int max_pages, const int32_t *kv_lens,
                        const int32_t *queries, int n_queries, double *out, double *lse, int nthreads) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || D <= 0 || P <= 0) return -1;
  int32_t *all = 0;
  if (!queries) {
    all = (int32_t *)malloc(sizeof(int32_t) * (size_t)B);
    for (int b = 0; b < B; ++b) all[b] = b;
    queries = all;
    n_queries = B;
  }
  for (int i = 0; i < n_queries; ++i) {
    int b = queries[i];
    if (b < 0 || b >= B) goto bad;
    int64_t n = kv_lens[b];
    if (n < 1 || n > (int64_t)max_pages * P) goto bad;
    for (int64_t p = 0; p < (n + P - 1) / P; ++p) {
      int64_t id = block_table[(size_t)b * max_pages + p];
      if (id < 0 || id >= num_pages) goto bad;
    }
  }
  paged_job j;
  j.B = B; j.Hq = Hq; j.Hkv = Hkv; j.D = D; j.P = P; j.max_pages = max_pages;
  j.scale = scale > 0 ? scale : 1.0 / sqrt((double)D);
  j.q = q; j.k_pool = k_pool; j.v_pool = v_pool;
  j.block_table = block_table; j.kv_lens = kv_lens;
  j.queries = queries; j.n_queries = n_queries;
  j.out = out; j.lse = lse; j.next = 0;
  pthread_mutex_init(&j.mu, 0);
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 512) nthreads = 512;
  pthread_t th[512];
  int started = 0;
  for (int t = 1; t < nthreads; ++t) {
    if (pthread_create(&th[t], 0, paged_worker, &j) != 0) break;
    started = t;
  }
  paged_worker(&j);
  for (int t = 1; t <= started; ++t) pthread_join(th[t], 0);
  pthread_mutex_destroy(&j.mu);
  free(all);
  return 0;
bad:
  free(all);
  return -1;
}
