/*
 * Seeded synthetic-input generator (host, C99 + pthreads).
 *
 * This module only draws random numbers and writes them into caller buffers.
 * It holds no attention arithmetic, and it is the one piece of code that both
 * the fp64 oracle (through the tests) and the CUDA path (through the tests and
 * the benchmark) consume.
 *
 * Generators, each from its published definition:
 *   - SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number
 *     generators", OOPSLA 2014; the 64-bit finaliser constants of Vigna's
 *     public-domain splitmix64.c) expands a 64-bit seed into xoshiro state.
 *   - xoshiro256** (Blackman and Vigna, "Scrambled linear pseudorandom number
 *     generators", ACM TOMS 2021) produces the stream.
 *   - Box-Muller (1958) turns two uniforms into two N(0,1) draws.
 *
 * Stream derivation: a stream is named by (seed, tag, index).  Its xoshiro
 * state is four consecutive SplitMix64 outputs started from
 *     seed ^ (tag * 0x9E3779B97F4A7C15) ^ (index * 0xD1B54A32D192ED03).
 * Every KV page is its own stream keyed by its physical page id, so pages can
 * be filled in parallel and the result does not depend on the thread count.
 *
 * Rounding: a normal draw is computed in double, rounded to float with the C
 * conversion (round-to-nearest-even), then to bf16 with round-to-nearest-even.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

typedef struct { uint64_t s[4]; } xo256;

static uint64_t splitmix64_next(uint64_t *x) {
  uint64_t z = (*x += 0x9E3779B97F4A7C15ULL);
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint64_t rotl64(uint64_t x, int k) { return (x << k) | (x >> (64 - k)); }

static uint64_t xo_next(xo256 *g) {
  uint64_t *s = g->s;
  const uint64_t result = rotl64(s[1] * 5, 7) * 9;
  const uint64_t t = s[1] << 17;
  s[2] ^= s[0];
  s[3] ^= s[1];
  s[1] ^= s[2];
  s[0] ^= s[3];
  s[2] ^= t;
  s[3] = rotl64(s[3], 45);
  return result;
}

static void xo_seed(xo256 *g, uint64_t seed, uint64_t tag, uint64_t index) {
  uint64_t x = seed ^ (tag * 0x9E3779B97F4A7C15ULL) ^ (index * 0xD1B54A32D192ED03ULL);
  for (int i = 0; i < 4; ++i) g->s[i] = splitmix64_next(&x);
}

/* uniform double in [0, 1) with 53 random bits */
static inline double xo_unit(xo256 *g) { return (double)(xo_next(g) >> 11) * 0x1.0p-53; }

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return 0x7FC0; /* NaN */
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

/* Fill n values of one stream with N(0,1) rounded to bf16 (Box-Muller pairs). */
static void fill_normal_bf16(xo256 *g, uint16_t *out, int64_t n) {
  const double two_pi = 6.283185307179586476925286766559;
  int64_t i = 0;
  while (i < n) {
    double u1 = 1.0 - xo_unit(g); /* (0, 1] so the log is finite */
    double u2 = xo_unit(g);
    double r = sqrt(-2.0 * log(u1));
    double z0 = r * cos(two_pi * u2);
    double z1 = r * sin(two_pi * u2);
    out[i++] = f32_to_bf16_rne((float)z0);
    if (i < n) out[i++] = f32_to_bf16_rne((float)z1);
  }
}

/* ---------------------------------------------------------------- exports */

/* n raw 64-bit outputs of stream (seed, tag, index). */
void pagen_u64(uint64_t seed, uint64_t tag, uint64_t index, int64_t n, uint64_t *out) {
  xo256 g;
  xo_seed(&g, seed, tag, index);
  for (int64_t i = 0; i < n; ++i) out[i] = xo_next(&g);
}

/* n uniform doubles in [0, 1) of stream (seed, tag, index). */
void pagen_unit(uint64_t seed, uint64_t tag, uint64_t index, int64_t n, double *out) {
  xo256 g;
  xo_seed(&g, seed, tag, index);
  for (int64_t i = 0; i < n; ++i) out[i] = xo_unit(&g);
}

/* n standard normals (double, before any rounding) of stream (seed, tag, index). */
void pagen_normal_f64(uint64_t seed, uint64_t tag, uint64_t index, int64_t n, double *out) {
  const double two_pi = 6.283185307179586476925286766559;
  xo256 g;
  xo_seed(&g, seed, tag, index);
  int64_t i = 0;
  while (i < n) {
    double u1 = 1.0 - xo_unit(&g);
    double u2 = xo_unit(&g);
    double r = sqrt(-2.0 * log(u1));
    out[i++] = r * cos(two_pi * u2);
    if (i < n) out[i++] = r * sin(two_pi * u2);
  }
}

/* n N(0,1) values rounded to bf16 bit patterns, stream (seed, tag, index). */
void pagen_normal_bf16(uint64_t seed, uint64_t tag, uint64_t index, int64_t n, uint16_t *out) {
  xo256 g;
  xo_seed(&g, seed, tag, index);
  fill_normal_bf16(&g, out, n);
}

/* Uniform random permutation of 0..n-1 (Fisher-Yates, stream (seed, tag, 0)). */
void pagen_permutation(uint64_t seed, uint64_t tag, int64_t n, int32_t *out) {
  xo256 g;
  xo_seed(&g, seed, tag, 0);
  for (int64_t i = 0; i < n; ++i) out[i] = (int32_t)i;
  for (int64_t i = n - 1; i > 0; --i) {
    int64_t j = (int64_t)(xo_unit(&g) * (double)(i + 1));
    if (j > i) j = i;
    int32_t t = out[i];
    out[i] = out[j];
    out[j] = t;
  }
}

typedef struct {
  uint64_t seed, tag;
  const int32_t *page_ids;
  int64_t lo, hi, elems_per_page;
  uint16_t *pool;
} page_job;

static void *page_worker(void *arg) {
  page_job *j = (page_job *)arg;
  for (int64_t i = j->lo; i < j->hi; ++i) {
    int64_t p = j->page_ids[i];
    xo256 g;
    xo_seed(&g, j->seed, j->tag, (uint64_t)p);
    fill_normal_bf16(&g, j->pool + p * j->elems_per_page, j->elems_per_page);
  }
  return 0;
}

/*
 * Fill pool pages page_ids[0..npages) with N(0,1) bf16 values.  Page p is the
 * stream (seed, tag, p) and holds elems_per_page contiguous values.
 */
void pagen_fill_pages(uint64_t seed, uint64_t tag, const int32_t *page_ids, int64_t npages,
                      int64_t elems_per_page, uint16_t *pool, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (npages < nthreads) nthreads = npages > 0 ? (int)npages : 1;
  pthread_t th[256];
  page_job jobs[256];
  for (int t = 0; t < nthreads; ++t) {
    jobs[t].seed = seed;
    jobs[t].tag = tag;
    jobs[t].page_ids = page_ids;
    jobs[t].lo = npages * t / nthreads;
    jobs[t].hi = npages * (t + 1) / nthreads;
    jobs[t].elems_per_page = elems_per_page;
    jobs[t].pool = pool;
  }
  int started = 0;
  for (int t = 1; t < nthreads; ++t) {
    if (pthread_create(&th[t], 0, page_worker, &jobs[t]) != 0) break;
    started = t;
  }
  page_worker(&jobs[0]);
  for (int t = 1; t <= started; ++t) pthread_join(th[t], 0);
  for (int t = started + 1; t < nthreads; ++t) page_worker(&jobs[t]); /* threads that failed to start */
}

/* Write value v into n consecutive uint16 slots (used for NaN poisoning). */
void pagen_fill_u16(uint16_t *p, int64_t n, uint16_t v) {
  for (int64_t i = 0; i < n; ++i) p[i] = v;
}
