/*
 * Seeded, counter-based input generators for the QSA c4 workloads.
 *
 * This file holds no arithmetic of the attention method itself: it only
 * turns (seed, stream, counter) triples into the random numbers that build
 * synthetic inputs (index keys, queries, K/V, head weights, page-table
 * permutations, context lengths).  Both the CPU oracle and the CUDA path
 * receive byte-identical inputs from here.
 *
 * Random source: SplitMix64 (Steele, Lea and Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014) used as a pure function of a
 * 64-bit counter, so any element can be produced independently and the
 * work splits across threads without changing a single byte.
 *
 *   key(seed, stream) = mix(seed * G + mix(stream + S0))
 *   u64(i)            = mix(key + (i + 1) * G)         G = golden-ratio odd constant
 *   U(i)              = (u64(i) >> 11) * 2^-53          uniform in [0, 1)
 *   normal pair j     = Box-Muller on (1 - U(2j), U(2j+1)) in FP64:
 *                       r = sqrt(-2 ln u1), n[2j] = r cos(2 pi u2), n[2j+1] = r sin(2 pi u2)
 *   bf16              = FP64 value rounded once, to nearest even, to 8 significant bits
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL
#define STREAM_SALT 0x632BE59BD9B4E019ULL

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint64_t stream) {
  return mix64(seed * GOLDEN + mix64(stream + STREAM_SALT));
}

static inline uint64_t draw(uint64_t key, uint64_t i) { return mix64(key + (i + 1) * GOLDEN); }

static inline double unit(uint64_t x) { return (double)(x >> 11) * 0x1.0p-53; }

/* FP64 -> bf16 bits, one round-to-nearest-even step at the 8th significant bit.
 * Valid for |x| in the normal range of float (all generated values are). */
static inline uint16_t bf16_rne(double x) {
  uint64_t b;
  memcpy(&b, &x, 8);
  const uint64_t lsb = (b >> 45) & 1ULL;
  b += ((1ULL << 44) - 1ULL) + lsb;
  b &= ~((1ULL << 45) - 1ULL);
  double y;
  memcpy(&y, &b, 8);
  const float f = (float)y; /* exact: y has at most 8 significant bits */
  uint32_t u;
  memcpy(&u, &f, 4);
  return (uint16_t)(u >> 16);
}

static inline double bf16_value(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* Normal deviate number i of a stream (FP64). */
static inline double normal_at(uint64_t key, uint64_t i) {
  const uint64_t j = i >> 1;
  const double u1 = 1.0 - unit(draw(key, 2 * j));
  const double u2 = unit(draw(key, 2 * j + 1));
  const double r = sqrt(-2.0 * log(u1));
  const double a = 2.0 * M_PI * u2;
  return (i & 1) ? r * sin(a) : r * cos(a);
}

/* ---------------------------------------------------------------------------
 * A tiny fork-join helper: splits [0, n) into equal, even-aligned ranges.
 * ------------------------------------------------------------------------- */
typedef void (*range_fn)(void* ctx, int64_t lo, int64_t hi);
typedef struct {
  range_fn fn;
  void* ctx;
  int64_t lo, hi;
} range_job;

static void* run_range(void* p) {
  range_job* j = (range_job*)p;
  j->fn(j->ctx, j->lo, j->hi);
  return NULL;
}

static void parallel_for(int64_t n, int nthreads, range_fn fn, void* ctx) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (n < 65536 || nthreads == 1) {
    fn(ctx, 0, n);
    return;
  }
  pthread_t th[256];
  range_job jobs[256];
  int64_t per = (n + nthreads - 1) / nthreads;
  per = (per + 1) & ~1LL;
  int used = 0;
  for (int t = 0; t < nthreads; ++t) {
    int64_t lo = (int64_t)t * per, hi = lo + per;
    if (lo >= n) break;
    if (hi > n) hi = n;
    jobs[t].fn = fn;
    jobs[t].ctx = ctx;
    jobs[t].lo = lo;
    jobs[t].hi = hi;
    if (pthread_create(&th[t], NULL, run_range, &jobs[t]) != 0) {
      run_range(&jobs[t]);
      th[t] = 0;
    }
    used = t + 1;
  }
  for (int t = 0; t < used; ++t)
    if (th[t]) pthread_join(th[t], NULL);
}

/* ---------------------------------------------------------------------------
 * Normal bf16 tensors.
 * ------------------------------------------------------------------------- */
typedef struct {
  uint64_t key, offset;
  double std;
  uint16_t* out;
} normal_ctx;

static void normal_range(void* p, int64_t lo, int64_t hi) {
  normal_ctx* c = (normal_ctx*)p;
  for (int64_t i = lo; i < hi; ++i) c->out[i] = bf16_rne(c->std * normal_at(c->key, c->offset + (uint64_t)i));
}

void qsa_gen_normal_bf16(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, uint16_t* out,
                         int nthreads) {
  normal_ctx c = {stream_key(seed, stream), offset, 1.0, out};
  parallel_for(n, nthreads, normal_range, &c);
}

/* N(0, std^2): the same deviates times std (in FP64), rounded once to bf16. */
void qsa_gen_normal_scaled_bf16(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, double std,
                                uint16_t* out, int nthreads) {
  normal_ctx c = {stream_key(seed, stream), offset, std, out};
  parallel_for(n, nthreads, normal_range, &c);
}

/* Uniform float in [lo, hi): lo + (hi - lo) * (24-bit uniform). */
void qsa_gen_uniform_f32(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, float lo, float hi,
                         float* out) {
  const uint64_t key = stream_key(seed, stream);
  for (int64_t i = 0; i < n; ++i) {
    const float u = (float)(draw(key, offset + (uint64_t)i) >> 40) * 0x1.0p-24f;
    out[i] = lo + (hi - lo) * u;
  }
}

/* Uniform integer in [lo, hi] (inclusive), by 64x64 -> high-64 multiply. */
void qsa_gen_uniform_i64(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, int64_t lo, int64_t hi,
                         int64_t* out) {
  const uint64_t key = stream_key(seed, stream);
  const uint64_t span = (uint64_t)(hi - lo) + 1ULL;
  for (int64_t i = 0; i < n; ++i) {
    const unsigned __int128 m = (unsigned __int128)draw(key, offset + (uint64_t)i) * span;
    out[i] = lo + (int64_t)(uint64_t)(m >> 64);
  }
}

/* Bernoulli(p) flags. */
void qsa_gen_bernoulli_u8(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, double p, uint8_t* out) {
  const uint64_t key = stream_key(seed, stream);
  for (int64_t i = 0; i < n; ++i) out[i] = unit(draw(key, offset + (uint64_t)i)) < p ? 1 : 0;
}

/* Uniform random permutation of 0..n-1 (Fisher-Yates, counter i drives step i). */
void qsa_gen_permutation_i32(uint64_t seed, uint64_t stream, int64_t n, int32_t* out) {
  const uint64_t key = stream_key(seed, stream);
  for (int64_t i = 0; i < n; ++i) out[i] = (int32_t)i;
  for (int64_t i = n - 1; i > 0; --i) {
    const unsigned __int128 m = (unsigned __int128)draw(key, (uint64_t)i) * (uint64_t)(i + 1);
    const int64_t j = (int64_t)(uint64_t)(m >> 64);
    const int32_t t = out[i];
    out[i] = out[j];
    out[j] = t;
  }
}

/* ---------------------------------------------------------------------------
 * Raw index keys with a planted signal: each 4-token block is "biased" with
 * probability p (its own counter stream), and then every key of the block is
 * N(0,1) + alpha * dir, where dir is a bf16 128-vector (the unrotated head-0
 * index query of the request).  Each element is rounded to bf16 once.
 * Token t of the request uses noise counters t*128 .. t*128+127 and bias
 * counter t/4, so any token range can be produced on its own.
 * ------------------------------------------------------------------------- */
typedef struct {
  uint64_t key_noise, key_bias;
  int64_t tok0;
  double p, alpha;
  double dir[128];
  uint16_t* out;
} keys_ctx;

static void keys_range(void* pc, int64_t lo, int64_t hi) {
  keys_ctx* c = (keys_ctx*)pc;
  for (int64_t t = lo; t < hi; ++t) {
    const int64_t tok = c->tok0 + t;
    const int biased = unit(draw(c->key_bias, (uint64_t)(tok >> 2))) < c->p;
    for (int d = 0; d < 128; ++d) {
      double x = normal_at(c->key_noise, (uint64_t)tok * 128ULL + (uint64_t)d);
      if (biased) x += c->alpha * c->dir[d];
      c->out[t * 128 + d] = bf16_rne(x);
    }
  }
}

void qsa_gen_index_keys_bf16(uint64_t seed, uint64_t stream_noise, uint64_t stream_bias, int64_t tok0,
                             int64_t n_tok, const uint16_t* dir_bf16, double p, double alpha, uint16_t* out,
                             int nthreads) {
  keys_ctx c;
  c.key_noise = stream_key(seed, stream_noise);
  c.key_bias = stream_key(seed, stream_bias);
  c.tok0 = tok0;
  c.p = p;
  c.alpha = alpha;
  for (int d = 0; d < 128; ++d) c.dir[d] = dir_bf16 ? bf16_value(dir_bf16[d]) : 0.0;
  c.out = out;
  parallel_for(n_tok, nthreads, keys_range, &c);
}

/* Bias flag of each block, as qsa_gen_index_keys_bf16 draws it (for checks). */
void qsa_gen_block_bias_u8(uint64_t seed, uint64_t stream_bias, int64_t b0, int64_t n, double p, uint8_t* out) {
  const uint64_t key = stream_key(seed, stream_bias);
  for (int64_t i = 0; i < n; ++i) out[i] = unit(draw(key, (uint64_t)(b0 + i))) < p ? 1 : 0;
}
