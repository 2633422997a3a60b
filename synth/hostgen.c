/*
 * hostgen.c -- a plain C twin of the seeded synthetic generator in
 * synth/__init__.py, for large host-side draws (the oracle of the full-size
 * workloads needs billions of them; NumPy makes about five million a second
 * per core).
 *
 * It draws random numbers and nothing else: the SplitMix64 stream
 * mix64(key + n * GAMMA) with the Mix13 finaliser of Steele, Lea and Flood,
 * "Fast splittable pseudorandom number generators" (OOPSLA 2014), the
 * counter packing of the NumPy module, the Irwin-Hall sum of twelve 16-bit
 * uniforms and the nearest-even bf16 rounding.  Every value must equal the
 * NumPy generator's bit for bit (a CPU test checks it); the NumPy module
 * stays the definition.
 *
 * Threads: each call splits its rows over up to n_threads POSIX threads.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

#define GAMMA 0x9E3779B97F4A7C15ull
#define IRWIN_HALL_CENTER 393210

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

uint64_t hostgen_stream_key(uint64_t seed, int stream) {
  return mix64(seed ^ ((uint64_t)stream << 56));
}

static inline uint64_t counter(uint64_t layer, uint64_t b, uint64_t pos, uint64_t head,
                               uint64_t d) {
  return (layer << 52) | (b << 44) | (pos << 20) | (head << 12) | (d << 2);
}

/* Irwin-Hall draw of one element as fp32 (exact: integer sum times 2^-16). */
static inline float draw(uint64_t key, uint64_t base) {
  int64_t total = 0;
  for (uint64_t k = 0; k < 3; ++k) {
    const uint64_t h = mix64(key + (base | k) * GAMMA);
    total += (int64_t)(h & 0xFFFF) + (int64_t)((h >> 16) & 0xFFFF) +
             (int64_t)((h >> 32) & 0xFFFF) + (int64_t)(h >> 48);
  }
  return (float)(total - IRWIN_HALL_CENTER) * (1.0f / 65536.0f);
}

static inline float round_bf16(float x) {
  uint32_t bits;
  memcpy(&bits, &x, 4);
  bits = (bits + 0x7FFFu + ((bits >> 16) & 1u)) & 0xFFFF0000u;
  memcpy(&x, &bits, 4);
  return x;
}

typedef struct {
  uint64_t key;
  int layer, b, head, D, bf16;
  const int64_t* pos;   /* rows given by position list (normal) */
  int64_t pos0;         /* or a contiguous range (amax) */
  int n_heads;
  int64_t r0, r1;       /* rows [r0, r1) of this thread */
  float* out;
} job_t;

static void* normal_rows(void* arg) {
  job_t* j = (job_t*)arg;
  for (int64_t r = j->r0; r < j->r1; ++r) {
    float* o = j->out + r * j->D;
    for (int d = 0; d < j->D; ++d) {
      const float x = draw(j->key, counter(j->layer, j->b, j->pos[r], j->head, d));
      o[d] = j->bf16 ? round_bf16(x) : x;
    }
  }
  return 0;
}

/* out[n_pos][D] = draws of (stream, layer, b, pos[i], head, 0..D-1). */
void hostgen_normal(uint64_t seed, int stream, int layer, int b, const int64_t* pos, int64_t n_pos,
                    int head, int D, int bf16, float* out, int n_threads) {
  job_t jobs[64];
  pthread_t th[64];
  if (n_threads < 1) n_threads = 1;
  if (n_threads > 64) n_threads = 64;
  if (n_pos < 64 * n_threads) n_threads = 1;
  const uint64_t key = hostgen_stream_key(seed, stream);
  for (int t = 0; t < n_threads; ++t) {
    job_t* j = &jobs[t];
    memset(j, 0, sizeof(*j));
    j->key = key;
    j->layer = layer;
    j->b = b;
    j->head = head;
    j->D = D;
    j->bf16 = bf16;
    j->pos = pos;
    j->r0 = n_pos * t / n_threads;
    j->r1 = n_pos * (t + 1) / n_threads;
    j->out = out;
  }
  for (int t = 1; t < n_threads; ++t) pthread_create(&th[t], 0, normal_rows, &jobs[t]);
  normal_rows(&jobs[0]);
  for (int t = 1; t < n_threads; ++t) pthread_join(th[t], 0);
}

/* amax rows: row r = (b, p) with b = r / n_pos, p = pos0 + r % n_pos; every
 * head h < n_heads keeps its own maximum in out[h] (per-thread copies). */
typedef struct {
  job_t base;
  int64_t n_pos;
  float hmax[256];
} ajob_t;

static void* amax_rows(void* arg) {
  ajob_t* j = (ajob_t*)arg;
  for (int h = 0; h < j->base.n_heads; ++h) j->hmax[h] = 0.0f;
  for (int64_t r = j->base.r0; r < j->base.r1; ++r) {
    const int b = (int)(r / j->n_pos);
    const int64_t p = j->base.pos0 + r % j->n_pos;
    for (int h = 0; h < j->base.n_heads; ++h) {
      float m = j->hmax[h];
      for (int d = 0; d < j->base.D; ++d) {
        float x = draw(j->base.key, counter(j->base.layer, b, p, h, d));
        if (j->base.bf16) x = round_bf16(x);
        x = fabsf(x);
        if (x > m) m = x;
      }
      j->hmax[h] = m;
    }
  }
  return 0;
}

/* out[h] = max |x| over sequences b < batch, positions pos0 .. pos0+n_pos-1
 * and elements d < D of (stream, layer, b, pos, h, d), for h < n_heads. */
void hostgen_amax(uint64_t seed, int stream, int layer, int batch, int64_t pos0, int64_t n_pos,
                  int n_heads, int D, int bf16, float* out, int n_threads) {
  ajob_t jobs[64];
  pthread_t th[64];
  if (n_threads < 1) n_threads = 1;
  if (n_threads > 64) n_threads = 64;
  if (n_heads > 256) n_heads = 256;
  const int64_t rows = (int64_t)batch * n_pos;
  if (rows < 64 * n_threads) n_threads = 1;
  const uint64_t key = hostgen_stream_key(seed, stream);
  for (int t = 0; t < n_threads; ++t) {
    ajob_t* j = &jobs[t];
    memset(&j->base, 0, sizeof(j->base));
    j->base.key = key;
    j->base.layer = layer;
    j->base.D = D;
    j->base.bf16 = bf16;
    j->base.pos0 = pos0;
    j->base.n_heads = n_heads;
    j->base.r0 = rows * t / n_threads;
    j->base.r1 = rows * (t + 1) / n_threads;
    j->n_pos = n_pos;
  }
  for (int t = 1; t < n_threads; ++t) pthread_create(&th[t], 0, amax_rows, &jobs[t]);
  amax_rows(&jobs[0]);
  for (int t = 1; t < n_threads; ++t) pthread_join(th[t], 0);
  for (int h = 0; h < n_heads; ++h) {
    float m = 0.0f;
    for (int t = 0; t < n_threads; ++t)
      if (jobs[t].hmax[h] > m) m = jobs[t].hmax[h];
    out[h] = m;
  }
}
