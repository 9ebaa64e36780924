/* Seeded synthetic inputs for the BitNet b1.58 W1.58A8 linear layer.
 *
 * Counter-based: every value is a pure function of (key, index), so any
 * slice of any tensor can be regenerated on its own, by the tests, the oracle
 * side and the bench alike. The generator is SplitMix64 (Steele, Lea and
 * Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014):
 * the 64-bit output of the finaliser applied to key + (index+1) * golden gamma.
 *
 * It holds none of the method's arithmetic: it only draws
 *   - ternary weights  {-1, 0, +1} with P(-1) = P(+1) = 0.3, P(0) = 0.4;
 *   - activations      N(0, 1) by Box-Muller in double precision, a fraction
 *                      p of entries multiplied by a factor (outliers), cast
 *                      to bf16 (round to nearest even via fp32);
 *   - uniform floats   for the per-tensor weight scale.
 * Work is split across host threads by index range; the result does not
 * depend on the thread count.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint64_t draw(uint64_t key, uint64_t index) {
  return mix64(key + (index + 1) * 0x9E3779B97F4A7C15ULL);
}

/* uniform double in [0, 1) with 53 random bits */
static inline double unif(uint64_t key, uint64_t index) {
  return (double)(draw(key, index) >> 11) * (1.0 / 9007199254740992.0);
}

uint64_t synth_key(uint64_t a, uint64_t b, uint64_t c, uint64_t d) {
  uint64_t k = mix64(a + 0x632BE59BD9B4E019ULL);
  k = mix64(k ^ (b + 0x8CB92BA72F3D8DD7ULL));
  k = mix64(k ^ (c + 0xD6E8FEB86659FD93ULL));
  k = mix64(k ^ (d + 0xA0761D6478BD642FULL));
  return k;
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  uint32_t lower = u & 0xFFFFu, upper = u >> 16;
  if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1;
  return (uint16_t)upper;
}

typedef struct {
  int kind;
  uint64_t key;
  int64_t start, n;
  double p, mult, lo, hi;
  void* out;
} job_t;

static void run_range(const job_t* j) {
  if (j->kind == 0) {
    int8_t* o = (int8_t*)j->out;
    for (int64_t i = 0; i < j->n; ++i) {
      double u = unif(j->key, (uint64_t)(j->start + i));
      o[i] = (int8_t)(u < 0.3 ? -1 : (u < 0.7 ? 0 : 1));
    }
  } else if (j->kind == 1) {
    uint16_t* o = (uint16_t*)j->out;
    const uint64_t okey = j->key ^ 0x5DEECE66DA5A5A5AULL;
    for (int64_t i = 0; i < j->n; ++i) {
      const uint64_t idx = (uint64_t)(j->start + i);
      double u1 = unif(j->key, 2 * idx);
      double u2 = unif(j->key, 2 * idx + 1);
      double z = sqrt(-2.0 * log(1.0 - u1)) * cos(6.283185307179586 * u2);
      if (j->p > 0.0 && unif(okey, idx) < j->p) z *= j->mult;
      o[i] = f32_to_bf16_rne((float)z);
    }
  } else {
    float* o = (float*)j->out;
    for (int64_t i = 0; i < j->n; ++i) {
      double u = unif(j->key, (uint64_t)(j->start + i));
      o[i] = (float)(j->lo + (j->hi - j->lo) * u);
    }
  }
}

static void* thread_main(void* arg) {
  run_range((const job_t*)arg);
  return 0;
}

static void run(job_t base, int nthreads, size_t elem) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (base.n < 65536 || nthreads == 1) {
    run_range(&base);
    return;
  }
  pthread_t th[256];
  int created[256];
  job_t jobs[256];
  int64_t per = (base.n + nthreads - 1) / nthreads;
  for (int t = 0; t < nthreads; ++t) {
    created[t] = 0;
    int64_t a = t * per, b = a + per < base.n ? a + per : base.n;
    if (a >= b) continue;
    jobs[t] = base;
    jobs[t].start = base.start + a;
    jobs[t].n = b - a;
    jobs[t].out = (char*)base.out + (size_t)a * elem;
    if (pthread_create(&th[t], 0, thread_main, &jobs[t]) == 0) {
      created[t] = 1;
    } else {
      run_range(&jobs[t]);
    }
  }
  for (int t = 0; t < nthreads; ++t)
    if (created[t]) pthread_join(th[t], 0);
}

/* n ternary weights of tensor `key`, elements [start, start + n). */
void synth_ternary(uint64_t key, int64_t start, int64_t n, int8_t* out,
                   int nthreads) {
  job_t j = {0, key, start, n, 0, 0, 0, 0, out};
  run(j, nthreads, 1);
}

/* n bf16 activations (raw bits) of tensor `key`, elements [start, start+n). */
void synth_act_bf16(uint64_t key, int64_t start, int64_t n, double outlier_p,
                    double outlier_mult, uint16_t* out, int nthreads) {
  job_t j = {1, key, start, n, outlier_p, outlier_mult, 0, 0, out};
  run(j, nthreads, 2);
}

/* n uniform fp32 values in [lo, hi) of tensor `key`. */
void synth_uniform_f32(uint64_t key, int64_t start, int64_t n, double lo,
                       double hi, float* out, int nthreads) {
  job_t j = {2, key, start, n, 0, 0, lo, hi, out};
  run(j, nthreads, 4);
}
