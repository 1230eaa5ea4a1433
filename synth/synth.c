/*
 * Seeded synthetic input generator shared by the tests, the benchmark and the
 * oracle runs.  It draws numbers and nothing else: no step of the MoE layer
 * lives here.
 *
 * Every element is a pure function of (seed, tag, index), so any slice of any
 * tensor can be regenerated independently and in parallel:
 *
 *   key      = splitmix64 output #tag of the sequence seeded with `seed`
 *   word(i)  = splitmix64 output #i  of the sequence seeded with `key`
 *
 * splitmix64 is the generator of Steele, Lea and Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014: the state advances by the
 * golden-ratio increment 0x9E3779B97F4A7C15 and each output is passed through
 * the published xor-shift/multiply finaliser.  Output #i (0-based) of the
 * sequence seeded with s is mix(s + (i + 1) * increment).
 *
 * Normals use the Box-Muller transform on two 53-bit uniforms taken from
 * words 2i and 2i+1.  bf16 outputs are the fp32 value rounded to nearest-even
 * on its top 16 bits.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

static inline uint64_t sm_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint64_t sm_word(uint64_t key, uint64_t i) {
  return sm_mix(key + (i + 1ULL) * 0x9E3779B97F4A7C15ULL);
}

uint64_t synth_stream_key(uint64_t seed, uint64_t tag) { return sm_word(seed, tag); }

uint64_t synth_word(uint64_t seed, uint64_t tag, uint64_t i) {
  return sm_word(sm_word(seed, tag), i);
}

static inline double gen_normal(uint64_t key, uint64_t i) {
  const double two_m53 = 1.0 / 9007199254740992.0;
  /* u1 in (0, 1): never exactly 0, so log() is finite */
  double u1 = ((double)(sm_word(key, 2 * i) >> 11) + 0.5) * two_m53;
  double u2 = (double)(sm_word(key, 2 * i + 1) >> 11) * two_m53;
  return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925 * u2);
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

enum { OUT_F32 = 0, OUT_BF16 = 1, OUT_INT = 2 };

typedef struct {
  uint64_t key;
  double mean, std;
  int32_t range;
  int64_t begin, end; /* element range [begin, end) */
  int64_t first;      /* global index of element 0 of out */
  int kind;
  void *out;
} job_t;

static void *run_job(void *p) {
  job_t *j = (job_t *)p;
  for (int64_t i = j->begin; i < j->end; ++i) {
    uint64_t gi = (uint64_t)(j->first + i);
    if (j->kind == OUT_INT) {
      ((int32_t *)j->out)[i] = (int32_t)(sm_word(j->key, gi) % (uint64_t)j->range);
    } else {
      float v = (float)(j->mean + j->std * gen_normal(j->key, gi));
      if (j->kind == OUT_F32)
        ((float *)j->out)[i] = v;
      else
        ((uint16_t *)j->out)[i] = f32_to_bf16_rne(v);
    }
  }
  return NULL;
}

static void run_parallel(job_t proto, int64_t n, int threads) {
  if (threads < 1) threads = 1;
  if (threads > 256) threads = 256;
  if (n < 65536) threads = 1;
  pthread_t tid[256];
  job_t jobs[256];
  int64_t chunk = (n + threads - 1) / threads;
  int started = 0;
  for (int t = 0; t < threads; ++t) {
    jobs[t] = proto;
    jobs[t].begin = (int64_t)t * chunk;
    jobs[t].end = jobs[t].begin + chunk < n ? jobs[t].begin + chunk : n;
    if (jobs[t].begin >= jobs[t].end) break;
    if (threads == 1) {
      run_job(&jobs[t]);
    } else if (pthread_create(&tid[t], NULL, run_job, &jobs[t]) != 0) {
      run_job(&jobs[t]);
      tid[t] = 0;
    }
    started = t + 1;
  }
  if (threads > 1)
    for (int t = 0; t < started; ++t)
      if (tid[t]) pthread_join(tid[t], NULL);
}

/* out[i] = mean + std * N(0,1) draw #(first + i) of stream (seed, tag), fp32 */
void synth_normal_f32(uint64_t seed, uint64_t tag, double mean, double std, int64_t first,
                      int64_t n, float *out, int threads) {
  job_t p = {synth_stream_key(seed, tag), mean, std, 0, 0, 0, first, OUT_F32, out};
  run_parallel(p, n, threads);
}

/* same draws as synth_normal_f32, each rounded to bf16 (bit patterns) */
void synth_normal_bf16(uint64_t seed, uint64_t tag, double mean, double std, int64_t first,
                       int64_t n, uint16_t *out, int threads) {
  job_t p = {synth_stream_key(seed, tag), mean, std, 0, 0, 0, first, OUT_BF16, out};
  run_parallel(p, n, threads);
}

/* out[i] = word #(first + i) of stream (seed, tag) modulo range, range >= 1 */
void synth_uniform_int(uint64_t seed, uint64_t tag, int32_t range, int64_t first, int64_t n,
                       int32_t *out, int threads) {
  job_t p = {synth_stream_key(seed, tag), 0.0, 0.0, range, 0, 0, first, OUT_INT, out};
  run_parallel(p, n, threads);
}
