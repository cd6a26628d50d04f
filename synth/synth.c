/*
 * Seeded synthetic input generator shared by the CPU oracle and the GPU path.
 *
 * This file holds none of the decode step's arithmetic: it only turns
 * (seed, tensor id, element index) into numbers.  Both sides of every parity
 * test receive the buffers it fills, so neither side draws random numbers.
 *
 * Generator definitions (all public):
 *   - SplitMix64 (G. Steele, D. Lea, C. Flood, "Fast splittable pseudorandom
 *     number generators", OOPSLA 2014; constants as in S. Vigna's reference
 *     code), used as a counter-based stream: element i of stream `key` is
 *     mix(key + (i + 1) * 0x9E3779B97F4A7C15).
 *   - stream key for (seed, tensor_id) = mix(seed ^ 0xD1B54A32D192ED03 +
 *     (tensor_id + 1) * 0x9E3779B97F4A7C15), i.e. element `tensor_id` of a
 *     stream keyed by the scrambled seed.
 *   - uniform double u = (z >> 11) * 2^-53 in [0, 1).
 *   - standard normal pairs by the Box-Muller transform (Box & Muller 1958):
 *     for pair k, u1 = U(2k), u2 = U(2k+1), r = sqrt(-2 ln(1 - u1)),
 *     n(2k) = r cos(2 pi u2), n(2k+1) = r sin(2 pi u2), in double.
 *   - a normal value mean + std * n is rounded double -> float (IEEE RNE) ->
 *     bfloat16 (round to nearest even on the upper 16 bits).
 *   - integers uniform in [lo, hi]: lo + floor(((z >> 11) * (hi - lo + 1)) / 2^53)
 *     computed exactly in 128-bit integer arithmetic.
 */
#include <math.h>
#include <pthread.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>

static inline uint64_t sm64_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint64_t sm64_at(uint64_t key, uint64_t i) {
  return sm64_mix(key + (i + 1ULL) * 0x9E3779B97F4A7C15ULL);
}

uint64_t synth_stream_key(uint64_t seed, uint64_t tensor_id) {
  return sm64_at(seed ^ 0xD1B54A32D192ED03ULL, tensor_id);
}

uint64_t synth_u64_at(uint64_t seed, uint64_t tensor_id, uint64_t i) {
  return sm64_at(synth_stream_key(seed, tensor_id), i);
}

static inline double u01(uint64_t z) { return (double)(z >> 11) * 0x1.0p-53; }

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u); /* NaN */
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7fffu + lsb;
  return (uint16_t)(u >> 16);
}

/* Standard normal for element index j of stream `key`. */
static inline double normal_at(uint64_t key, uint64_t j) {
  const double two_pi = 6.283185307179586476925286766559;
  uint64_t k = j >> 1;
  double u1 = u01(sm64_at(key, 2 * k));
  double u2 = u01(sm64_at(key, 2 * k + 1));
  double r = sqrt(-2.0 * log(1.0 - u1));
  return (j & 1) ? r * sin(two_pi * u2) : r * cos(two_pi * u2);
}

typedef struct {
  uint16_t *out;
  size_t begin, end;
  uint64_t key, offset;
  double mean, std;
} normal_job;

static void *normal_worker(void *arg) {
  normal_job *jb = (normal_job *)arg;
  for (size_t i = jb->begin; i < jb->end; ++i) {
    double v = jb->mean + jb->std * normal_at(jb->key, jb->offset + i);
    jb->out[i] = f32_to_bf16_rne((float)v);
  }
  return NULL;
}

/*
 * Fill out[0..n) with elements [offset, offset + n) of the bf16 normal stream
 * (seed, tensor_id) with the given mean and standard deviation.
 * nthreads <= 1 runs on the calling thread.  Returns 0 on success.
 */
int synth_normal_bf16(uint16_t *out, size_t n, uint64_t seed, uint64_t tensor_id,
                      uint64_t offset, double mean, double std, int nthreads) {
  uint64_t key = synth_stream_key(seed, tensor_id);
  if (nthreads < 1) nthreads = 1;
  if ((size_t)nthreads > n / 65536 + 1) nthreads = (int)(n / 65536 + 1);
  if (nthreads > 256) nthreads = 256;
  normal_job jobs[256];
  pthread_t th[256];
  size_t per = (n + (size_t)nthreads - 1) / (size_t)nthreads;
  for (int t = 0; t < nthreads; ++t) {
    size_t b = (size_t)t * per, e = b + per;
    if (b > n) b = n;
    if (e > n) e = n;
    jobs[t] = (normal_job){out, b, e, key, offset, mean, std};
  }
  if (nthreads == 1) {
    normal_worker(&jobs[0]);
    return 0;
  }
  int started = 0;
  for (int t = 0; t < nthreads; ++t) {
    if (pthread_create(&th[t], NULL, normal_worker, &jobs[t]) != 0) break;
    ++started;
  }
  for (int t = started; t < nthreads; ++t) normal_worker(&jobs[t]);
  for (int t = 0; t < started; ++t) pthread_join(th[t], NULL);
  return 0;
}

/* Fill out[0..n) with integers uniform in [lo, hi] from stream (seed, tensor_id). */
int synth_uniform_int(int32_t *out, size_t n, uint64_t seed, uint64_t tensor_id,
                      uint64_t offset, int64_t lo, int64_t hi) {
  if (hi < lo) return -1;
  uint64_t key = synth_stream_key(seed, tensor_id);
  unsigned __int128 span = (unsigned __int128)(uint64_t)(hi - lo) + 1;
  for (size_t i = 0; i < n; ++i) {
    uint64_t z = sm64_at(key, offset + i) >> 11;
    unsigned __int128 v = ((unsigned __int128)z * span) >> 53;
    out[i] = (int32_t)(lo + (int64_t)v);
  }
  return 0;
}
