/*
 * mk_inputs.c -- seeded synthetic inputs for the decode megakernel and its oracle.
 *
 * This module is the ONLY code shared by the CPU oracle and the CUDA path, and it
 * holds none of the decoder's arithmetic: it turns (seed, tensor_id, index) into
 * random bits, normal deviates, rounded bf16/fp16 values and token ids.
 *
 * Generator definition (fixed here, used by every test, the bench and the oracle):
 *   - SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
 *     generators", OOPSLA 2014): state += 0x9E3779B97F4A7C15; z = state;
 *     z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9; z = (z ^ (z >> 27)) * 0x94D049BB133111EB;
 *     out = z ^ (z >> 31).  Because the state advances by a constant, output k of a
 *     stream is mix(base + (k + 1) * gamma): random access, so generation is
 *     counter-based and any thread count gives the same bytes.
 *   - Stream base for (seed, tensor_id): mix(mix(seed) ^ (tensor_id * 0xD1B54A32D192ED03)).
 *   - Normal deviates by Box-Muller (1958) in double: for pair i, u1 = 1 - (o(2i) >> 11) 2^-53
 *     in (0, 1], u2 = (o(2i+1) >> 11) 2^-53; rad = sqrt(-2 ln u1); element 2i gets
 *     rad cos(2 pi u2), element 2i+1 gets rad sin(2 pi u2).
 *   - A scaled deviate sigma * z is rounded to fp32 (round to nearest even), then to
 *     bf16 (RNE) or fp16 (RNE, via _Float16).
 *   - Token ids: o(k) mod vocab with rejection of the biased top range; token i tries
 *     k = 4i, 4i+1, 4i+2, 4i+3 in turn (a rejection has probability < 2^-46 per try for
 *     vocab < 2^18, so the fourth try is never reached in practice; it falls back to
 *     plain modulo if it were).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

/* SplitMix64 as published: advance the state, then mix it. */
uint64_t mki_splitmix64_next(uint64_t* state) {
  *state += GAMMA;
  return mix64(*state);
}

uint64_t mki_stream_base(uint64_t seed, uint64_t tensor_id) {
  return mix64(mix64(seed) ^ (tensor_id * 0xD1B54A32D192ED03ULL));
}

/* Output k (0-based) of the SplitMix64 stream that starts from state `base`. */
uint64_t mki_stream_u64(uint64_t base, uint64_t k) { return mix64(base + (k + 1) * GAMMA); }

static inline void normal_pair(uint64_t base, uint64_t pair, double* z0, double* z1) {
  const double two_m53 = 1.0 / 9007199254740992.0;
  double u1 = 1.0 - (double)(mki_stream_u64(base, 2 * pair) >> 11) * two_m53;
  double u2 = (double)(mki_stream_u64(base, 2 * pair + 1) >> 11) * two_m53;
  double rad = sqrt(-2.0 * log(u1));
  double ang = 6.283185307179586476925286766559 * u2;
  *z0 = rad * cos(ang);
  *z1 = rad * sin(ang);
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7f800000u) == 0x7f800000u) return (uint16_t)((u >> 16) | ((u & 0xffff) ? 0x40 : 0));
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

static inline uint16_t f32_to_f16_rne(float f) {
  _Float16 h = (_Float16)f;
  uint16_t r;
  memcpy(&r, &h, 2);
  return r;
}

enum { KIND_BF16 = 0, KIND_F16 = 1, KIND_F32 = 2 };

typedef struct {
  uint64_t base, lo, hi; /* element range [lo, hi) */
  double sigma, mean;
  int kind;
  void* out;
} job_t;

static void fill_range(const job_t* j) {
  uint64_t i = j->lo;
  while (i < j->hi) {
    double z[2];
    uint64_t pair = i >> 1;
    normal_pair(j->base, pair, &z[0], &z[1]);
    for (int s = (int)(i & 1); s < 2 && i < j->hi; ++s, ++i) {
      float v = (float)(j->mean + j->sigma * z[s]);
      if (j->kind == KIND_BF16) ((uint16_t*)j->out)[i] = f32_to_bf16_rne(v);
      else if (j->kind == KIND_F16) ((uint16_t*)j->out)[i] = f32_to_f16_rne(v);
      else ((float*)j->out)[i] = v;
    }
  }
}

static void* fill_thread(void* p) {
  fill_range((const job_t*)p);
  return NULL;
}

static void fill_normal(uint64_t seed, uint64_t tensor_id, uint64_t n, double mean, double sigma, int kind,
                        void* out, int nthreads) {
  uint64_t base = mki_stream_base(seed, tensor_id);
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (n < (1u << 20)) nthreads = 1;
  job_t jobs[256];
  pthread_t th[256];
  uint64_t per = (n + (uint64_t)nthreads - 1) / (uint64_t)nthreads;
  per = (per + 1) & ~1ULL; /* even split points keep pairs on one thread (cosmetic) */
  int joined[256] = {0};
  for (int t = 0; t < nthreads; ++t) {
    uint64_t lo = (uint64_t)t * per, hi = lo + per;
    if (lo >= n) break;
    if (hi > n) hi = n;
    jobs[t] = (job_t){base, lo, hi, sigma, mean, kind, out};
    if (nthreads == 1 || pthread_create(&th[t], NULL, fill_thread, &jobs[t]) != 0) {
      fill_range(&jobs[t]); /* inline when single-threaded or when a thread cannot start */
      continue;
    }
    joined[t] = 1;
  }
  for (int t = 0; t < nthreads; ++t)
    if (joined[t]) pthread_join(th[t], NULL);
}

/* bf16 bits of round(mean + sigma * N(0,1)) for elements [0, n) of stream (seed, tensor_id). */
void mki_normal_bf16(uint64_t seed, uint64_t tensor_id, uint64_t n, double mean, double sigma, uint16_t* out,
                     int nthreads) {
  fill_normal(seed, tensor_id, n, mean, sigma, KIND_BF16, out, nthreads);
}

/* fp16 bits, same stream definition. */
void mki_normal_f16(uint64_t seed, uint64_t tensor_id, uint64_t n, double mean, double sigma, uint16_t* out,
                    int nthreads) {
  fill_normal(seed, tensor_id, n, mean, sigma, KIND_F16, out, nthreads);
}

/* fp32 values, same stream definition. */
void mki_normal_f32(uint64_t seed, uint64_t tensor_id, uint64_t n, double mean, double sigma, float* out,
                    int nthreads) {
  fill_normal(seed, tensor_id, n, mean, sigma, KIND_F32, out, nthreads);
}

/* Uniform token ids in [0, vocab). */
void mki_tokens(uint64_t seed, uint64_t tensor_id, uint64_t n, uint32_t vocab, int32_t* out) {
  uint64_t base = mki_stream_base(seed, tensor_id);
  uint64_t v = vocab ? vocab : 1;
  /* largest multiple of v that fits in 2^64: accept r < limit */
  uint64_t limit = (uint64_t)0 - ((uint64_t)0 - v) % v; /* 2^64 - (2^64 mod v), 0 means all accepted */
  for (uint64_t i = 0; i < n; ++i) {
    uint64_t r = 0;
    int ok = 0;
    for (int t = 0; t < 4 && !ok; ++t) {
      r = mki_stream_u64(base, 4 * i + (uint64_t)t);
      ok = (limit == 0) || (r < limit);
    }
    out[i] = (int32_t)(r % v);
  }
}

/* Fill `n` bf16 values with a constant (norm gains are exactly 1). */
void mki_const_bf16(uint64_t n, float value, uint16_t* out) {
  uint16_t b = f32_to_bf16_rne(value);
  for (uint64_t i = 0; i < n; ++i) out[i] = b;
}
