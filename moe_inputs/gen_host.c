/*
 * Seeded synthetic inputs, host side.
 *
 * Shared test/bench infrastructure: it holds none of the layer's arithmetic.
 * Every value is a pure function of (seed, tensor id, flat index), so any
 * slice can be regenerated independently, in any order, on any thread.
 *
 * Definition (identical in gen_device.cu, checked bit for bit by the tests):
 *   c  = seed << 56 | tensor_id << 48 | index            (index < 2^48)
 *   h  = SplitMix64 output function applied to c
 *        (Steele, Lea, Flood, "Fast splittable pseudorandom number
 *        generators", OOPSLA 2014; constants as published by Vigna)
 *   approximately normal value (Irwin-Hall sum of four 16-bit uniforms):
 *        s = sum of the four 16-bit fields of h, in [0, 262140]
 *        v = (double)(s - 131070) * factor
 *        factor = std / sqrt(1431655765)  (computed by the caller in fp64;
 *        1431655765 = 4 * (65536^2 - 1) / 12 is the variance of s)
 *   uniform value in [lo, hi):
 *        u = (h >> 11) * 2^-53 ;  v = lo + (hi - lo) * u
 *   stored dtype: fp64 -> fp32 round-to-nearest-even, then for bf16 a second
 *        round-to-nearest-even fp32 -> bf16 on the bit pattern.
 * Only integer operations and single IEEE multiplies/adds are used, so the
 * host and the device produce the same bits (no FMA contraction: build with
 * -ffp-contract=off).
 */
#include <stdint.h>
#include <string.h>
#include <pthread.h>

static inline uint64_t splitmix64_out(uint64_t z) {
  z += 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

static inline uint64_t gen_counter(uint32_t seed, uint32_t tid, uint64_t index) {
  return ((uint64_t)(seed & 0xFF) << 56) | ((uint64_t)(tid & 0xFF) << 48) |
         (index & 0xFFFFFFFFFFFFull);
}

static inline double irwin_hall4(uint64_t h, double factor) {
  int64_t s = (int64_t)(h & 0xFFFF) + (int64_t)((h >> 16) & 0xFFFF) +
              (int64_t)((h >> 32) & 0xFFFF) + (int64_t)(h >> 48);
  return (double)(s - 131070) * factor;
}

static inline double uniform_lohi(uint64_t h, double lo, double hi) {
  double u = (double)(h >> 11) * (1.0 / 9007199254740992.0); /* 2^-53, exact */
  double w = hi - lo;
  double p = w * u;
  return lo + p;
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40u);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

typedef struct {
  uint32_t seed, tid, kind, out_bf16;
  uint64_t offset, begin, end;
  double a, b;
  void* out;
} job_t;

static void* run_job(void* p) {
  job_t* j = (job_t*)p;
  for (uint64_t i = j->begin; i < j->end; ++i) {
    uint64_t h = splitmix64_out(gen_counter(j->seed, j->tid, j->offset + i));
    double v = j->kind == 0 ? irwin_hall4(h, j->a) : uniform_lohi(h, j->a, j->b);
    float f = (float)v;
    if (j->out_bf16) ((uint16_t*)j->out)[i] = f32_to_bf16_rne(f);
    else ((float*)j->out)[i] = f;
  }
  return 0;
}

static void run(uint32_t seed, uint32_t tid, uint32_t kind, uint32_t out_bf16, uint64_t offset,
                uint64_t n, double a, double b, void* out, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (n < (uint64_t)nthreads * 65536ull) nthreads = (int)(n / 65536ull) + 1;
  job_t jobs[256];
  pthread_t th[256];
  uint64_t chunk = (n + nthreads - 1) / nthreads;
  for (int t = 0; t < nthreads; ++t) {
    uint64_t b0 = chunk * t, b1 = b0 + chunk;
    if (b0 > n) b0 = n;
    if (b1 > n) b1 = n;
    jobs[t] = (job_t){seed, tid, kind, out_bf16, offset, b0, b1, a, b, out};
  }
  for (int t = 1; t < nthreads; ++t) pthread_create(&th[t], 0, run_job, &jobs[t]);
  run_job(&jobs[0]);
  for (int t = 1; t < nthreads; ++t) pthread_join(th[t], 0);
}

/* Approximately normal values with standard deviation std = factor * sqrt(1431655765). */
void gen_normal(uint32_t seed, uint32_t tid, uint64_t offset, uint64_t n, double factor,
                int out_bf16, void* out, int nthreads) {
  run(seed, tid, 0, (uint32_t)out_bf16, offset, n, factor, 0.0, out, nthreads);
}

/* Uniform values in [lo, hi). */
void gen_uniform(uint32_t seed, uint32_t tid, uint64_t offset, uint64_t n, double lo, double hi,
                 int out_bf16, void* out, int nthreads) {
  run(seed, tid, 1, (uint32_t)out_bf16, offset, n, lo, hi, out, nthreads);
}

/* Raw 64-bit hashes (used by the tests to pin the definition, and for seeded permutations). */
void gen_hash(uint32_t seed, uint32_t tid, uint64_t offset, uint64_t n, uint64_t* out) {
  for (uint64_t i = 0; i < n; ++i) out[i] = splitmix64_out(gen_counter(seed, tid, offset + i));
}
