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
#include <math.h>

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

/*
 * FP8 (e4m3) weights with one power-of-two scale per 128 x 128 block.
 * For element i of a [rows, cols] matrix (flat row-major index i, cols a
 * multiple of 128): block b = (r / 128) * (cols / 128) + c / 128 has the
 * exponent e_b = e0 + (hash(seed, tid_scale, b) & 3); the code is the
 * e4m3 value nearest (ties to even) to v_i * 2^-e_b, v_i the approximately
 * normal value above (before any rounding), saturated to +-448. The scale
 * byte of block b is e_b + 127 (UE8M0: value 2^(byte - 127)).
 * e4m3: 1 sign, 4 exponent (bias 7), 3 mantissa bits; no infinities;
 * 0x7F / 0xFF are NaN and never produced; largest finite 0x7E = 448.
 */
static inline uint8_t e4m3_rne(double x) {
  uint8_t sign = (x < 0.0) ? 0x80 : 0x00;
  double a = x < 0.0 ? -x : x;
  if (a >= 464.0) return (uint8_t)(sign | 0x7E);            /* saturate (never reached here) */
  if (a < 0.015625) {                                         /* below 2^-6: subnormal steps of 2^-9 */
    int m = (int)rint(a * 512.0);                             /* exact scaling, ties to even */
    return (uint8_t)(sign | m);                               /* m == 8 is the smallest normal, 0x08 */
  }
  int e;
  double f = frexp(a, &e);                                    /* a = f 2^e, f in [0.5, 1) */
  e -= 1;                                                     /* a = (2 f) 2^e, 2 f in [1, 2) */
  int mant = (int)rint((ldexp(f, 1) - 1.0) * 8.0);
  if (mant == 8) { mant = 0; e += 1; }
  if (e > 8 || (e == 8 && mant > 6)) return (uint8_t)(sign | 0x7E);
  return (uint8_t)(sign | ((e + 7) << 3) | mant);
}

static inline int block_exp(uint32_t seed, uint32_t tid_scale, uint64_t block, int e0) {
  return e0 + (int)(splitmix64_out(gen_counter(seed, tid_scale, block)) & 3u);
}

typedef struct {
  uint32_t seed, tid, tid_scale;
  int e0;
  uint64_t cols, offset, begin, end;
  double factor;
  uint8_t* out;
} fp8_job_t;

static void* run_fp8_job(void* p) {
  fp8_job_t* j = (fp8_job_t*)p;
  const uint64_t bcols = j->cols / 128;
  for (uint64_t i = j->begin; i < j->end; ++i) {
    const uint64_t g = j->offset + i, r = g / j->cols, c = g % j->cols;
    const int e = block_exp(j->seed, j->tid_scale, (r / 128) * bcols + c / 128, j->e0);
    const double v = irwin_hall4(splitmix64_out(gen_counter(j->seed, j->tid, g)), j->factor);
    j->out[i] = e4m3_rne(ldexp(v, -e));
  }
  return 0;
}

/* e4m3 codes of elements [offset, offset + n) of a [rows, cols] matrix. */
void gen_fp8(uint32_t seed, uint32_t tid, uint32_t tid_scale, int e0, uint64_t cols, uint64_t offset, uint64_t n,
             double factor, uint8_t* out, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (n < (uint64_t)nthreads * 65536ull) nthreads = (int)(n / 65536ull) + 1;
  fp8_job_t jobs[256];
  pthread_t th[256];
  uint64_t chunk = (n + nthreads - 1) / nthreads;
  for (int t = 0; t < nthreads; ++t) {
    uint64_t b0 = chunk * t, b1 = b0 + chunk;
    if (b0 > n) b0 = n;
    if (b1 > n) b1 = n;
    jobs[t] = (fp8_job_t){seed, tid, tid_scale, e0, cols, offset, b0, b1, factor, out};
  }
  for (int t = 1; t < nthreads; ++t) pthread_create(&th[t], 0, run_fp8_job, &jobs[t]);
  run_fp8_job(&jobs[0]);
  for (int t = 1; t < nthreads; ++t) pthread_join(th[t], 0);
}

/* UE8M0 scale bytes of blocks [offset, offset + n). */
void gen_fp8_scales(uint32_t seed, uint32_t tid_scale, int e0, uint64_t offset, uint64_t n, uint8_t* out) {
  for (uint64_t i = 0; i < n; ++i) out[i] = (uint8_t)(block_exp(seed, tid_scale, offset + i, e0) + 127);
}

/* Raw 64-bit hashes (used by the tests to pin the definition, and for seeded permutations). */
void gen_hash(uint32_t seed, uint32_t tid, uint64_t offset, uint64_t n, uint64_t* out) {
  for (uint64_t i = 0; i < n; ++i) out[i] = splitmix64_out(gen_counter(seed, tid, offset + i));
}
