/*
 * Seeded synthetic inputs for the fused W4A4 + low-rank linear layer.
 *
 * This module draws random numbers and rounds them to BF16. It holds none of
 * the layer's arithmetic (no quantizer, no matmul), so the oracle and the CUDA
 * path can both be fed from it without sharing any of the method.
 *
 * Generator (stated so that it can be re-implemented elsewhere):
 *   mix64(z)        the splitmix64 output function (Steele, Lea and Flood,
 *                   "Fast splittable pseudorandom number generators", 2014):
 *                   z ^= z>>30; z *= 0xBF58476D1CE4E5B9; z ^= z>>27;
 *                   z *= 0x94D049BB133111EB; z ^= z>>31.
 *   stream key      K = mix64(seed*16 + tensor_id)
 *   element state   s_e = mix64(K + (e+1)*GAMMA), GAMMA = 0x9E3779B97F4A7C15,
 *                   e = row*cols + col (row-major element index).
 *   element draws   the splitmix64 sequence started at s_e:
 *                   s += GAMMA; out = mix64(s).
 *   uniform (0,1)   ((out >> 11) + 0.5) * 2^-53.
 *   normal          Box-Muller, cosine branch: sqrt(-2 ln u1) * cos(2 pi u2).
 *   gamma(a >= 1)   Marsaglia and Tsang (2000) squeeze/rejection method.
 *   Student-t(nu)   Z / sqrt(2*Gamma(nu/2)/nu).
 *   BF16            double -> float (round to nearest even) -> bf16 (RNE).
 * Each element's value depends only on (seed, tensor_id, e), never on the
 * number of threads used to fill the tensor.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define SYNTH_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ULL;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBULL;
  z ^= z >> 31;
  return z;
}

static inline uint64_t next64(uint64_t* s) {
  *s += SYNTH_GAMMA;
  return mix64(*s);
}

static inline double u01(uint64_t* s) {
  return ((double)(next64(s) >> 11) + 0.5) * 0x1.0p-53;
}

static inline double draw_normal(uint64_t* s) {
  const double two_pi = 6.283185307179586476925286766559;
  double u1 = u01(s);
  double u2 = u01(s);
  return sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
}

static double draw_gamma(uint64_t* s, double a) {
  const double d = a - 1.0 / 3.0;
  const double c = 1.0 / sqrt(9.0 * d);
  for (;;) {
    double x = draw_normal(s);
    double v = 1.0 + c * x;
    if (v <= 0.0) continue;
    v = v * v * v;
    double u = u01(s);
    if (log(u) < 0.5 * x * x + d - d * v + d * log(v)) return d * v;
  }
}

static inline double draw_t(uint64_t* s, double nu) {
  double z = draw_normal(s);
  double g = draw_gamma(s, 0.5 * nu);
  return z / sqrt(2.0 * g / nu);
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return 0x7FC0;
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

uint64_t synth_stream_key(uint64_t seed, int tensor_id) {
  return mix64(seed * 16u + (uint64_t)tensor_id);
}

/* Distribution codes. */
enum { SYNTH_NORMAL = 0, SYNTH_STUDENT_T = 1 };

typedef struct {
  uint16_t* out;
  double* value_out; /* optional: the double before rounding (tests only) */
  int64_t row0, row1, cols;
  int dist;
  double p1, p2; /* normal: mean, sigma; t: nu, scale */
  uint64_t key;
  const double* colmul; /* per-column multiplier (outlier channels) or NULL */
} fill_job;

static void* fill_worker(void* arg) {
  fill_job* j = (fill_job*)arg;
  for (int64_t r = j->row0; r < j->row1; ++r) {
    for (int64_t c = 0; c < j->cols; ++c) {
      uint64_t e = (uint64_t)(r * j->cols + c);
      uint64_t st = mix64(j->key + (e + 1u) * SYNTH_GAMMA);
      double v;
      if (j->dist == SYNTH_NORMAL)
        v = j->p1 + j->p2 * draw_normal(&st);
      else
        v = j->p2 * draw_t(&st, j->p1);
      if (j->colmul) v *= j->colmul[c];
      if (j->value_out) j->value_out[r * j->cols + c] = v;
      j->out[r * j->cols + c] = f32_to_bf16_rne((float)v);
    }
  }
  return NULL;
}

/*
 * Fill a rows x cols row-major BF16 tensor. colmul (length cols) may be NULL.
 * Returns 0 on success.
 */
int synth_fill_bf16(uint16_t* out, double* value_out, int64_t rows, int64_t cols, int dist,
                    double p1, double p2, uint64_t seed, int tensor_id, const double* colmul,
                    int nthreads) {
  if (!out || rows < 0 || cols < 0) return 1;
  if (dist == SYNTH_STUDENT_T && !(p1 >= 2.0)) return 2; /* gamma(nu/2) needs nu/2 >= 1 */
  uint64_t key = synth_stream_key(seed, tensor_id);
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (rows < nthreads) nthreads = rows > 0 ? (int)rows : 1;
  pthread_t th[256];
  fill_job jobs[256];
  for (int t = 0; t < nthreads; ++t) {
    jobs[t].out = out;
    jobs[t].value_out = value_out;
    jobs[t].row0 = rows * t / nthreads;
    jobs[t].row1 = rows * (t + 1) / nthreads;
    jobs[t].cols = cols;
    jobs[t].dist = dist;
    jobs[t].p1 = p1;
    jobs[t].p2 = p2;
    jobs[t].key = key;
    jobs[t].colmul = colmul;
  }
  if (nthreads == 1) {
    fill_worker(&jobs[0]);
    return 0;
  }
  for (int t = 0; t < nthreads; ++t) pthread_create(&th[t], NULL, fill_worker, &jobs[t]);
  for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
  return 0;
}

/*
 * Seeded Fisher-Yates shuffle of 0..n-1 (Durstenfeld's in-place form), drawing
 * from the sequential splitmix64 stream that starts at the stream key. The
 * index j for position i is the high 64 bits of draw * (i+1).
 */
int synth_permutation(int32_t* perm, int64_t n, uint64_t seed, int tensor_id) {
  if (!perm || n < 0) return 1;
  for (int64_t i = 0; i < n; ++i) perm[i] = (int32_t)i;
  uint64_t st = synth_stream_key(seed, tensor_id);
  for (int64_t i = n - 1; i >= 1; --i) {
    uint64_t x = next64(&st);
    uint64_t j = (uint64_t)(((__uint128_t)x * (__uint128_t)(i + 1)) >> 64);
    int32_t t = perm[i];
    perm[i] = perm[j];
    perm[j] = t;
  }
  return 0;
}

/* Raw stream access for tests: the first `count` uniforms of element e. */
int synth_element_uniforms(double* out, int count, uint64_t seed, int tensor_id, uint64_t e) {
  uint64_t key = synth_stream_key(seed, tensor_id);
  uint64_t st = mix64(key + (e + 1u) * SYNTH_GAMMA);
  for (int i = 0; i < count; ++i) out[i] = u01(&st);
  return 0;
}

uint64_t synth_mix64(uint64_t z) { return mix64(z); }
