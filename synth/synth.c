/*
 * Seeded synthetic inputs for the DyT workloads.
 *
 * This module draws random numbers and encodes them in a storage dtype. It
 * holds none of the DyT arithmetic: both the CPU oracle and the CUDA path are
 * fed the bytes it writes, so they see identical inputs.
 *
 * Generator: Philox4x64-10, the counter-based generator of Salmon, Moraes,
 * Dror and Shaw, "Parallel random numbers: as easy as 1, 2, 3" (SC'11),
 * followed by the Box-Muller transform (Box & Muller, 1958).
 *
 *   key     = (seed, stream)      one stream per tensor (x, dy, gamma, beta)
 *   counter = (block, attempt, 0, 0)
 *
 * One Philox block gives four 64-bit words w0..w3. Words (w0, w1) make the
 * first normal pair and (w2, w3) the second: u1 = (hi53(w_even) + 1) * 2^-53
 * lies in (0, 1], u2 = hi53(w_odd) * 2^-53 lies in [0, 1), and
 *   z_cos = sqrt(-2 ln u1) cos(2 pi u2),  z_sin = sqrt(-2 ln u1) sin(2 pi u2).
 * Element i takes lane i mod 4 of block i / 4 (lanes: cos0, sin0, cos1, sin1).
 * The value mean + std * z is rounded to binary32 (ties to even) and then to
 * the storage dtype (ties to even). With `nonzero`, an element whose stored
 * value is +-0 is drawn again from attempt 1, 2, ... of the same block.
 *
 * Element values depend only on (seed, stream, i): the thread count changes
 * nothing.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

enum { SYNTH_F32 = 0, SYNTH_BF16 = 1, SYNTH_F16 = 2, SYNTH_F64 = 3 };

/* Philox4x64 multipliers and Weyl key increments (SC'11, Table 2). */
#define PHILOX_M0 0xD2E7470EE14C6C93ULL
#define PHILOX_M1 0xCA5A826395121157ULL
#define PHILOX_W0 0x9E3779B97F4A7C15ULL
#define PHILOX_W1 0xBB67AE8584CAA73BULL

static inline void mulhilo64(uint64_t a, uint64_t b, uint64_t *hi, uint64_t *lo) {
  unsigned __int128 p = (unsigned __int128)a * (unsigned __int128)b;
  *hi = (uint64_t)(p >> 64);
  *lo = (uint64_t)p;
}

void synth_philox4x64_10(const uint64_t ctr_in[4], const uint64_t key_in[2], uint64_t out[4]) {
  uint64_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
  uint64_t k0 = key_in[0], k1 = key_in[1];
  for (int round = 0; round < 10; ++round) {
    uint64_t hi0, lo0, hi1, lo1;
    mulhilo64(PHILOX_M0, c0, &hi0, &lo0);
    mulhilo64(PHILOX_M1, c2, &hi1, &lo1);
    uint64_t n0 = hi1 ^ c1 ^ k0;
    uint64_t n1 = lo1;
    uint64_t n2 = hi0 ^ c3 ^ k1;
    uint64_t n3 = lo0;
    c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    k0 += PHILOX_W0;
    k1 += PHILOX_W1;
  }
  out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

static double lane_normal(uint64_t seed, uint64_t stream, uint64_t block, uint64_t attempt, int lane) {
  const uint64_t ctr[4] = {block, attempt, 0, 0};
  const uint64_t key[2] = {seed, stream};
  uint64_t w[4];
  synth_philox4x64_10(ctr, key, w);
  const int pair = lane >> 1;
  const double u1 = (double)((w[2 * pair] >> 11) + 1) * 0x1.0p-53;
  const double u2 = (double)(w[2 * pair + 1] >> 11) * 0x1.0p-53;
  const double rad = sqrt(-2.0 * log(u1));
  const double ang = 6.283185307179586476925286766559 * u2;
  return (lane & 1) ? rad * sin(ang) : rad * cos(ang);
}

/* binary32 -> bfloat16 bits, ties to even; NaN stays a quiet NaN. */
static uint16_t f32_to_bf16_bits(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x0040u);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

static int store_one(void *out, int64_t i, int dtype, double v) {
  const float f = (float)v;
  switch (dtype) {
    case SYNTH_F32: ((float *)out)[i] = f; return f == 0.0f;
    case SYNTH_F64: ((double *)out)[i] = (double)f; return f == 0.0f;
    case SYNTH_BF16: {
      uint16_t b = f32_to_bf16_bits(f);
      ((uint16_t *)out)[i] = b;
      return (b & 0x7FFFu) == 0;
    }
    case SYNTH_F16: {
      _Float16 h = (_Float16)f;
      memcpy((uint16_t *)out + i, &h, 2);
      return h == (_Float16)0.0f;
    }
  }
  return 0;
}

typedef struct {
  void *out;
  int64_t begin, end;
  int dtype;
  double mean, stddev;
  uint64_t seed, stream;
  int nonzero;
} synth_job;

static void *synth_worker(void *arg) {
  const synth_job *j = (const synth_job *)arg;
  for (int64_t i = j->begin; i < j->end; ++i) {
    const uint64_t block = (uint64_t)i >> 2;
    const int lane = (int)(i & 3);
    uint64_t attempt = 0;
    for (;;) {
      const double v = j->mean + j->stddev * lane_normal(j->seed, j->stream, block, attempt, lane);
      const int is_zero = store_one(j->out, i, j->dtype, v);
      if (!j->nonzero || !is_zero || attempt >= 64) break;
      ++attempt;
    }
  }
  return NULL;
}

/*
 * Fill out[0..n) with mean + std * N(0,1) samples in `dtype` storage.
 * Returns 0 on success, -1 on a bad argument.
 */
int synth_normal(void *out, int64_t n, int dtype, double mean, double stddev,
                 uint64_t seed, uint64_t stream, int nonzero, int nthreads) {
  if (n < 0 || (n > 0 && !out) || dtype < 0 || dtype > 3) return -1;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (n < (int64_t)1 << 16) nthreads = 1;
  pthread_t tid[256];
  synth_job jobs[256];
  const int64_t chunk = (n + nthreads - 1) / nthreads;
  int started = 0;
  for (int t = 0; t < nthreads; ++t) {
    int64_t b = (int64_t)t * chunk, e = b + chunk;
    if (b > n) b = n;
    if (e > n) e = n;
    jobs[t] = (synth_job){out, b, e, dtype, mean, stddev, seed, stream, nonzero};
    if (nthreads == 1) {
      synth_worker(&jobs[t]);
    } else if (pthread_create(&tid[t], NULL, synth_worker, &jobs[t]) == 0) {
      ++started;
    } else {
      synth_worker(&jobs[t]);
      tid[t] = 0;
    }
  }
  if (nthreads > 1)
    for (int t = 0; t < nthreads; ++t)
      if (tid[t]) pthread_join(tid[t], NULL);
  (void)started;
  return 0;
}
