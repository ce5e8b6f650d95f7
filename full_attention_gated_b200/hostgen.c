/* hostgen.c -- host-side twin of the counter-based cache generator, threaded.
 *
 * Input generation only; none of the layer's arithmetic.  Element i of a tensor
 * (seed, stream) is the bf16 rounding (to nearest, ties to even) of
 *     (sum of the eight 16-bit halves of Philox4x32-10(ctr, key) - 262140) * inv_sigma
 * with ctr = (i mod 2^32, i / 2^32, stream, 0x48480000), key = (seed mod 2^32,
 * seed / 2^32) and inv_sigma = 1 / sqrt(8 (65536^2 - 1) / 12) rounded to float:
 * an Irwin-Hall(8) approximation of N(0, 1).  Philox4x32-10 is the generator of
 * Salmon, Moraes, Dror and Shaw, "Parallel random numbers: as easy as 1, 2, 3"
 * (SC'11).  inputs.py holds the same definition in numpy (the reference the
 * tests compare this file against bit for bit); this version exists because the
 * numpy one takes seconds per 131,072-token cache slice.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

static uint16_t bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  const uint32_t lsb = (u >> 16) & 1u;
  return (uint16_t)((u + 0x7FFFu + lsb) >> 16);
}

static uint16_t counter_normal(uint64_t i, uint64_t seed, uint32_t stream, float inv_sigma) {
  uint32_t c0 = (uint32_t)i, c1 = (uint32_t)(i >> 32), c2 = stream, c3 = 0x48480000u;
  uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);
  for (int r = 0; r < 10; ++r) {
    const uint64_t p0 = (uint64_t)0xD2511F53u * c0, p1 = (uint64_t)0xCD9E8D57u * c2;
    const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0, n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
    c0 = n0;
    c1 = (uint32_t)p1;
    c2 = n2;
    c3 = (uint32_t)p0;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  const int s = (int)(c0 & 0xFFFFu) + (int)(c0 >> 16) + (int)(c1 & 0xFFFFu) + (int)(c1 >> 16) +
                (int)(c2 & 0xFFFFu) + (int)(c2 >> 16) + (int)(c3 & 0xFFFFu) + (int)(c3 >> 16);
  return bf16_rne((float)(s - 262140) * inv_sigma);
}

/* q8_0 twin: value = clip(rint(32 z), -127, 127) with z the bf16 normal (32 z is exact); scale =
 * (64 + (bits & 63)) / 4096, whose fp16 pattern is exponent 9 (2^-6), mantissa (m - 64) << 4 for m = 64 + h. */
static int8_t q8_value(uint64_t i, uint64_t seed, uint32_t stream, float inv_sigma) {
  const uint32_t b = (uint32_t)counter_normal(i, seed, stream, inv_sigma) << 16;
  float z;
  memcpy(&z, &b, 4);
  float x = rintf(32.0f * z);
  x = x < -127.0f ? -127.0f : (x > 127.0f ? 127.0f : x);
  return (int8_t)(int)x;
}
static uint16_t q8_scale_bits(uint64_t j, uint64_t seed, uint32_t stream, float inv_sigma) {
  const uint32_t h = counter_normal(j, seed, stream, inv_sigma) & 63u;
  return (uint16_t)((9u << 10) | (h << 4));
}

typedef struct {
  uint16_t *out;
  int8_t *vals;
  uint16_t *scales;
  uint32_t stream_s;
  uint64_t seed;
  uint32_t stream;
  int64_t Tc, Hkv, d, b, hk, t0, t1, r0, r1;
  float inv_sigma;
} Job;

static void *run(void *arg) {
  const Job *j = (const Job *)arg;
  for (int64_t t = j->t0 + j->r0; t < j->t0 + j->r1; ++t) {
    const uint64_t row_id = (uint64_t)((j->b * j->Tc + t) * j->Hkv + j->hk);
    const uint64_t base = row_id * (uint64_t)j->d;
    if (j->vals) {
      int8_t *row = j->vals + (t - j->t0) * j->d;
      uint16_t *srow = j->scales + (t - j->t0) * (j->d / 32);
      for (int64_t e = 0; e < j->d; ++e) row[e] = q8_value(base + (uint64_t)e, j->seed, j->stream, j->inv_sigma);
      for (int64_t e = 0; e < j->d / 32; ++e)
        srow[e] = q8_scale_bits(row_id * (uint64_t)(j->d / 32) + (uint64_t)e, j->seed, j->stream_s, j->inv_sigma);
    } else {
      uint16_t *row = j->out + (t - j->t0) * j->d;
      for (int64_t e = 0; e < j->d; ++e) row[e] = counter_normal(base + (uint64_t)e, j->seed, j->stream, j->inv_sigma);
    }
  }
  return 0;
}

static int slice(uint16_t *out, int8_t *vals, uint16_t *scales, uint64_t seed, uint32_t stream, uint32_t stream_s,
                 int64_t Tc, int64_t Hkv, int64_t d, int64_t b, int64_t hk, int64_t t0, int64_t t1, int n_threads) {
  if ((!out && !vals) || t0 < 0 || t1 < t0 || t1 > Tc || hk < 0 || hk >= Hkv || b < 0 || d <= 0) return -1;
  if (n_threads < 1) n_threads = 1;
  if (n_threads > 256) n_threads = 256;
  const float inv_sigma = (float)(1.0 / sqrt(8.0 * (65536.0 * 65536.0 - 1.0) / 12.0));
  const int64_t rows = t1 - t0;
  pthread_t th[256];
  int live[256];
  Job jobs[256];
  for (int w = 0; w < n_threads; ++w) {
    Job *j = &jobs[w];
    j->out = out;
    j->vals = vals;
    j->scales = scales;
    j->stream_s = stream_s;
    j->seed = seed;
    j->stream = stream;
    j->Tc = Tc;
    j->Hkv = Hkv;
    j->d = d;
    j->b = b;
    j->hk = hk;
    j->t0 = t0;
    j->t1 = t1;
    j->r0 = rows * w / n_threads;
    j->r1 = rows * (w + 1) / n_threads;
    j->inv_sigma = inv_sigma;
    live[w] = pthread_create(&th[w], 0, run, j) == 0;
    if (!live[w]) run(j); /* no thread: do this share here */
  }
  for (int w = 0; w < n_threads; ++w)
    if (live[w]) pthread_join(th[w], 0);
  return 0;
}

/* Rows [t0, t1) of kv head hk of sequence b of a [B, Tc, Hkv, d] generated cache, written to out as
 * [t1 - t0, d] bf16 bits.  Returns 0, or -1 on a bad argument. */
int hostgen_cache_slice(uint16_t *out, uint64_t seed, uint32_t stream, int64_t Tc, int64_t Hkv, int64_t d,
                        int64_t b, int64_t hk, int64_t t0, int64_t t1, int n_threads) {
  return slice(out, 0, 0, seed, stream, 0, Tc, Hkv, d, b, hk, t0, t1, n_threads);
}

/* The same rows of a generated q8_0 cache: values [t1 - t0, d] int8 and scales [t1 - t0, d / 32] fp16 bits. */
int hostgen_q8_0_slice(int8_t *vals, uint16_t *scales, uint64_t seed, uint32_t stream_x, uint32_t stream_s,
                       int64_t Tc, int64_t Hkv, int64_t d, int64_t b, int64_t hk, int64_t t0, int64_t t1,
                       int n_threads) {
  if (!vals || !scales || d % 32) return -1;
  return slice(0, vals, scales, seed, stream_x, stream_s, Tc, Hkv, d, b, hk, t0, t1, n_threads);
}
