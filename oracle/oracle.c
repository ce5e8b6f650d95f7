/*
 * oracle.c -- plain, slow, fp64 CPU reference for the hybrid linear/full
 * attention hot path.  TEST INFRASTRUCTURE ONLY: only the tests, the smoke
 * check and the benchmark's CPU-baseline leg may load this library.  It shares
 * no code, header, table or helper with the CUDA library.
 *
 * Every input arrives as fp64 (the exact bf16 / fp32 values the GPU is given,
 * widened), every intermediate and output is fp64.  No blocking, no fusion, no
 * chunking: each function is the plain definition written out, one token / one
 * query row at a time.
 *
 * Sources (the pages name the layers; none prints a formula):
 *  - "The Hybrid Attention in Qwen3.8-27B -- Only 16 of 64 Layers Grow a KV
 *    Cache", sections "Why 27B parameters can carry 262K tokens" (Gated
 *    DeltaNet layers, a fixed-size state that does not grow with the sequence)
 *    and "Grouped-query attention multiplies on top of that" (24 query heads
 *    over 4 key/value heads at head dim 256; 48 value heads over 16 q/k heads
 *    at head dim 128).
 *  - "The economics of hybrid attention", TL;DR (the fixed ~150 MiB
 *    recurrent state) and "What a token of context costs" (KV per token).
 *  - "HydraHead: From Head-Level Functional Heterogeneity to Specialized
 *    Attention Hybridization", abstract (FA and LA heads in one layer, joined
 *    by a scale-normalized fusion module).
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *  - Gated delta rule, per value head h (q/k head h / (H_v/H_qk)):
 *        S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *        o_t = scale * S_t q_t
 *    S is d_v x d_k.  The product S (I - beta k k^T) is evaluated as
 *    S - beta (S k) k^T, which is the same matrix up to rounding order; a
 *    CPU test checks it against the explicit (I - beta k k^T) products.
 *  - Attention: o_t = sum_{j<limit} softmax_j(scale q_t . k_j) v_j, optionally
 *    multiplied elementwise by sigmoid(G_t); causal means limit = t + 1.
 *  - Scale-normalized fusion: y = x / sqrt(mean_i x_i^2 + eps), no gain.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* a tiny static work splitter: job j of n_jobs goes to thread j % n_threads  */
/* ------------------------------------------------------------------------ */
typedef void (*job_fn)(void *ctx, int64_t job);
typedef struct {
  job_fn fn;
  void *ctx;
  int64_t n_jobs;
  int tid, n_threads;
} worker_arg;

static void *worker_main(void *p) {
  worker_arg *w = (worker_arg *)p;
  for (int64_t j = w->tid; j < w->n_jobs; j += w->n_threads) w->fn(w->ctx, j);
  return NULL;
}

static void run_jobs(job_fn fn, void *ctx, int64_t n_jobs, int n_threads) {
  if (n_threads < 1) n_threads = 1;
  if (n_threads > 256) n_threads = 256;
  if ((int64_t)n_threads > n_jobs) n_threads = (int)(n_jobs > 0 ? n_jobs : 1);
  pthread_t th[256];
  worker_arg args[256];
  for (int i = 0; i < n_threads; ++i) {
    args[i].fn = fn;
    args[i].ctx = ctx;
    args[i].n_jobs = n_jobs;
    args[i].tid = i;
    args[i].n_threads = n_threads;
  }
  for (int i = 1; i < n_threads; ++i) pthread_create(&th[i], NULL, worker_main, &args[i]);
  worker_main(&args[0]);
  for (int i = 1; i < n_threads; ++i) pthread_join(th[i], NULL);
}

/* ------------------------------------------------------------------------ */
/* Gated delta rule, token by token                                          */
/* ------------------------------------------------------------------------ */
typedef struct {
  const double *q, *k, *v, *g, *beta, *S0;
  double *o, *S_out;
  int64_t B, T, Hqk, Hv, dk, dv;
  double scale;
} gdn_ctx;

static void gdn_job(void *p, int64_t job) {
  const gdn_ctx *c = (const gdn_ctx *)p;
  const int64_t b = job / c->Hv, h = job % c->Hv;
  const int64_t hq = h / (c->Hv / c->Hqk); /* contiguous groups of value heads */
  const int64_t dk = c->dk, dv = c->dv;
  double *S = (double *)calloc((size_t)(dv * dk), sizeof(double));
  double *r = (double *)malloc((size_t)dv * sizeof(double));
  double *u = (double *)malloc((size_t)dv * sizeof(double));
  if (c->S0) memcpy(S, c->S0 + (b * c->Hv + h) * dv * dk, (size_t)(dv * dk) * sizeof(double));

  for (int64_t t = 0; t < c->T; ++t) {
    const double *qt = c->q + ((b * c->T + t) * c->Hqk + hq) * dk;
    const double *kt = c->k + ((b * c->T + t) * c->Hqk + hq) * dk;
    const double *vt = c->v + ((b * c->T + t) * c->Hv + h) * dv;
    const double gt = c->g[(b * c->T + t) * c->Hv + h];
    const double bt = c->beta[(b * c->T + t) * c->Hv + h];
    double *ot = c->o + ((b * c->T + t) * c->Hv + h) * dv;

    /* S <- exp(g_t) S */
    const double a = exp(gt);
    for (int64_t i = 0; i < dv * dk; ++i) S[i] *= a;
    /* S <- S (I - beta k k^T) + beta v k^T  ==  S + beta (v - S k) k^T */
    for (int64_t i = 0; i < dv; ++i) {
      double acc = 0.0;
      for (int64_t j = 0; j < dk; ++j) acc += S[i * dk + j] * kt[j];
      r[i] = acc;
    }
    for (int64_t i = 0; i < dv; ++i) u[i] = bt * (vt[i] - r[i]);
    for (int64_t i = 0; i < dv; ++i)
      for (int64_t j = 0; j < dk; ++j) S[i * dk + j] += u[i] * kt[j];
    /* o_t = scale * S_t q_t */
    for (int64_t i = 0; i < dv; ++i) {
      double acc = 0.0;
      for (int64_t j = 0; j < dk; ++j) acc += S[i * dk + j] * qt[j];
      ot[i] = c->scale * acc;
    }
  }
  if (c->S_out) memcpy(c->S_out + (b * c->Hv + h) * dv * dk, S, (size_t)(dv * dk) * sizeof(double));
  free(S);
  free(r);
  free(u);
}

/*
 * q, k  [B, T, Hqk, dk]      v, o [B, T, Hv, dv]      g, beta [B, T, Hv]
 * S0, S_out [B, Hv, dv, dk]  (S0 may be NULL = zeros; S_out may be NULL)
 * Returns 0, or -1 on bad sizes.
 */
int oracle_gdn(const double *q, const double *k, const double *v, const double *g,
               const double *beta, const double *S0, double *o, double *S_out, int64_t B,
               int64_t T, int64_t Hqk, int64_t Hv, int64_t dk, int64_t dv, double scale,
               int n_threads) {
  if (B < 0 || T < 0 || Hqk <= 0 || Hv <= 0 || dk <= 0 || dv <= 0 || Hv % Hqk != 0) return -1;
  gdn_ctx c = {q, k, v, g, beta, S0, o, S_out, B, T, Hqk, Hv, dk, dv, scale};
  run_jobs(gdn_job, &c, B * Hv, n_threads);
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Softmax attention, one query row at a time                                */
/* ------------------------------------------------------------------------ */
typedef struct {
  const double *q, *k, *v, *gate;
  const int64_t *limit;
  double *o;
  int64_t B, R, Tk, Hq, Hkv, d;
  double scale;
} attn_ctx;

static void attn_job(void *p, int64_t job) {
  const attn_ctx *c = (const attn_ctx *)p;
  const int64_t h = job % c->Hq, r = (job / c->Hq) % c->R, b = job / (c->Hq * c->R);
  const int64_t hk = h / (c->Hq / c->Hkv); /* contiguous groups of query heads */
  const int64_t d = c->d;
  int64_t n = c->limit[b * c->R + r];
  if (n > c->Tk) n = c->Tk;
  const double *qr = c->q + ((b * c->R + r) * c->Hq + h) * d;
  double *orow = c->o + ((b * c->R + r) * c->Hq + h) * d;
  if (n <= 0) { /* nothing visible: defined as a zero row */
    for (int64_t i = 0; i < d; ++i) orow[i] = 0.0;
    return;
  }
  double *s = (double *)malloc((size_t)n * sizeof(double));
  double m = -INFINITY;
  for (int64_t j = 0; j < n; ++j) {
    const double *kj = c->k + ((b * c->Tk + j) * c->Hkv + hk) * d;
    double acc = 0.0;
    for (int64_t i = 0; i < d; ++i) acc += qr[i] * kj[i];
    s[j] = c->scale * acc;
    if (s[j] > m) m = s[j];
  }
  double l = 0.0;
  for (int64_t j = 0; j < n; ++j) {
    s[j] = exp(s[j] - m);
    l += s[j];
  }
  for (int64_t i = 0; i < d; ++i) orow[i] = 0.0;
  for (int64_t j = 0; j < n; ++j) {
    const double *vj = c->v + ((b * c->Tk + j) * c->Hkv + hk) * d;
    for (int64_t i = 0; i < d; ++i) orow[i] += s[j] * vj[i];
  }
  for (int64_t i = 0; i < d; ++i) orow[i] /= l;
  if (c->gate) {
    const double *gr = c->gate + ((b * c->R + r) * c->Hq + h) * d;
    for (int64_t i = 0; i < d; ++i) orow[i] *= 1.0 / (1.0 + exp(-gr[i]));
  }
  free(s);
}

/*
 * Attention for R selected query rows per sequence.
 * q, gate, o [B, R, Hq, d]   k, v [B, Tk, Hkv, d]
 * limit [B, R]: query (b, r) sees keys 0 .. limit-1 (causal prefill: pos+1;
 * decode: the cache length).  gate may be NULL.
 */
int oracle_attention_rows(const double *q, const double *k, const double *v,
                          const double *gate, const int64_t *limit, double *o, int64_t B,
                          int64_t R, int64_t Tk, int64_t Hq, int64_t Hkv, int64_t d,
                          double scale, int n_threads) {
  if (B < 0 || R < 0 || Tk < 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || Hq % Hkv != 0) return -1;
  attn_ctx c = {q, k, v, gate, limit, o, B, R, Tk, Hq, Hkv, d, scale};
  run_jobs(attn_job, &c, B * R * Hq, n_threads);
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Scale-normalized fusion: y = x / sqrt(mean(x^2) + eps) per row of d       */
/* ------------------------------------------------------------------------ */
int oracle_rms_rows(const double *x, double *y, int64_t n_rows, int64_t d, double eps) {
  if (n_rows < 0 || d <= 0) return -1;
  for (int64_t r = 0; r < n_rows; ++r) {
    double ss = 0.0;
    for (int64_t i = 0; i < d; ++i) ss += x[r * d + i] * x[r * d + i];
    const double inv = 1.0 / sqrt(ss / (double)d + eps);
    for (int64_t i = 0; i < d; ++i) y[r * d + i] = x[r * d + i] * inv;
  }
  return 0;
}
