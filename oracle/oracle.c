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

/* ------------------------------------------------------------------------ */
/* PHBA: top-K block routing with block-aligned prefix states                */
/* ("PHBA: Prefix-State Hybrid Block Attention", abstract and Figure 1).     */
/* The page names the parts and prints no formula; the readings, one per     */
/* part, are:                                                                */
/*  - blocks: token t is in block t / C; nb = ceil(T / C).                   */
/*  - prefix states: a gated slot memory of M slots over the raw keys and    */
/*    the values, Kt_{t+1}[m] = a_{t,m} Kt_t[m] + (1 - a_{t,m}) kraw_t and    */
/*    Vt_{t+1}[m] = a_{t,m} Vt_t[m] + (1 - a_{t,m}) v_t from zero; the state  */
/*    of block j is the memory after the j C tokens before it (block 0's is  */
/*    empty and never attended).                                             */
/*  - routing: query t scores every earlier block j < t / C by               */
/*    qrope_t . mean_{s in block j} krope_s and keeps the min(K, t / C)       */
/*    best (a tie goes to the lower block index).                            */
/*  - attention: one softmax over the tokens of the kept blocks, the tokens  */
/*    s <= t of the query's own block (logits scale qrope_t . krope_s,       */
/*    values v_s) and the M slots of the prefix state of every kept block    */
/*    and of the own block, where that state is not empty (logits           */
/*    scale qraw_t . Kt[m], values Vt[m]).                                   */
/* ------------------------------------------------------------------------ */
typedef struct {
  const double *kraw, *v, *alpha;
  double *kst, *vst;
  int64_t B, T, H, d, M, C, nb;
} phba_state_ctx;

static void phba_state_job(void *p, int64_t job) {
  const phba_state_ctx *c = (const phba_state_ctx *)p;
  const int64_t h = job % c->H, b = job / c->H, d = c->d, M = c->M;
  double *K = (double *)calloc((size_t)(M * d), sizeof(double));
  double *V = (double *)calloc((size_t)(M * d), sizeof(double));
  for (int64_t t = 0; t <= c->T; ++t) {
    if (t % c->C == 0 && t / c->C < c->nb) { /* the state before block t / C */
      const int64_t j = t / c->C;
      double *ko = c->kst + (((b * c->H + h) * c->nb + j) * M) * d;
      double *vo = c->vst + (((b * c->H + h) * c->nb + j) * M) * d;
      memcpy(ko, K, (size_t)(M * d) * sizeof(double));
      memcpy(vo, V, (size_t)(M * d) * sizeof(double));
    }
    if (t == c->T) break;
    const double *kt = c->kraw + ((b * c->T + t) * c->H + h) * d;
    const double *vt = c->v + ((b * c->T + t) * c->H + h) * d;
    const double *at = c->alpha + ((b * c->T + t) * c->H + h) * M;
    for (int64_t m = 0; m < M; ++m)
      for (int64_t i = 0; i < d; ++i) {
        K[m * d + i] = at[m] * K[m * d + i] + (1.0 - at[m]) * kt[i];
        V[m * d + i] = at[m] * V[m * d + i] + (1.0 - at[m]) * vt[i];
      }
  }
  free(K);
  free(V);
}

/*
 * kraw, v [B, T, H, d]; alpha [B, T, H, M] (each in (0, 1)); kst, vst [B, H, nb, M, d]:
 * entry j is the slot memory after tokens 0 .. jC - 1 (entry 0 is zero).
 */
int oracle_phba_states(const double *kraw, const double *v, const double *alpha, double *kst, double *vst,
                       int64_t B, int64_t T, int64_t H, int64_t d, int64_t M, int64_t C, int n_threads) {
  if (B < 0 || T <= 0 || H <= 0 || d <= 0 || M <= 0 || C <= 0) return -1;
  phba_state_ctx c = {kraw, v, alpha, kst, vst, B, T, H, d, M, C, (T + C - 1) / C};
  run_jobs(phba_state_job, &c, B * H, n_threads);
  return 0;
}

typedef struct {
  const double *qrope, *krope;
  int64_t *sel;
  double *scores;
  int64_t B, T, H, d, C, K, nb;
} phba_route_ctx;

static void phba_route_job(void *p, int64_t job) {
  const phba_route_ctx *c = (const phba_route_ctx *)p;
  const int64_t h = job % c->H, b = job / c->H, d = c->d, nb = c->nb, C = c->C;
  /* mean key of every complete block */
  const int64_t nfull = c->T / C;
  double *kbar = (double *)calloc((size_t)((nfull > 0 ? nfull : 1) * d), sizeof(double));
  for (int64_t j = 0; j < nfull; ++j) {
    for (int64_t s = j * C; s < (j + 1) * C; ++s) {
      const double *ks = c->krope + ((b * c->T + s) * c->H + h) * d;
      for (int64_t i = 0; i < d; ++i) kbar[j * d + i] += ks[i];
    }
    for (int64_t i = 0; i < d; ++i) kbar[j * d + i] /= (double)C;
  }
  char *taken = (char *)malloc((size_t)nb);
  for (int64_t t = 0; t < c->T; ++t) {
    const int64_t nt = t / C; /* candidates: blocks 0 .. nt - 1, all complete */
    const double *qt = c->qrope + ((b * c->T + t) * c->H + h) * d;
    double *sc = c->scores + ((b * c->T + t) * c->H + h) * nb;
    for (int64_t j = 0; j < nb; ++j) {
      if (j < nt) {
        double acc = 0.0;
        for (int64_t i = 0; i < d; ++i) acc += qt[i] * kbar[j * d + i];
        sc[j] = acc;
      } else {
        sc[j] = -INFINITY;
      }
      taken[j] = 0;
    }
    int64_t *st = c->sel + ((b * c->T + t) * c->H + h) * c->K;
    const int64_t n_keep = nt < c->K ? nt : c->K;
    for (int64_t r = 0; r < n_keep; ++r) { /* r-th best: highest score, lower index on a tie */
      int64_t best = -1;
      for (int64_t j = 0; j < nt; ++j)
        if (!taken[j] && (best < 0 || sc[j] > sc[best])) best = j;
      if (best < 0) break;
      taken[best] = 1;
    }
    int64_t w = 0; /* kept blocks in ascending order, then -1 */
    for (int64_t j = 0; j < nt; ++j)
      if (taken[j]) st[w++] = j;
    while (w < c->K) st[w++] = -1;
  }
  free(taken);
  free(kbar);
}

/*
 * qrope, krope [B, T, H, d]; sel [B, T, H, K] (out: the kept blocks, ascending, -1 past the
 * last); scores [B, T, H, nb] (out: the routing scores, -inf for blocks that are not candidates).
 */
int oracle_phba_route(const double *qrope, const double *krope, int64_t *sel, double *scores, int64_t B,
                      int64_t T, int64_t H, int64_t d, int64_t C, int64_t K, int n_threads) {
  if (B < 0 || T <= 0 || H <= 0 || d <= 0 || C <= 0 || K < 0) return -1;
  phba_route_ctx c = {qrope, krope, sel, scores, B, T, H, d, C, K, (T + C - 1) / C};
  run_jobs(phba_route_job, &c, B * H, n_threads);
  return 0;
}

typedef struct {
  const double *qrope, *krope, *qraw, *v, *kst, *vst;
  const int64_t *sel, *rows;
  double *o;
  int64_t B, T, R, H, d, M, C, K, nb;
  double scale;
} phba_attn_ctx;

static void phba_attn_job(void *p, int64_t job) {
  const phba_attn_ctx *c = (const phba_attn_ctx *)p;
  const int64_t h = job % c->H, r = (job / c->H) % c->R, b = job / (c->H * c->R);
  const int64_t t = c->rows ? c->rows[r] : r;
  const int64_t d = c->d, M = c->M, C = c->C, nt = t / C;
  const double *qr = c->qrope + ((b * c->T + t) * c->H + h) * d;
  const double *qw = c->qraw + ((b * c->T + t) * c->H + h) * d;
  const int64_t *st = c->sel + ((b * c->T + t) * c->H + h) * c->K;
  /* the attended blocks: the kept ones and the own block */
  int64_t nblk = 0;
  int64_t *blk = (int64_t *)malloc((size_t)(c->K + 1) * sizeof(int64_t));
  for (int64_t r = 0; r < c->K; ++r)
    if (st[r] >= 0) blk[nblk++] = st[r];
  blk[nblk++] = nt;
  const int64_t cap = nblk * (C + M);
  double *lg = (double *)malloc((size_t)cap * sizeof(double));
  const double **val = (const double **)malloc((size_t)cap * sizeof(double *));
  int64_t n = 0;
  for (int64_t u = 0; u < nblk; ++u) {
    const int64_t j = blk[u];
    const int64_t s_end = j == nt ? t + 1 : (j + 1) * C; /* own block: causal */
    for (int64_t s = j * C; s < s_end; ++s) {
      const double *ks = c->krope + ((b * c->T + s) * c->H + h) * d;
      double acc = 0.0;
      for (int64_t i = 0; i < d; ++i) acc += qr[i] * ks[i];
      lg[n] = c->scale * acc;
      val[n++] = c->v + ((b * c->T + s) * c->H + h) * d;
    }
    if (j >= 1) { /* the prefix state of block j */
      const double *kj = c->kst + (((b * c->H + h) * c->nb + j) * M) * d;
      const double *vj = c->vst + (((b * c->H + h) * c->nb + j) * M) * d;
      for (int64_t m = 0; m < M; ++m) {
        double acc = 0.0;
        for (int64_t i = 0; i < d; ++i) acc += qw[i] * kj[m * d + i];
        lg[n] = c->scale * acc;
        val[n++] = vj + m * d;
      }
    }
  }
  double mx = -INFINITY;
  for (int64_t e = 0; e < n; ++e)
    if (lg[e] > mx) mx = lg[e];
  double l = 0.0;
  double *orow = c->o + ((b * c->R + r) * c->H + h) * d;
  for (int64_t i = 0; i < d; ++i) orow[i] = 0.0;
  for (int64_t e = 0; e < n; ++e) {
    const double w = exp(lg[e] - mx);
    l += w;
    for (int64_t i = 0; i < d; ++i) orow[i] += w * val[e][i];
  }
  for (int64_t i = 0; i < d; ++i) orow[i] /= l;
  free(val);
  free(lg);
  free(blk);
}

/*
 * qrope, krope, qraw, v [B, T, H, d]; kst, vst [B, H, nb, M, d] (oracle_phba_states);
 * sel [B, T, H, K]: the kept blocks of every query (oracle_phba_route's, or any other valid
 * choice), -1 for none.  rows [R]: the query positions to compute (NULL: all, R = T);
 * o [B, R, H, d].
 */
int oracle_phba_attention(const double *qrope, const double *krope, const double *qraw, const double *v,
                          const double *kst, const double *vst, const int64_t *sel, const int64_t *rows,
                          double *o, int64_t B, int64_t T, int64_t R, int64_t H, int64_t d, int64_t M,
                          int64_t C, int64_t K, double scale, int n_threads) {
  if (B < 0 || T <= 0 || R < 0 || H <= 0 || d <= 0 || M <= 0 || C <= 0 || K < 0) return -1;
  if (!rows && R != T) return -1;
  for (int64_t r = 0; rows && r < R; ++r)
    if (rows[r] < 0 || rows[r] >= T) return -1;
  phba_attn_ctx c = {qrope, krope, qraw, v, kst, vst, sel, rows, o, B, T, R, H, d, M, C, K, (T + C - 1) / C,
                     scale};
  run_jobs(phba_attn_job, &c, B * R * H, n_threads);
  return 0;
}
