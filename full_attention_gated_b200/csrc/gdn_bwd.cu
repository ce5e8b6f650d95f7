// gdn_bwd.cu -- gradients of the gated delta rule over a sequence: the backward pass of
// gdn_chunk_fwd.
//
// The layers are trained ("HydraHead: From Head-Level Functional Heterogeneity to
// Specialized Attention Hybridization", abstract: the hybrid heads come out of a transfer
// and distillation pipeline; "PHBA: Prefix-State Hybrid Block Attention", Figure 3: training
// throughput), which needs the gradients of
//     L = sum_t o_t . dO_t + S_T . dS_T
// through S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T, o_t = scale S_t q_t,
// with respect to q, k, v, g, beta and S_0.  In the chunked form (C = 64) the chunk map is
// affine, S_{c+1} = S_c A_c + B_c, and the chunk's output is O_c = scale (Qt_c S_c^T + P_c U'_c),
// so the backward splits into
//   1. the forward pass with the start state S_c of every chunk kept (gdn_scan's chunk_states);
//   2. a reverse scan over chunks carrying the state's cotangent,
//          dS_c = dS_{c+1} A_c^T + scale dO_c^T Qt_c,      dS_n = dS_T,  dS_0 -> dS0;
//   3. per chunk, independently, the cotangents of the chunk's maps,
//          dA = S_c^T dS_{c+1},  dB = dS_{c+1},  dQt = scale dO S_c,  dP = scale dO U'^T,
//          dU' = scale P^T dO,
//      pulled back through B = U'^T diag(e) K, A = gamma_C I - W^T diag(e) K, Qt = diag(gamma) Q - P W,
//      P = tril(D o Q K^T), W = T diag(beta gamma) K, U' = T diag(beta) V, T = (I + A_in)^-1 with
//      A_in = strict_tril(beta_i D_ij k_i.k_j), D_ij = exp(G_i - G_j), G = cumsum(g), to q, k, v, g
//      and beta.
// Steps 2 and 3 run in fp32 on the CUDA cores (products tiled through shared memory); the chunk's
// forward quantities are recomputed in fp32 from the inputs.  Step 1 is the forward pass itself.
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"

namespace hh {

namespace {

constexpr int kC = 64;
constexpr int kD = 128;
constexpr int kBT = 256;  // threads per CTA of both kernels

__device__ __forceinline__ float ldf(const float *p) { return *p; }
__device__ __forceinline__ float ldf(const bf16_t *p) { return bf16_to_f(*p); }

// C = alpha op(A) op(B) + beta C on the whole CTA (256 threads).  op(A) is M x K: A row-major with
// leading dimension lda, or its transpose (ta); op(B) is K x N likewise (tb).  M and N multiples of 64,
// K a multiple of 32.  beta = 0 does not read C.  `sm` holds 2 x 32 x 68 floats.  Each 64 x 64 tile of C
// runs over K in steps of 32: the next step's operands are loaded into registers while the current
// step's multiply-adds run from shared memory.  Ends with a barrier.
constexpr int kKS = 32;
constexpr int kMmSmem = 2 * kKS * 68;
template <typename TA, typename TB>
__device__ void cta_mm(float *C, int ldc, const TA *A, int lda, bool ta, const TB *B, int ldb, bool tb, int M, int N,
                       int K, float alpha, float beta, float *sm) {
  const int tid = threadIdx.x, tr = tid >> 4, tcol = tid & 15;
  float *As = sm, *Bs = sm + kKS * 68;  // As[k][m], Bs[k][n] (padded rows)
  float ra[8], rb[8];
  auto load = [&](int m0, int n0, int k0) {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int i = tid + r * kBT;  // 0 .. 2047
      ra[r] = ta ? ldf(A + (size_t)(k0 + (i >> 6)) * lda + m0 + (i & 63)) : ldf(A + (size_t)(m0 + (i >> 5)) * lda + k0 + (i & 31));
      rb[r] = tb ? ldf(B + (size_t)(n0 + (i >> 5)) * ldb + k0 + (i & 31)) : ldf(B + (size_t)(k0 + (i >> 6)) * ldb + n0 + (i & 63));
    }
  };
  auto stage = [&]() {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int i = tid + r * kBT;
      if (ta) As[(i >> 6) * 68 + (i & 63)] = ra[r]; else As[(i & 31) * 68 + (i >> 5)] = ra[r];
      if (tb) Bs[(i & 31) * 68 + (i >> 5)] = rb[r]; else Bs[(i >> 6) * 68 + (i & 63)] = rb[r];
    }
  };
  for (int m0 = 0; m0 < M; m0 += 64)
    for (int n0 = 0; n0 < N; n0 += 64) {
      float acc[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
      load(m0, n0, 0);
      stage();
      __syncthreads();
      for (int k0 = 0; k0 < K; k0 += kKS) {
        const bool more = k0 + kKS < K;
        if (more) load(m0, n0, k0 + kKS);
#pragma unroll 8
        for (int kk = 0; kk < kKS; ++kk) {
          const float4 a = *reinterpret_cast<const float4 *>(As + kk * 68 + tr * 4);
          const float4 b = *reinterpret_cast<const float4 *>(Bs + kk * 68 + tcol * 4);
          const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        __syncthreads();
        if (more) {
          stage();
          __syncthreads();
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float4 *c = reinterpret_cast<float4 *>(C + (size_t)(m0 + tr * 4 + i) * ldc + n0 + tcol * 4);
        float4 v = make_float4(alpha * acc[i][0], alpha * acc[i][1], alpha * acc[i][2], alpha * acc[i][3]);
        if (beta != 0.f) {
          const float4 o = *c;
          v.x = fmaf(beta, o.x, v.x);
          v.y = fmaf(beta, o.y, v.y);
          v.z = fmaf(beta, o.z, v.z);
          v.w = fmaf(beta, o.w, v.w);
        }
        *c = v;
      }
    }
  __syncthreads();
}

// rows [t0, t0 + 64) of head h of a [B, T, H, 128] bf16 tensor -> fp32 [64][128], zero past T
__device__ void load_rows(float *dst, const bf16_t *src, int b, int T, int H, int h, int t0) {
  for (int i = threadIdx.x; i < kC * kD; i += kBT) {
    const int t = i >> 7, j = i & 127;
    dst[i] = t0 + t < T ? bf16_to_f(src[(((size_t)b * T + t0 + t) * H + h) * kD + j]) : 0.f;
  }
}

struct BwdParams {
  const bf16_t *q, *k, *v, *dO;
  const float *g, *beta, *dS_T;  // dS_T nullable
  const float *chunk_states;     // [B, H_v, n_chunks, 128 (k), 128 (v)]: S^T at each chunk's start
  const bf16_t *rec_w, *rec_q;   // forward records: -W_e^T, Qt^T [B, H_v, n_chunks][128][64] bf16
  const float *rec_f;            // [B, H_v, n_chunks][2][64]: gamma, exp(G_C - G)
  float *dS;                     // [B, H_v, n_chunks][128 (v)][128 (k)]: dS_{c+1} of every chunk
  float *dq, *dk, *dv, *dg, *dbeta, *dS0;  // dS0 nullable
  float *scan_scratch;           // per (b, head, row block): X [64][64], K [64][128], dO [64][128]
  float *chunk_scratch;          // per pullback CTA: kChunkScratch floats
  int B, T, H_qk, H_v, group, n_chunks, n_items;
  float scale;
};

// ---- reverse scan, chunks from last to first.  Row v of dS_c depends only on row v of dS_{c+1}
// (A_c^T acts on the right), so each CTA carries 64 rows of one (head, sequence): grid (heads, B, 2). ----
__global__ void __launch_bounds__(kBT) gdn_bwd_scan_kernel(const __grid_constant__ BwdParams p) {
  __shared__ __align__(16) float sm[kMmSmem];
  const int h = blockIdx.x, b = blockIdx.y, rb = blockIdx.z;  // rows 64 rb .. 64 rb + 63 of dS
  const size_t rec0 = ((size_t)b * p.H_v + h) * p.n_chunks;
  float *X = p.scan_scratch + (((size_t)b * p.H_v + h) * 2 + rb) * (3 * kC * kD), *Kc = X + kC * kD, *dOc = Kc + kC * kD;
  const int n = p.n_chunks;
  const size_t roff = (size_t)rb * 64 * kD;  // first element of this CTA's rows
  {  // dS_n = dS_T (or zero)
    float *last = p.dS + (rec0 + n - 1) * kD * kD + roff;
    const float *src = p.dS_T ? p.dS_T + ((size_t)b * p.H_v + h) * kD * kD + roff : nullptr;
    for (int i = threadIdx.x; i < 64 * kD; i += kBT) last[i] = src ? src[i] : 0.f;
  }
  __syncthreads();
  for (int c = n - 1; c >= 0; --c) {
    const float *cur = p.dS + (rec0 + c) * kD * kD + roff;  // dS_{c+1}, this CTA's rows
    float *nxt = c > 0 ? p.dS + (rec0 + c - 1) * kD * kD + roff
                       : (p.dS0 ? p.dS0 + ((size_t)b * p.H_v + h) * kD * kD + roff : nullptr);
    if (!nxt) break;
    load_rows(Kc, p.k, b, p.T, p.H_qk, h / p.group, c * kC);
    load_rows(dOc, p.dO, b, p.T, p.H_v, h, c * kC);
    const float gC = p.rec_f[(rec0 + c) * 128 + kC - 1];
    for (int i = threadIdx.x; i < 64 * kD; i += kBT) nxt[i] = gC * cur[i];
    __syncthreads();
    // X = dS_{c+1} K^T  [v][t]
    cta_mm(X, kC, cur, kD, false, Kc, kD, true, 64, kC, kD, 1.f, 0.f, sm);
    // + X (-W_e): (-W_e)[t][m] = rec_w[m][t]
    const bf16_t *rw = p.rec_w + (rec0 + c) * kD * kC, *rq = p.rec_q + (rec0 + c) * kD * kC;
    cta_mm(nxt, kD, X, kC, false, rw, kC, true, 64, kD, kC, 1.f, 1.f, sm);
    // + scale dO^T Qt (this CTA's value columns of dO): Qt[t][m] = rec_q[m][t]
    cta_mm(nxt, kD, dOc + rb * 64, kD, true, rq, kC, true, 64, kD, kC, p.scale, 1.f, sm);
  }
}

// per-CTA scratch of the pullback (floats)
constexpr int kMat = kC * kD;  // 64 x 128
constexpr int kSq = kC * kC;   // 64 x 64
enum : int {
  oQf = 0, oKf = oQf + kMat, oVf = oKf + kMat, oDO = oVf + kMat, oW = oDO + kMat, oUp = oW + kMat, oRW = oUp + kMat,
  oRU = oRW + kMat, odQt = oRU + kMat, odUp = odQt + kMat, odW = odUp + kMat, odQ = odW + kMat, odK = odQ + kMat,
  odV = odK + kMat, oT1 = odV + kMat, oT2 = oT1 + kMat, odA = oT2 + kMat, oKK = odA + kD * kD, oQK = oKK + kSq,
  oDm = oQK + kSq, oTm = oDm + kSq, oP = oTm + kSq, odP = oP + kSq, odD = odP + kSq, odTm = odD + kSq, oS1 = odTm + kSq,
  oS2 = oS1 + kSq, kChunkScratch = oS2 + kSq
};

// ---- per-chunk pullback: a persistent grid over (chunk, head, sequence) ----
__global__ void __launch_bounds__(kBT, 2) gdn_bwd_chunk_kernel(const __grid_constant__ BwdParams p) {
  __shared__ __align__(16) float sm[kMmSmem];  // product tiles; A_in while T = (I + A_in)^-1 is formed
  __shared__ float Tsh[kC][kC + 1];
  float(*Ash)[kC + 1] = reinterpret_cast<float(*)[kC + 1]>(sm);
  static_assert(kC * (kC + 1) <= kMmSmem, "A_in fits in the product tiles");
  __shared__ float G[kC], gam[kC], ee[kC], bb[kC], dgam[kC], de[kC], dbeta[kC], dG[kC];
  __shared__ float red[2];
  float *sc = p.chunk_scratch + (size_t)blockIdx.x * kChunkScratch;
  float *Qf = sc + oQf, *Kf = sc + oKf, *Vf = sc + oVf, *dOf = sc + oDO, *W = sc + oW, *Up = sc + oUp, *RW = sc + oRW,
        *RU = sc + oRU, *dQt = sc + odQt, *dUp = sc + odUp, *dW = sc + odW, *dQ = sc + odQ, *dK = sc + odK,
        *dV = sc + odV, *T1 = sc + oT1, *T2 = sc + oT2, *dA = sc + odA, *KK = sc + oKK, *QK = sc + oQK, *Dm = sc + oDm,
        *Tm = sc + oTm, *P = sc + oP, *dP = sc + odP, *dD = sc + odD, *dTm = sc + odTm, *S1 = sc + oS1, *S2 = sc + oS2;
  const int tid = threadIdx.x;
  for (int item = blockIdx.x; item < p.n_items; item += gridDim.x) {
    const int h = item % p.H_v, rest = item / p.H_v, c = rest % p.n_chunks, b = rest / p.n_chunks;
    const int qh = h / p.group, t0 = c * kC, nv = min(kC, p.T - t0);
    const size_t rec = ((size_t)b * p.H_v + h) * p.n_chunks + c;
    const float *ST = p.chunk_states + rec * kD * kD;  // S_c^T [k][v]
    const float *dS = p.dS + rec * kD * kD;            // dS_{c+1} [v][k]
    // ---- inputs of the chunk (zero past T) and its gates ----
    load_rows(Qf, p.q, b, p.T, p.H_qk, qh, t0);
    load_rows(Kf, p.k, b, p.T, p.H_qk, qh, t0);
    load_rows(Vf, p.v, b, p.T, p.H_v, h, t0);
    load_rows(dOf, p.dO, b, p.T, p.H_v, h, t0);
    if (tid < 32) {
      float gv[2], bv[2];
#pragma unroll
      for (int e2 = 0; e2 < 2; ++e2) {
        const int t = 2 * tid + e2;
        const size_t idx = ((size_t)b * p.T + t0 + t) * p.H_v + h;
        gv[e2] = t < nv ? p.g[idx] : 0.f;
        bv[e2] = t < nv ? p.beta[idx] : 0.f;
      }
      float run = gv[0] + gv[1];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float o = __shfl_up_sync(0xffffffffu, run, off);
        if (tid >= off) run += o;
      }
      const float GC = __shfl_sync(0xffffffffu, run, 31);
      G[2 * tid] = run - gv[1];
      G[2 * tid + 1] = run;
      gam[2 * tid] = expf(run - gv[1]);
      gam[2 * tid + 1] = expf(run);
      ee[2 * tid] = expf(GC - (run - gv[1]));
      ee[2 * tid + 1] = expf(GC - run);
      bb[2 * tid] = bv[0];
      bb[2 * tid + 1] = bv[1];
    }
    __syncthreads();
    // ---- forward quantities of the chunk, fp32 ----
    cta_mm(KK, kC, Kf, kD, false, Kf, kD, true, kC, kC, kD, 1.f, 0.f, sm);
    cta_mm(QK, kC, Qf, kD, false, Kf, kD, true, kC, kC, kD, 1.f, 0.f, sm);
    for (int i = tid; i < kSq; i += kBT) {  // D (lower with the diagonal; zero above), A_in, P
      const int r = i >> 6, cc = i & 63;
      const float d = cc <= r ? expf(G[r] - G[cc]) : 0.f;
      Dm[i] = d;
      Ash[r][cc] = cc < r ? bb[r] * d * KK[i] : 0.f;
      P[i] = d * QK[i];
    }
    __syncthreads();
    if (tid < kC) {  // column tid of (I + A_in)^-1 by forward substitution
      const int j = tid;
      for (int t = 0; t < kC; ++t) Tsh[t][j] = t == j ? 1.f : 0.f;
      for (int t = j + 1; t < kC; ++t) {
        float s = 0.f;
        for (int i = j; i < t; ++i) s = fmaf(Ash[t][i], Tsh[i][j], s);
        Tsh[t][j] = -s;
      }
    }
    __syncthreads();
    for (int i = tid; i < kSq; i += kBT) Tm[i] = Tsh[i >> 6][i & 63];
    for (int i = tid; i < kMat; i += kBT) {
      const int t = i >> 7;
      RW[i] = bb[t] * gam[t] * Kf[i];
      RU[i] = bb[t] * Vf[i];
    }
    __syncthreads();
    cta_mm(W, kD, Tm, kC, false, RW, kD, false, kC, kD, kC, 1.f, 0.f, sm);
    cta_mm(Up, kD, Tm, kC, false, RU, kD, false, kC, kD, kC, 1.f, 0.f, sm);
    // ---- cotangents of the chunk's maps ----
    cta_mm(dA, kD, ST, kD, false, dS, kD, false, kD, kD, kD, 1.f, 0.f, sm);         // S_c^T dS_{c+1}
    cta_mm(dQt, kD, dOf, kD, false, ST, kD, true, kC, kD, kD, p.scale, 0.f, sm);     // scale dO S_c
    cta_mm(dP, kC, dOf, kD, false, Up, kD, true, kC, kC, kD, p.scale, 0.f, sm);      // scale dO U'^T
    cta_mm(dUp, kD, P, kC, true, dOf, kD, false, kC, kD, kC, p.scale, 0.f, sm);      // scale P^T dO
    // ---- B = U'^T diag(e) K ----
    cta_mm(T1, kD, Up, kD, false, dS, kD, false, kC, kD, kD, 1.f, 0.f, sm);          // U' dB
    cta_mm(T2, kD, Kf, kD, false, dS, kD, true, kC, kD, kD, 1.f, 0.f, sm);           // K dB^T
    for (int i = tid; i < kMat; i += kBT) {
      const int t = i >> 7;
      dK[i] = ee[t] * T1[i];
      dUp[i] += ee[t] * T2[i];
    }
    if (tid < kC) {
      float s = 0.f;
      for (int j = 0; j < kD; ++j) s = fmaf(T1[tid * kD + j], Kf[tid * kD + j], s);
      de[tid] = s;
    }
    __syncthreads();
    // ---- A = gamma_C I - W^T diag(e) K ----
    cta_mm(T1, kD, W, kD, false, dA, kD, false, kC, kD, kD, 1.f, 0.f, sm);           // W dA
    cta_mm(T2, kD, Kf, kD, false, dA, kD, true, kC, kD, kD, 1.f, 0.f, sm);           // K dA^T
    for (int i = tid; i < kMat; i += kBT) {
      const int t = i >> 7;
      dK[i] -= ee[t] * T1[i];
      dW[i] = -ee[t] * T2[i];
      dQ[i] = gam[t] * dQt[i];  // Qt = diag(gamma) Q - P W: the gamma Q part
    }
    if (tid < kC) {
      float s = 0.f, s2 = 0.f;
      for (int j = 0; j < kD; ++j) {
        s = fmaf(T1[tid * kD + j], Kf[tid * kD + j], s);
        s2 = fmaf(dQt[tid * kD + j], Qf[tid * kD + j], s2);
      }
      de[tid] -= s;
      dgam[tid] = s2;
    }
    if (tid == kC) {
      float tr = 0.f;
      for (int j = 0; j < kD; ++j) tr += dA[j * kD + j];
      red[0] = tr;  // d gamma_C
    }
    __syncthreads();
    // ---- Qt = diag(gamma) Q - P W ----
    cta_mm(dP, kC, dQt, kD, false, W, kD, true, kC, kC, kD, -1.f, 1.f, sm);          // dP -= dQt W^T
    cta_mm(dW, kD, P, kC, true, dQt, kD, false, kC, kD, kC, -1.f, 1.f, sm);          // dW -= P^T dQt
    // ---- P = tril(D o Q K^T) ----
    for (int i = tid; i < kSq; i += kBT) {
      const int r = i >> 6, cc = i & 63;
      const float dpm = cc <= r ? dP[i] : 0.f;
      dD[i] = dpm * QK[i];
      S1[i] = dpm * Dm[i];  // dQK
    }
    __syncthreads();
    cta_mm(dQ, kD, S1, kC, false, Kf, kD, false, kC, kD, kC, 1.f, 1.f, sm);          // dQ += dQK K
    cta_mm(dK, kD, S1, kC, true, Qf, kD, false, kC, kD, kC, 1.f, 1.f, sm);           // dK += dQK^T Q
    // ---- W = T diag(beta gamma) K, U' = T diag(beta) V ----
    cta_mm(dTm, kC, dW, kD, false, RW, kD, true, kC, kC, kD, 1.f, 0.f, sm);          // dW RW^T
    cta_mm(dTm, kC, dUp, kD, false, RU, kD, true, kC, kC, kD, 1.f, 1.f, sm);         // + dUp RU^T
    cta_mm(T1, kD, Tm, kC, true, dW, kD, false, kC, kD, kC, 1.f, 0.f, sm);           // dRW = T^T dW
    cta_mm(T2, kD, Tm, kC, true, dUp, kD, false, kC, kD, kC, 1.f, 0.f, sm);          // dRU = T^T dU'
    for (int i = tid; i < kMat; i += kBT) {
      const int t = i >> 7;
      dK[i] += bb[t] * gam[t] * T1[i];
      dV[i] = bb[t] * T2[i];
    }
    if (tid < kC) {
      float sw = 0.f, su = 0.f;
      for (int j = 0; j < kD; ++j) {
        sw = fmaf(T1[tid * kD + j], Kf[tid * kD + j], sw);
        su = fmaf(T2[tid * kD + j], Vf[tid * kD + j], su);
      }
      dbeta[tid] = gam[tid] * sw + su;
      dgam[tid] += bb[tid] * sw;
    }
    __syncthreads();
    // ---- T = (I + A_in)^-1: dA_in = strict_tril(-T^T dT T^T) ----
    cta_mm(S1, kC, Tm, kC, true, dTm, kC, false, kC, kC, kC, 1.f, 0.f, sm);          // T^T dT
    cta_mm(S2, kC, S1, kC, false, Tm, kC, true, kC, kC, kC, -1.f, 0.f, sm);          // -(T^T dT) T^T
    // ---- A_in = strict_tril(beta_i D_ij K K^T_ij) ----
    for (int i = tid; i < kSq; i += kBT) {
      const int r = i >> 6, cc = i & 63;
      const float dain = cc < r ? S2[i] : 0.f;
      S1[i] = bb[r] * dain * Dm[i];  // dKK
      dD[i] += bb[r] * dain * KK[i];
      S2[i] = dain * Dm[i] * KK[i];  // for d beta
    }
    __syncthreads();
    if (tid < kC) {
      float s = 0.f;
      for (int j = 0; j < kC; ++j) s += S2[tid * kC + j];
      dbeta[tid] += s;
    }
    cta_mm(dK, kD, S1, kC, false, Kf, kD, false, kC, kD, kC, 1.f, 1.f, sm);          // dK += dKK K
    cta_mm(dK, kD, S1, kC, true, Kf, kD, false, kC, kD, kC, 1.f, 1.f, sm);           // dK += dKK^T K
    // ---- D_ij = exp(G_i - G_j), gamma = exp(G), e = exp(G_C - G), gamma_C = exp(G_C), G = cumsum(g) ----
    if (tid < kC) {
      float rs = 0.f, cs = 0.f;
      for (int j = 0; j < kC; ++j) {
        rs += dD[tid * kC + j] * Dm[tid * kC + j];
        cs += dD[j * kC + tid] * Dm[j * kC + tid];
      }
      dG[tid] = rs - cs + dgam[tid] * gam[tid] - de[tid] * ee[tid];
    }
    __syncthreads();
    if (tid == 0) {
      float s = 0.f;
      for (int j = 0; j < kC; ++j) s += de[j] * ee[j];
      dG[kC - 1] += s + red[0] * expf(G[kC - 1]);
      float run = 0.f;  // dg_t = sum_{u >= t} dG_u
      for (int t = kC - 1; t >= 0; --t) {
        run += dG[t];
        dG[t] = run;
      }
    }
    __syncthreads();
    // ---- outputs (the q/k gradients of the value heads sharing a q/k head accumulate) ----
    for (int i = tid; i < nv * kD; i += kBT) {
      const int t = i >> 7, j = i & 127;
      const size_t rq = (((size_t)b * p.T + t0 + t) * p.H_qk + qh) * kD + j;
      atomicAdd(p.dq + rq, dQ[i]);
      atomicAdd(p.dk + rq, dK[i]);
      p.dv[(((size_t)b * p.T + t0 + t) * p.H_v + h) * kD + j] = dV[i];
    }
    if (tid < nv) {
      const size_t idx = ((size_t)b * p.T + t0 + tid) * p.H_v + h;
      p.dg[idx] = dG[tid];
      p.dbeta[idx] = dbeta[tid];
    }
    __syncthreads();
  }
}

}  // namespace

size_t gdn_bwd_chunk_ctas(int B, int T, int H_v) {
  const size_t n_chunks = ((size_t)T + kC - 1) / kC;
  const size_t items = (size_t)B * H_v * n_chunks;
  return items < 296 ? items : 296;
}

size_t gdn_bwd_workspace_bytes(int B, int T, int H_v) {
  const size_t n_chunks = ((size_t)T + kC - 1) / kC;
  const size_t heads = (size_t)B * H_v;
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  return al(gdn_workspace_bytes(B, T, H_v)) + al((size_t)B * T * H_v * kD * 2) +       // records, forward o
         2 * al(heads * n_chunks * kD * kD * 4) +                                        // chunk states, dS
         al(heads * 2 * 3 * kC * kD * 4) + al(gdn_bwd_chunk_ctas(B, T, H_v) * kChunkScratch * 4);
}

cudaError_t launch_gdn_bwd(const GdnBwdArgs &a, cudaStream_t s) {
  const int n_chunks = (a.T + kC - 1) / kC;
  const size_t heads = (size_t)a.B * a.H_v;
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  uint8_t *w = reinterpret_cast<uint8_t *>(a.workspace);
  uint8_t *rec = w;
  w += al(gdn_workspace_bytes(a.B, a.T, a.H_v));
  bf16_t *o_fwd = reinterpret_cast<bf16_t *>(w);
  w += al((size_t)a.B * a.T * a.H_v * kD * 2);
  float *states = reinterpret_cast<float *>(w);
  w += al(heads * n_chunks * kD * kD * 4);
  float *dS = reinterpret_cast<float *>(w);
  w += al(heads * n_chunks * kD * kD * 4);
  float *scan_scratch = reinterpret_cast<float *>(w);
  w += al(heads * 2 * 3 * kC * kD * 4);
  float *chunk_scratch = reinterpret_cast<float *>(w);

  // 1. the forward pass, keeping every chunk's start state
  GdnChunkArgs f;
  memset(&f, 0, sizeof(f));
  f.q = a.q;
  f.k = a.k;
  f.v = a.v;
  f.g = a.g;
  f.beta = a.beta;
  f.state_in = a.state_in;
  f.o = o_fwd;
  f.B = a.B;
  f.T = a.T;
  f.n_heads = a.H_v;
  f.group = a.H_v / a.H_qk;
  f.qk_heads = a.H_qk;
  f.v_heads = a.H_v;
  f.scale = a.scale;
  f.workspace = rec;
  f.chunk_states = states;
  cudaError_t e = launch_gdn_chunk(f, s);
  if (e != cudaSuccess) return e;
  // the record layout of gdn_chunk.cu: -W_e^T | U'^T | P | Qt^T | factors
  const size_t nrec = heads * n_chunks;
  BwdParams p;
  memset(&p, 0, sizeof(p));
  p.q = a.q;
  p.k = a.k;
  p.v = a.v;
  p.dO = a.dO;
  p.g = a.g;
  p.beta = a.beta;
  p.dS_T = a.dS_T;
  p.chunk_states = states;
  p.rec_w = reinterpret_cast<const bf16_t *>(rec);
  p.rec_q = reinterpret_cast<const bf16_t *>(rec + nrec * (2 * kD * kC * 2 + kC * kC * 2));
  p.rec_f = reinterpret_cast<const float *>(rec + nrec * (3 * kD * kC * 2 + kC * kC * 2));
  p.dS = dS;
  p.dq = a.dq;
  p.dk = a.dk;
  p.dv = a.dv;
  p.dg = a.dg;
  p.dbeta = a.dbeta;
  p.dS0 = a.dS0;
  p.scan_scratch = scan_scratch;
  p.chunk_scratch = chunk_scratch;
  p.B = a.B;
  p.T = a.T;
  p.H_qk = a.H_qk;
  p.H_v = a.H_v;
  p.group = a.H_v / a.H_qk;
  p.n_chunks = n_chunks;
  p.n_items = (int)nrec;
  p.scale = a.scale;
  // 2. the reverse scan of the state's cotangent
  gdn_bwd_scan_kernel<<<dim3(a.H_v, a.B, 2), kBT, 0, s>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // 3. the per-chunk pullback; q and k gradients accumulate over the value heads of a q/k head
  if ((e = cudaMemsetAsync(a.dq, 0, (size_t)a.B * a.T * a.H_qk * kD * 4, s)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(a.dk, 0, (size_t)a.B * a.T * a.H_qk * kD * 4, s)) != cudaSuccess) return e;
  gdn_bwd_chunk_kernel<<<(unsigned)gdn_bwd_chunk_ctas(a.B, a.T, a.H_v), kBT, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace hh
