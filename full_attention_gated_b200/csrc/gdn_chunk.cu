// gdn_chunk.cu -- chunked gated delta rule over a sequence (prefill).
//
// The Gated DeltaNet layers keep one fixed-size state per value head ("The
// Hybrid Attention in Qwen3.8-27B", "Why 27B parameters can carry 262K
// tokens"; "The economics of hybrid attention", TL;DR).  The recurrence, per
// value head with S a d_v x d_k fp32 matrix,
//     S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
//     o_t = scale S_t q_t,
// is evaluated C = 64 tokens at a time.  Inside a chunk, with G the in-chunk
// cumulative sum of g and gamma = exp(G):
//     A_ti = beta_t exp(G_t - G_i) k_t.k_i   (i < t),   T = (I + A)^-1
//     W  = T diag(beta gamma) K,   U' = T diag(beta) V           (state-free)
//     P_ti = exp(G_t - G_i) q_t.k_i          (i <= t)
//     U  = U' - W S^T
//     O  = scale (diag(gamma) Q S^T + P U)
//     S <- gamma_C S + (diag(exp(G_C - G)) U)^T K
// (A derivation of these identities from the recurrence is checked on the CPU
// against the token-by-token oracle.)  The state never leaves the CTA between
// chunks: the fp32 master lives in MMA accumulator registers, a bf16 copy in
// shared memory feeds the tensor cores.
//
// CTA = (sequence, value head, d_v slice).  State rows evolve independently
// (row j of S only needs row j), so d_v may be split over 2 CTAs.  A producer
// warp streams q, k (shared by the group of value heads) and the v slice with
// TMA into a 2-stage ring; 8 consumer warps run the chunk: warp-level bf16 MMAs
// with fp32 accumulation for every product, a blocked fp32 triangular inverse
// (16 x 16 diagonal blocks by forward substitution, off-diagonal blocks by
// products), and the per-head RMS fusion when the hybrid layer asks for it.
// A last partial chunk is padded with k = 0, beta = 0, g = 0 tokens, which
// leave the state untouched and whose outputs are not written.
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"

namespace hh {

namespace {

constexpr int kC = 64;       // chunk length
constexpr int kDK = 128;     // key dim
constexpr int kCW = 8;       // consumer warps
constexpr int kGThreads = (kCW + 1) * 32;
constexpr int kCT = kCW * 32;  // consumer threads

struct GdnParams {
  CUtensorMap tm_q, tm_k, tm_v;  // 4-D (d, heads, T, B), box (64, 1, 64, 1), 128B swizzle
  const float *g, *beta;
  const float *state_in;
  float *state_out;
  bf16_t *o;
  int B, T, n_heads, group, qk_heads, v_heads, n_slices;
  int use_map;
  int map[kMaxMappedHeads];
  float scale;
  int rms;
  float eps;
  unsigned *status;
};

// Boxed 128-byte-swizzled bf16 matrix [R][cols]: cols/64 boxes of R rows x 128 B
// (the layout a TMA SWIZZLE_128B load of 64-column boxes produces).
__device__ __forceinline__ uint32_t boxed(int R, int r, int c) {
  return (uint32_t)(c >> 6) * (uint32_t)R * 128u + sw128(r, (c & 63) >> 3) + (uint32_t)(c & 7) * 2u;
}

template <int DV>
struct GdnSmem {
  static constexpr int kQK = kC * kDK * 2;         // 16 KiB
  static constexpr int kV = kC * DV * 2;
  static constexpr int kStage = 2 * kQK + kV;
  static constexpr int kRing = 2 * kStage;
  static constexpr int kR1 = kC * kDK * 2;         // Af fp32 [64][64] | -W bf16 [64][128]
  static constexpr int kR2 = kC * 64 * 4;          // Tf fp32 [64][64] | U bf16 [64][DV]
  static constexpr int kR3 = kC * 64 * 4;          // Yf fp32 | Uhat bf16 [64][DV]
  static constexpr int kT = kC * kC * 2;           // one bf16 [64][64]
  static constexpr int kS = DV * kDK * 2;          // bf16 state copy
  static constexpr int oR1 = kRing, oR2 = oR1 + kR1, oR3 = oR2 + kR2;
  static constexpr int oTbg = oR3 + kR3, oTb = oTbg + kT, oP = oTb + kT, oS = oP + kT;
  static constexpr int oSmall = oS + kS;
  // small: G[64], beta[64], gamma[64], rss[64][2], barriers
  static constexpr int kSmall = 64 * 4 * 3 + 64 * 2 * 4 + 8 * 8;
  static constexpr int kTotal = oSmall + kSmall + 1024;
  static_assert(kC * DV * 2 <= kR2 && kC * DV * 2 <= kR3, "U buffers fit");
};

__device__ __forceinline__ void cbar() { asm volatile("bar.sync 1, %0;\n" ::"n"(kCT) : "memory"); }
// consumer barrier that also counts the threads whose predicate is true
__device__ __forceinline__ int cbar_count(bool pred) {
  int r;
  asm volatile("{\n .reg .pred p;\n setp.ne.u32 p, %1, 0;\n bar.red.popc.u32 %0, 1, %2, p;\n}\n"
               : "=r"(r)
               : "r"((int)pred), "n"(kCT)
               : "memory");
  return r;
}

template <int DV>
__global__ void __launch_bounds__(kGThreads, 1) gdn_chunk_kernel(const __grid_constant__ GdnParams p) {
  using L = GdnSmem<DV>;
  constexpr int UN = DV / 16;                 // n-tiles of a [16 x DV/2] output half
  constexpr int SN = DV == 128 ? 16 : 8;      // n-tiles of this warp's share of S
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float *Af = reinterpret_cast<float *>(sm + L::oR1);
  float *Tf = reinterpret_cast<float *>(sm + L::oR2);
  float *Yf = reinterpret_cast<float *>(sm + L::oR3);
  const uint32_t ring_u = smem_u32(sm), Wb = smem_u32(sm + L::oR1), Ub = smem_u32(sm + L::oR2),
                 Uh = smem_u32(sm + L::oR3), Tbg = smem_u32(sm + L::oTbg), Tb = smem_u32(sm + L::oTb),
                 Pb = smem_u32(sm + L::oP), Sb = smem_u32(sm + L::oS);
  uint8_t *Wp = sm + L::oR1, *Up = sm + L::oR2, *Uhp = sm + L::oR3, *Tbgp = sm + L::oTbg, *Tbp = sm + L::oTb,
          *Pp = sm + L::oP, *Sp = sm + L::oS;
  float *Gs = reinterpret_cast<float *>(sm + L::oSmall);
  float *Bs = Gs + 64, *Eg = Bs + 64, *rss = Eg + 64;
  uint64_t *full = reinterpret_cast<uint64_t *>(rss + 128);
  uint64_t *empty = full + 2;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slice = blockIdx.x % p.n_slices, hi = blockIdx.x / p.n_slices, b = blockIdx.y;
  const int vh = p.use_map ? p.map[hi] : hi;
  const int qh = p.use_map ? p.map[hi] : hi / p.group;
  const int dv0 = slice * DV;
  const int n_chunks = (p.T + kC - 1) / kC;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCW);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kCW) {
    // ---------------- producer: q, k (group head) and the v slice of each chunk ----------------
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      for (int c = 0; c < n_chunks; ++c) {
        const int s = c & 1;
        if (c >= 2 && !mbar_wait(&empty[s], ((c >> 1) - 1) & 1, p.status)) break;
        mbar_arrive_expect_tx(&full[s], L::kStage);
        const uint32_t dq = ring_u + s * L::kStage, dk = dq + L::kQK, dvv = dk + L::kQK;
        for (int bx = 0; bx < 2; ++bx) {
          tma_load_4d(dq + bx * 8192, &p.tm_q, &full[s], bx * 64, qh, c * kC, b);
          tma_load_4d(dk + bx * 8192, &p.tm_k, &full[s], bx * 64, qh, c * kC, b);
        }
        for (int bx = 0; bx < DV / 64; ++bx) tma_load_4d(dvv + bx * 8192, &p.tm_v, &full[s], dv0 + bx * 64, vh, c * kC, b);
      }
    }
    return;
  }

  // ---------------- consumers ----------------
  const int ct = threadIdx.x;
  const int mt = warp & 3, nh = warp >> 2;  // token-row tile, column half
  const int s_m = DV == 128 ? warp : (warp & 3);
  const int s_n0 = DV == 128 ? 0 : (warp >> 2) * 8;
  const int arow = mt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;  // A-operand ldmatrix row
  const int r_lo = mt * 16 + (lane >> 2);                         // accumulator rows r_lo, r_lo + 8
  const size_t st_base = ((size_t)b * p.v_heads + vh) * kDK * kDK;

  // fp32 state master in accumulator fragments: rows 16*s_m + lane/4 (+8), cols (s_n0+j)*8 + 2*(lane%4) (+1)
  float Sacc[SN][4];
#pragma unroll
  for (int j = 0; j < SN; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int r = dv0 + s_m * 16 + (lane >> 2) + (e >> 1) * 8;
      const int c = (s_n0 + j) * 8 + (lane & 3) * 2 + (e & 1);
      Sacc[j][e] = p.state_in ? p.state_in[st_base + (size_t)r * kDK + c] : 0.f;
    }
#pragma unroll
  for (int j = 0; j < SN; ++j) {
    const int r = s_m * 16 + (lane >> 2), c = (s_n0 + j) * 8 + (lane & 3) * 2;
    *reinterpret_cast<uint32_t *>(Sp + boxed(DV, r, c)) = pack_bf16(Sacc[j][0], Sacc[j][1]);
    *reinterpret_cast<uint32_t *>(Sp + boxed(DV, r + 8, c)) = pack_bf16(Sacc[j][2], Sacc[j][3]);
  }

  bool ok = true;
  for (int c = 0; c < n_chunks; ++c) {
    const int s = c & 1;
    const int t0 = c * kC;
    const int nvalid = min(kC, p.T - t0);
    // ---- step 0: gates of the chunk, in-chunk cumulative log-decay G ----
    if (warp == 0) {
      float gv[2], bv[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int t = 2 * lane + e;
        const size_t idx = ((size_t)b * p.T + t0 + t) * p.v_heads + vh;
        gv[e] = t < nvalid ? p.g[idx] : 0.f;
        bv[e] = t < nvalid ? p.beta[idx] : 0.f;
      }
      float run = gv[0] + gv[1];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float n = __shfl_up_sync(0xffffffffu, run, off);
        if (lane >= off) run += n;
      }
      Gs[2 * lane + 1] = run;
      Gs[2 * lane] = run - gv[1];
      Eg[2 * lane + 1] = expf(run);
      Eg[2 * lane] = expf(run - gv[1]);
      Bs[2 * lane] = bv[0];
      Bs[2 * lane + 1] = bv[1];
    }
    const bool waited = mbar_wait(&full[s], (c >> 1) & 1, p.status);
    if (cbar_count(!waited) != 0) {  // CTA-uniform decision
      ok = false;
      break;
    }
    const uint32_t qb = ring_u + s * L::kStage, kb = qb + L::kQK, vb = kb + L::kQK;

    // ---- step 1: K K^T and Q K^T -> A (fp32), P (bf16), decay-masked ----
    {
      float kk[4][4], qk[4][4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) kk[j][e] = qk[j][e] = 0.f;
      if (nh * 32 <= mt * 16 + 15) {
#pragma unroll
        for (int ks = 0; ks < kDK / 16; ++ks) {
          uint32_t ak[4], aq[4];
          const uint32_t off = (ks >> 2) * 8192 + sw128(arow, (ks & 3) * 2 + (lane >> 4));
          ldsm_x4(kb + off, ak[0], ak[1], ak[2], ak[3]);
          ldsm_x4(qb + off, aq[0], aq[1], aq[2], aq[3]);
#pragma unroll
          for (int nj = 0; nj < 2; ++nj) {
            uint32_t b0, b1, b2, b3;
            const int krow = nh * 32 + nj * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
            ldsm_x4(kb + (ks >> 2) * 8192 + sw128(krow, (ks & 3) * 2 + ((lane >> 3) & 1)), b0, b1, b2, b3);
            mma_bf16_16816(kk[2 * nj], ak, b0, b1);
            mma_bf16_16816(kk[2 * nj + 1], ak, b2, b3);
            mma_bf16_16816(qk[2 * nj], aq, b0, b1);
            mma_bf16_16816(qk[2 * nj + 1], aq, b2, b3);
          }
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int t = r_lo + (e >> 1) * 8;
          const int i = nh * 32 + j * 8 + (lane & 3) * 2 + (e & 1);
          const float dec = i <= t ? expf(Gs[t] - Gs[i]) : 0.f;
          Af[t * 64 + i] = i < t ? Bs[t] * dec * kk[j][e] : 0.f;
          *reinterpret_cast<uint16_t *>(Pp + boxed(64, t, i)) = f_to_bf16(dec * qk[j][e]);
        }
    }
    cbar();

    // ---- step 2: T = (I + A)^-1, blocked: 16x16 diagonal blocks, then off-diagonal levels ----
    if (ct < 64) {
      const int I = ct >> 4, cc = ct & 15;
      const float *Ab = Af + (16 * I) * 64 + 16 * I;
      float x[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < r; ++j) acc = fmaf(Ab[r * 64 + j], x[j], acc);
        x[r] = r < cc ? 0.f : (r == cc ? 1.f : -acc);
      }
#pragma unroll
      for (int r = 0; r < 16; ++r) Tf[(16 * I + r) * 64 + 16 * I + cc] = x[r];
    }
    cbar();
    for (int lev = 1; lev <= 3; ++lev) {
      const int nel = (4 - lev) * 256;
      for (int e = ct; e < nel; e += kCT) {
        const int blk = e >> 8, r = (e >> 4) & 15, cc = e & 15, I = lev + blk, J = I - lev;
        float y = 0.f;
        for (int K = J; K < I; ++K)
#pragma unroll
          for (int j = 0; j < 16; ++j) y = fmaf(Af[(16 * I + r) * 64 + 16 * K + j], Tf[(16 * K + j) * 64 + 16 * J + cc], y);
        Yf[e] = y;
      }
      cbar();
      for (int e = ct; e < nel; e += kCT) {
        const int blk = e >> 8, r = (e >> 4) & 15, cc = e & 15, I = lev + blk, J = I - lev;
        float t = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) t = fmaf(Tf[(16 * I + r) * 64 + 16 * I + j], Yf[(blk * 16 + j) * 16 + cc], t);
        Tf[(16 * I + r) * 64 + 16 * J + cc] = -t;
      }
      cbar();
    }
    for (int e = ct; e < 64 * 64; e += kCT) {
      const int t = e >> 6, i = e & 63;
      const float tv = i <= t ? Tf[t * 64 + i] : 0.f;
      const float tb = tv * Bs[i];
      *reinterpret_cast<uint16_t *>(Tbgp + boxed(64, t, i)) = f_to_bf16(tb * Eg[i]);
      *reinterpret_cast<uint16_t *>(Tbp + boxed(64, t, i)) = f_to_bf16(tb);
    }
    cbar();
    // ---- step 3: -W = -T diag(beta gamma) K  (smem, bf16),  U' = T diag(beta) V  (registers) ----
    float u[UN][4];
    {
      float w[8][4];
#pragma unroll
      for (int j = 0; j < 8; ++j) w[j][0] = w[j][1] = w[j][2] = w[j][3] = 0.f;
#pragma unroll
      for (int j = 0; j < UN; ++j) u[j][0] = u[j][1] = u[j][2] = u[j][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        if (kk > mt) break;  // T is lower triangular
        uint32_t a[4], at[4];
        ldsm_x4(Tbg + sw128(arow, kk * 2 + (lane >> 4)), a[0], a[1], a[2], a[3]);
        ldsm_x4(Tb + sw128(arow, kk * 2 + (lane >> 4)), at[0], at[1], at[2], at[3]);
        const int vkey = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int nd = 0; nd < 4; ++nd) {
          uint32_t b0, b1, b2, b3;
          const int dcol = nh * 64 + nd * 16 + ((lane >> 4) & 1) * 8;
          ldsm_x4_t(kb + (dcol >> 6) * 8192 + sw128(vkey, (dcol & 63) >> 3), b0, b1, b2, b3);
          mma_bf16_16816(w[2 * nd], a, b0, b1);
          mma_bf16_16816(w[2 * nd + 1], a, b2, b3);
        }
#pragma unroll
        for (int nd = 0; nd < UN / 2; ++nd) {
          uint32_t b0, b1, b2, b3;
          const int dcol = nh * (DV / 2) + nd * 16 + ((lane >> 4) & 1) * 8;
          ldsm_x4_t(vb + (dcol >> 6) * 8192 + sw128(vkey, (dcol & 63) >> 3), b0, b1, b2, b3);
          mma_bf16_16816(u[2 * nd], at, b0, b1);
          mma_bf16_16816(u[2 * nd + 1], at, b2, b3);
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int col = nh * 64 + j * 8 + (lane & 3) * 2;
        *reinterpret_cast<uint32_t *>(Wp + boxed(64, r_lo, col)) = pack_bf16(-w[j][0], -w[j][1]);
        *reinterpret_cast<uint32_t *>(Wp + boxed(64, r_lo + 8, col)) = pack_bf16(-w[j][2], -w[j][3]);
      }
    }
    cbar();

    // ---- step 4: U = U' - W S^T  -> U and diag(exp(G_C - G)) U in smem (bf16) ----
#pragma unroll
    for (int ks = 0; ks < kDK / 16; ++ks) {
      uint32_t a[4];
      ldsm_x4(Wb + (ks >> 2) * 8192 + sw128(arow, (ks & 3) * 2 + (lane >> 4)), a[0], a[1], a[2], a[3]);
#pragma unroll
      for (int nd = 0; nd < UN / 2; ++nd) {
        uint32_t b0, b1, b2, b3;
        const int srow = nh * (DV / 2) + nd * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
        ldsm_x4(Sb + (ks >> 2) * (DV * 128) + sw128(srow, (ks & 3) * 2 + ((lane >> 3) & 1)), b0, b1, b2, b3);
        mma_bf16_16816(u[2 * nd], a, b0, b1);
        mma_bf16_16816(u[2 * nd + 1], a, b2, b3);
      }
    }
    {
      const float GC = Gs[63];
      const float f0 = expf(GC - Gs[r_lo]), f1 = expf(GC - Gs[r_lo + 8]);
#pragma unroll
      for (int j = 0; j < UN; ++j) {
        const int col = nh * (DV / 2) + j * 8 + (lane & 3) * 2;
        *reinterpret_cast<uint32_t *>(Up + boxed(64, r_lo, col)) = pack_bf16(u[j][0], u[j][1]);
        *reinterpret_cast<uint32_t *>(Up + boxed(64, r_lo + 8, col)) = pack_bf16(u[j][2], u[j][3]);
        *reinterpret_cast<uint32_t *>(Uhp + boxed(64, r_lo, col)) = pack_bf16(f0 * u[j][0], f0 * u[j][1]);
        *reinterpret_cast<uint32_t *>(Uhp + boxed(64, r_lo + 8, col)) = pack_bf16(f1 * u[j][2], f1 * u[j][3]);
      }
    }
    cbar();

    // ---- step 5a: O = scale (diag(gamma) Q S^T + P U) ----
    {
      float oa[UN][4];
#pragma unroll
      for (int j = 0; j < UN; ++j) oa[j][0] = oa[j][1] = oa[j][2] = oa[j][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < kDK / 16; ++ks) {
        uint32_t a[4];
        ldsm_x4(qb + (ks >> 2) * 8192 + sw128(arow, (ks & 3) * 2 + (lane >> 4)), a[0], a[1], a[2], a[3]);
#pragma unroll
        for (int nd = 0; nd < UN / 2; ++nd) {
          uint32_t b0, b1, b2, b3;
          const int srow = nh * (DV / 2) + nd * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
          ldsm_x4(Sb + (ks >> 2) * (DV * 128) + sw128(srow, (ks & 3) * 2 + ((lane >> 3) & 1)), b0, b1, b2, b3);
          mma_bf16_16816(oa[2 * nd], a, b0, b1);
          mma_bf16_16816(oa[2 * nd + 1], a, b2, b3);
        }
      }
      const float e0 = Eg[r_lo], e1 = Eg[r_lo + 8];
#pragma unroll
      for (int j = 0; j < UN; ++j) {
        oa[j][0] *= e0;
        oa[j][1] *= e0;
        oa[j][2] *= e1;
        oa[j][3] *= e1;
      }
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        if (kk > mt) break;  // P is lower triangular
        uint32_t a[4];
        ldsm_x4(Pb + sw128(arow, kk * 2 + (lane >> 4)), a[0], a[1], a[2], a[3]);
        const int vkey = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int nd = 0; nd < UN / 2; ++nd) {
          uint32_t b0, b1, b2, b3;
          const int dcol = nh * (DV / 2) + nd * 16 + ((lane >> 4) & 1) * 8;
          ldsm_x4_t(Ub + (dcol >> 6) * 8192 + sw128(vkey, (dcol & 63) >> 3), b0, b1, b2, b3);
          mma_bf16_16816(oa[2 * nd], a, b0, b1);
          mma_bf16_16816(oa[2 * nd + 1], a, b2, b3);
        }
      }
      float rs0 = p.scale, rs1 = p.scale;
      if (p.rms) {  // uniform over the CTA; only used with DV == 128 (whole rows in this CTA)
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int j = 0; j < UN; ++j) {
          s0 += oa[j][0] * oa[j][0] + oa[j][1] * oa[j][1];
          s1 += oa[j][2] * oa[j][2] + oa[j][3] * oa[j][3];
        }
        s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
        s0 += __shfl_xor_sync(0xffffffffu, s0, 2);
        s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
        s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
        if ((lane & 3) == 0) {
          rss[r_lo * 2 + nh] = s0;
          rss[(r_lo + 8) * 2 + nh] = s1;
        }
        cbar();
        const float sc2 = p.scale * p.scale;
        rs0 = p.scale * rsqrtf(sc2 * (rss[r_lo * 2] + rss[r_lo * 2 + 1]) / (float)kDK + p.eps);
        rs1 = p.scale * rsqrtf(sc2 * (rss[(r_lo + 8) * 2] + rss[(r_lo + 8) * 2 + 1]) / (float)kDK + p.eps);
      }
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int t = r_lo + h2 * 8;
        if (t < nvalid) {
          const float rsv = h2 ? rs1 : rs0;
          bf16_t *dst = p.o + (((size_t)b * p.T + t0 + t) * p.v_heads + vh) * kDK + dv0 + nh * (DV / 2) + (lane & 3) * 2;
#pragma unroll
          for (int j = 0; j < UN; ++j)
            *reinterpret_cast<uint32_t *>(dst + j * 8) = pack_bf16(oa[j][2 * h2] * rsv, oa[j][2 * h2 + 1] * rsv);
        }
      }
    }

    // ---- step 5b: S <- gamma_C S + Uhat^T K  (fp32 master in registers) ----
    {
      const float gC = Eg[63];
#pragma unroll
      for (int j = 0; j < SN; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) Sacc[j][e] *= gC;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        uint32_t a[4];
        const int tok = kk * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
        const int dvc = s_m * 16 + ((lane >> 3) & 1) * 8;
        ldsm_x4_t(Uh + (dvc >> 6) * 8192 + sw128(tok, (dvc & 63) >> 3), a[0], a[1], a[2], a[3]);
        const int vkey = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int nd = 0; nd < SN / 2; ++nd) {
          uint32_t b0, b1, b2, b3;
          const int dcol = (s_n0 + 2 * nd) * 8 + ((lane >> 4) & 1) * 8;
          ldsm_x4_t(kb + (dcol >> 6) * 8192 + sw128(vkey, (dcol & 63) >> 3), b0, b1, b2, b3);
          mma_bf16_16816(Sacc[2 * nd], a, b0, b1);
          mma_bf16_16816(Sacc[2 * nd + 1], a, b2, b3);
        }
      }
    }
    // ---- step 6: release the ring stage, refresh the bf16 state copy ----
    cbar();
    if (lane == 0) mbar_arrive(&empty[s]);
#pragma unroll
    for (int j = 0; j < SN; ++j) {
      const int r = s_m * 16 + (lane >> 2), cc = (s_n0 + j) * 8 + (lane & 3) * 2;
      *reinterpret_cast<uint32_t *>(Sp + boxed(DV, r, cc)) = pack_bf16(Sacc[j][0], Sacc[j][1]);
      *reinterpret_cast<uint32_t *>(Sp + boxed(DV, r + 8, cc)) = pack_bf16(Sacc[j][2], Sacc[j][3]);
    }
  }
  if (p.state_out && ok) {
#pragma unroll
    for (int j = 0; j < SN; ++j)
#pragma unroll
      for (int e = 0; e < 4; e += 2) {
        const int r = dv0 + s_m * 16 + (lane >> 2) + (e >> 1) * 8;
        const int cc = (s_n0 + j) * 8 + (lane & 3) * 2;
        *reinterpret_cast<float2 *>(p.state_out + st_base + (size_t)r * kDK + cc) = make_float2(Sacc[j][e], Sacc[j][e + 1]);
      }
  }
}
}  // namespace
// T == 0: the state passes through unchanged
__global__ void gdn_state_copy_kernel(const float *__restrict__ in, float *__restrict__ out, int n_heads, int v_heads,
                                      int use_map, GdnChunkArgs a) {
  const int hi = blockIdx.x, b = blockIdx.y;
  const int vh = use_map ? a.map[hi] : hi;
  const size_t base = ((size_t)b * v_heads + vh) * kDK * kDK;
  for (int i = threadIdx.x; i < kDK * kDK; i += blockDim.x) out[base + i] = in ? in[base + i] : 0.f;
}

template <int DV>
cudaError_t launch_gdn_dv(const GdnParams &p, cudaStream_t s) {
  auto kern = gdn_chunk_kernel<DV>;
  const int smem = GdnSmem<DV>::kTotal;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.n_heads * p.n_slices, p.B);
  kern<<<grid, kGThreads, smem, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_gdn_chunk(const GdnChunkArgs &a, cudaStream_t s) {
  if (a.B == 0 || a.n_heads == 0) return cudaSuccess;
  if (a.T == 0) {
    if (!a.state_out) return cudaSuccess;
    gdn_state_copy_kernel<<<dim3(a.n_heads, a.B), 256, 0, s>>>(a.state_in, a.state_out, a.n_heads, a.v_heads,
                                                                 a.use_map, a);
    return cudaGetLastError();
  }
  GdnParams p;
  memset(&p, 0, sizeof(p));
  const uint32_t box[4] = {64, 1, (uint32_t)kC, 1};
  const uint64_t dq[4] = {(uint64_t)kDK, (uint64_t)a.qk_heads, (uint64_t)a.T, (uint64_t)a.B};
  const uint64_t sq[3] = {(uint64_t)kDK * 2, (uint64_t)a.qk_heads * kDK * 2, (uint64_t)a.T * a.qk_heads * kDK * 2};
  const uint64_t dv[4] = {(uint64_t)kDK, (uint64_t)a.v_heads, (uint64_t)a.T, (uint64_t)a.B};
  const uint64_t sv[3] = {(uint64_t)kDK * 2, (uint64_t)a.v_heads * kDK * 2, (uint64_t)a.T * a.v_heads * kDK * 2};
  if (encode_tmap(&p.tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.q, dq, sq, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
      encode_tmap(&p.tm_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.k, dq, sq, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
      encode_tmap(&p.tm_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.v, dv, sv, box, CU_TENSOR_MAP_SWIZZLE_128B)) {
    set_error("gdn_chunk_fwd: cuTensorMapEncodeTiled failed");
    return cudaErrorInvalidValue;
  }
  p.g = a.g;
  p.beta = a.beta;
  p.state_in = a.state_in;
  p.state_out = a.state_out;
  p.o = a.o;
  p.B = a.B;
  p.T = a.T;
  p.n_heads = a.n_heads;
  p.group = a.group;
  p.qk_heads = a.qk_heads;
  p.v_heads = a.v_heads;
  p.use_map = a.use_map;
  memcpy(p.map, a.map, sizeof(p.map));
  p.scale = a.scale;
  p.rms = a.rms;
  p.eps = a.eps;
  p.status = device_status_ptr();
  // Too few (sequence, head) chains to fill the GPU: split d_v over two CTAs.
  // The fused RMS needs whole rows, so the hybrid path keeps one CTA per head.
  const bool split = !a.rms && (long long)a.B * a.n_heads < 148;
  p.n_slices = split ? 2 : 1;
  return split ? launch_gdn_dv<64>(p, s) : launch_gdn_dv<128>(p, s);
}
}  // namespace hh
