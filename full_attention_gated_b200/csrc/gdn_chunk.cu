// gdn_chunk.cu -- chunked gated delta rule over a sequence (prefill).
//
// The Gated DeltaNet layers keep one fixed-size state per value head ("The
// Hybrid Attention in Qwen3.8-27B", "Why 27B parameters can carry 262K
// tokens"; "The economics of hybrid attention", TL;DR).  The recurrence, per
// value head with S a d_v x d_k fp32 matrix,
//     S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
//     o_t = scale S_t q_t,
// is evaluated C = 64 tokens at a time.  Inside a chunk, with G the in-chunk
// cumulative sum of g, gamma = exp(G) and e = exp(G_C - G):
//     A_ti = beta_t exp(G_t - G_i) k_t.k_i   (i < t),   T = (I + A)^-1
//     W  = T diag(beta gamma) K,   U' = T diag(beta) V
//     P_ti = exp(G_t - G_i) q_t.k_i          (i <= t)
//     O  = scale (Qt S^T + P U'),             Qt = diag(gamma) Q - P W
//     S <- gamma_C S - S M + B,               M = W^T diag(e) K,  B = U'^T diag(e) K
// The chunk update is affine in S because the scalar gates commute with the
// rank-one factors: the chunk's product of exp(g_t)(I - beta_t k_t k_t^T) is
// gamma_C (I - M / gamma_C).  (These identities are checked on the CPU against
// the token-by-token oracle.)
//
// Two kernels, so that only the state-dependent products sit on the
// sequential chain over chunks:
//   gdn_prep   parallel over (value head, chunk): K K^T, Q K^T, the blocked
//              triangular solve, -diag(e) W, U'^T, P, Qt and the decay factors,
//              written to a caller-provided workspace (bf16 matrices, fp32
//              factors), each record flagged once complete;
//   gdn_scan   one CTA per (sequence, value head) runs the chain on the 5th-
//              generation tensor cores with the fp32 state in tensor memory.
// When the scan's CTAs leave room, gdn_prep runs beside it on a second stream
// and the scan consumes each chunk's record as soon as its flag is set.  A last
// partial chunk is padded with k = 0, beta = 0, g = 0 tokens, which leave the
// state unchanged and whose outputs are not written.  The head-level hybrid
// layer's RMS fusion is a small row pass after the scan.
#include <math.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace hh {

namespace {

constexpr int kC = 64;    // chunk length
constexpr int kDK = 128;  // key (and value) dim

// workspace record per (sequence, value head, chunk)
constexpr size_t kWBytes = (size_t)kC * kDK * 2;  // -W_e = -diag(e) W [64][128] bf16
constexpr size_t kUBytes = (size_t)kC * kDK * 2;  // U'^T [128][64] bf16 (d_v rows, token columns)
constexpr size_t kPBytes = (size_t)kC * kC * 2;   // P    [64][64]  bf16
constexpr size_t kQBytes = (size_t)kC * kDK * 2;  // Qt = diag(gamma) Q - P W [64][128] bf16
constexpr size_t kFBytes = (size_t)2 * kC * 4;    // gamma[64], e = exp(G_C - G)[64] fp32

struct GdnWs {
  bf16_t *wn, *up, *pm, *qt;  // [B, Hn, n_chunks] x (-W_e | U'^T | P | Qt)
  float *fc;                  // [B, Hn, n_chunks, 2, 64]
  unsigned *flag;             // [B, Hn, n_chunks]: 1 once gdn_prep has written the record
};

GdnWs carve(void *ws, int B, int Hn, int n_chunks) {
  const size_t rec = (size_t)B * Hn * n_chunks;
  uint8_t *p = reinterpret_cast<uint8_t *>(ws);
  GdnWs w;
  w.wn = reinterpret_cast<bf16_t *>(p);
  w.up = reinterpret_cast<bf16_t *>(p + rec * kWBytes);
  w.pm = reinterpret_cast<bf16_t *>(p + rec * (kWBytes + kUBytes));
  w.qt = reinterpret_cast<bf16_t *>(p + rec * (kWBytes + kUBytes + kPBytes));
  w.fc = reinterpret_cast<float *>(p + rec * (kWBytes + kUBytes + kPBytes + kQBytes));
  w.flag = reinterpret_cast<unsigned *>(p + rec * (kWBytes + kUBytes + kPBytes + kQBytes + kFBytes));
  return w;
}

// Boxed 128-byte-swizzled bf16 matrix [R][cols]: cols/64 boxes of R rows x 128 B
// (the layout a TMA SWIZZLE_128B load of 64-column boxes produces).
__device__ __forceinline__ uint32_t boxed(int R, int r, int c) {
  return (uint32_t)(c >> 6) * (uint32_t)R * 128u + sw128(r, (c & 63) >> 3) + (uint32_t)(c & 7) * 2u;
}

template <int NT>
__device__ __forceinline__ void named_bar(int id) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "n"(NT) : "memory");
}
// barrier over NT threads that also counts the threads whose predicate is true
template <int NT>
__device__ __forceinline__ int named_bar_count(int id, bool pred) {
  int r;
  asm volatile("{\n .reg .pred p;\n setp.ne.u32 p, %2, 0;\n bar.red.popc.u32 %0, %1, %3, p;\n}\n"
               : "=r"(r)
               : "r"(id), "r"((int)pred), "n"(NT)
               : "memory");
  return r;
}

struct Heads {
  int n_heads, group, qk_heads, v_heads, use_map;
  int map[kMaxMappedHeads];
  __device__ __forceinline__ int vh(int i) const { return use_map ? map[i] : i; }
  __device__ __forceinline__ int qh(int i) const { return use_map ? map[i] : i / group; }
};

// ============================================================================
// gdn_prep: one CTA per (head, chunk, sequence), heads fastest so that the records of
// chunk c complete before those of chunk c + 1; 8 MMA warps, thread 0 issues TMA.
// W and U' come from a block forward substitution on (I + A) X = R with
// R = [diag(beta gamma) K | diag(beta) V] and 16-row blocks:
//     X_I = (I + A_II)^-1 (R_I - sum_{J<I} A_IJ X_J),   W = X[:, :128], U' = X[:, 128:]
// The four 16 x 16 diagonal inverses are formed in fp32 by forward substitution;
// every other product is a warp MMA (bf16 operands, fp32 accumulation).  Warp w
// owns columns 32w .. 32w+31 of X through all four block rows, so the solve
// needs no CTA-wide synchronisation and X overwrites its right-hand side in place.
// ============================================================================
constexpr int kPW = 8;            // warps
constexpr int kPT = kPW * 32;     // threads
constexpr int kPThreads = kPT;

struct PrepParams {
  CUtensorMap tm_q, tm_k, tm_v;         // 4-D (d, heads, T, B), box (64, 1, 64, 1)
  CUtensorMap tm_w, tm_u, tm_p, tm_qt;  // workspace records (TMA stores), as read by the scan
  const float *g, *beta;
  GdnWs ws;
  int B, T, n_chunks;
  Heads h;
  unsigned *status;
};

struct PrepSmem {
  // TMA tiles [64][128] bf16 (2 boxes each).  X = [W | U'] (4 boxes of 64 columns) is
  // solved in place over K | V; Qt is formed in place over Q, -W_e in place over W.
  static constexpr int oQ = 0, oK = 16384, oV = 32768, oX = oK;
  static constexpr int oUt = 49152;        // U'^T [128][64] bf16, staged for the TMA store (1 box)
  static constexpr int oP = oUt + 16384;   // P [64][64] bf16 (1 box): staged, and the A operand of Qt
  static constexpr int oAb = oP + 8192;    // -A off-diagonal blocks, bf16 [64][64] (1 box)
  static constexpr int oAd = oAb + 8192;   // A diagonal blocks fp32 [4][16][16]
  static constexpr int oTd = oAd + 4096;   // (I + A_II)^-1 fp32 [4][16][16]
  static constexpr int kYRow = 80;         // per-warp bf16 [16][32] scratch, rows padded to 80 bytes
  static constexpr int oY = oTd + 4096;
  static constexpr int oSmall = oY + kPW * 16 * kYRow;  // G, beta, gamma, e [64] each, barrier
  static constexpr int kTotal = oSmall + 4 * 256 + 16 + 1024;
};

__global__ void __launch_bounds__(kPThreads, 2) gdn_prep_kernel(const __grid_constant__ PrepParams p) {
  using L = PrepSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float *Ad = reinterpret_cast<float *>(sm + L::oAd);
  float *Td = reinterpret_cast<float *>(sm + L::oTd);
  float *Gs = reinterpret_cast<float *>(sm + L::oSmall);
  float *Bs = Gs + 64, *Eg = Bs + 64, *Ee = Eg + 64;
  uint64_t *full = reinterpret_cast<uint64_t *>(Ee + 64);
  const uint32_t qb = smem_u32(sm + L::oQ), kb = smem_u32(sm + L::oK), vb = smem_u32(sm + L::oV),
                 Xs = smem_u32(sm + L::oX), Abs = smem_u32(sm + L::oAb), Ps = smem_u32(sm + L::oP);
  uint8_t *Xp = sm + L::oX, *Abp = sm + L::oAb, *Pp = sm + L::oP;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hi = blockIdx.x, c = blockIdx.y, b = blockIdx.z;  // heads fastest: chunks complete in order
  const int vh = p.h.vh(hi), qh = p.h.qh(hi);
  const int t0 = c * kC, nvalid = min(kC, p.T - t0);
  const size_t rec = ((size_t)b * p.h.n_heads + hi) * p.n_chunks + c;

  if (threadIdx.x == 0) {
    mbar_init(full, 1);
    fence_barrier_init();
    mbar_arrive_expect_tx(full, 3 * 16384);
    for (int bx = 0; bx < 2; ++bx) {
      tma_load_4d(qb + bx * 8192, &p.tm_q, full, bx * 64, qh, t0, b);
      tma_load_4d(kb + bx * 8192, &p.tm_k, full, bx * 64, qh, t0, b);
      tma_load_4d(vb + bx * 8192, &p.tm_v, full, bx * 64, vh, t0, b);
    }
  }
  // gates -> G (in-chunk cumulative log decay), gamma = exp(G), beta; padded tokens: g = beta = 0
  if (warp == 0) {
    float gv[2], bv[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int t = 2 * lane + e;
      const size_t idx = ((size_t)b * p.T + t0 + t) * p.h.v_heads + vh;
      gv[e] = t < nvalid ? p.g[idx] : 0.f;
      bv[e] = t < nvalid ? p.beta[idx] : 0.f;
    }
    float run = gv[0] + gv[1];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float n = __shfl_up_sync(0xffffffffu, run, off);
      if (lane >= off) run += n;
    }
    const float g_lo = run - gv[1];
    Gs[2 * lane + 1] = run;
    Gs[2 * lane] = g_lo;
    Eg[2 * lane + 1] = expf(run);
    Eg[2 * lane] = expf(g_lo);
    Bs[2 * lane] = bv[0];
    Bs[2 * lane + 1] = bv[1];
    // decay factors for the scan: gamma_t and exp(G_C - G_t)
    const float GC = __shfl_sync(0xffffffffu, run, 31);
    Ee[2 * lane] = expf(GC - g_lo);
    Ee[2 * lane + 1] = expf(GC - run);
    p.ws.fc[rec * 128 + 2 * lane] = expf(g_lo);
    p.ws.fc[rec * 128 + 2 * lane + 1] = expf(run);
    p.ws.fc[rec * 128 + 64 + 2 * lane] = expf(GC - g_lo);
    p.ws.fc[rec * 128 + 64 + 2 * lane + 1] = expf(GC - run);
  }
  __syncthreads();
  const bool waited = mbar_wait(full, 0, p.status);
  if (__syncthreads_or(!waited)) {  // CTA-uniform
    if (threadIdx.x == 0) mbar_wait(full, 0, p.status);  // the loads it issued land before the CTA exits (bounded)
    return;
  }

  // ---- step 1: K K^T and Q K^T -> -A (off-diagonal bf16, diagonal fp32), P (bf16, workspace) ----
  {
    const int mt = warp & 3, nh = warp >> 2;  // rows 16*mt.., columns 32*nh..
    const int arow = mt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
    const int r_lo = mt * 16 + (lane >> 2);
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
      for (int h2 = 0; h2 < 2; ++h2) {
        const int t = r_lo + h2 * 8;
        const int i = nh * 32 + j * 8 + (lane & 3) * 2;
        const float d0 = i <= t ? expf(Gs[t] - Gs[i]) : 0.f;
        const float d1 = i + 1 <= t ? expf(Gs[t] - Gs[i + 1]) : 0.f;
        const float a0 = i < t ? Bs[t] * d0 * kk[j][2 * h2] : 0.f;
        const float a1 = i + 1 < t ? Bs[t] * d1 * kk[j][2 * h2 + 1] : 0.f;
        if ((i >> 4) == (t >> 4)) {  // diagonal 16 x 16 block: fp32 for the forward substitution
          float *ad = Ad + (t >> 4) * 256 + (t & 15) * 16 + (i & 15);
          ad[0] = a0;
          ad[1] = a1;
        }
        *reinterpret_cast<uint32_t *>(Abp + boxed(64, t, i)) = pack_bf16(-a0, -a1);
        *reinterpret_cast<uint32_t *>(Pp + boxed(64, t, i)) = pack_bf16(d0 * qk[j][2 * h2], d1 * qk[j][2 * h2 + 1]);
      }
  }
  tc::fence_proxy_async_smem();  // P is final; its TMA store is issued during step 2
  __syncthreads();
  // Each finished tile's TMA store is issued by thread 0 once its own share of the next
  // step is done (so that warp 0 does not hold up that step's barrier); all complete
  // before the record is flagged.
  const int wrow = (int)(rec * kC);  // first workspace row of this record

  // ---- step 2: the four diagonal inverses (I + A_II)^-1, fp32 forward substitution, one column
  // per thread (64 threads) ----
  if (threadIdx.x < 64) {
    const int I = threadIdx.x >> 4, cc = threadIdx.x & 15;
    const float *Ab = Ad + I * 256;
    float x[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      float acc = 0.f;
#pragma unroll
      for (int j = 0; j < r; ++j) acc = fmaf(Ab[r * 16 + j], x[j], acc);
      x[r] = r < cc ? 0.f : (r == cc ? 1.f : -acc);
    }
#pragma unroll
    for (int r = 0; r < 16; ++r) Td[I * 256 + r * 16 + cc] = x[r];
  }
  if (threadIdx.x == 0) {
    tma_store_2d(&p.tm_p, Ps, 0, wrow);
    bulk_commit();
  }
  __syncthreads();

  // ---- step 3: block forward substitution; warp w owns columns 32w .. 32w+31 of X ----
  {
    const bool is_w = warp < 4;                      // columns 0..127: W (from K), 128..255: U' (from V)
    const uint8_t *src = sm + (is_w ? L::oK : L::oV);
    const int cbase = (warp & 3) * 32;               // column inside the K or V tile
    const int xcol = warp * 32;                      // column inside X
    uint8_t *Yp = sm + L::oY + warp * 16 * L::kYRow;  // [16][32] bf16, padded rows
    const uint32_t Ys = smem_u32(Yp);
    const int g8 = lane >> 2, c2 = (lane & 3) * 2;
#pragma unroll 1
    for (int I = 0; I < 4; ++I) {
      float acc[4][4];
      // R_I: rows 16I + g8 (+8), columns c2 (+1) of each 8-column tile, scaled per row
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int t = 16 * I + g8 + 8 * h2;
        const float sc = is_w ? Bs[t] * Eg[t] : Bs[t];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
          const uint32_t v = *reinterpret_cast<const uint32_t *>(src + boxed(64, t, cbase + nt * 8 + c2));
          acc[nt][2 * h2] = sc * bf16_lo(v);
          acc[nt][2 * h2 + 1] = sc * bf16_hi(v);
        }
      }
      // - sum_{J<I} A_IJ X_J
#pragma unroll 1
      for (int J = 0; J < I; ++J) {
        uint32_t a[4];
        ldsm_x4(Abs + sw128(16 * I + (lane & 7) + ((lane >> 3) & 1) * 8, J * 2 + (lane >> 4)), a[0], a[1], a[2], a[3]);
        const int vkey = 16 * J + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int nd = 0; nd < 2; ++nd) {
          uint32_t b0, b1, b2, b3;
          const int dcol = xcol + nd * 16 + ((lane >> 4) & 1) * 8;
          ldsm_x4_t(Xs + (dcol >> 6) * 8192 + sw128(vkey, (dcol & 63) >> 3), b0, b1, b2, b3);
          mma_bf16_16816(acc[2 * nd], a, b0, b1);
          mma_bf16_16816(acc[2 * nd + 1], a, b2, b3);
        }
      }
      // Y_I -> bf16 scratch, then X_I = (I + A_II)^-1 Y_I
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        *reinterpret_cast<uint32_t *>(Yp + g8 * L::kYRow + (nt * 8 + c2) * 2) = pack_bf16(acc[nt][0], acc[nt][1]);
        *reinterpret_cast<uint32_t *>(Yp + (g8 + 8) * L::kYRow + (nt * 8 + c2) * 2) = pack_bf16(acc[nt][2], acc[nt][3]);
      }
      __syncwarp();
      uint32_t ta[4];
      {
        const float *Ti = Td + I * 256;
        ta[0] = pack_bf16(Ti[g8 * 16 + c2], Ti[g8 * 16 + c2 + 1]);
        ta[1] = pack_bf16(Ti[(g8 + 8) * 16 + c2], Ti[(g8 + 8) * 16 + c2 + 1]);
        ta[2] = pack_bf16(Ti[g8 * 16 + c2 + 8], Ti[g8 * 16 + c2 + 9]);
        ta[3] = pack_bf16(Ti[(g8 + 8) * 16 + c2 + 8], Ti[(g8 + 8) * 16 + c2 + 9]);
      }
      float xo[4][4];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) xo[nt][0] = xo[nt][1] = xo[nt][2] = xo[nt][3] = 0.f;
#pragma unroll
      for (int nd = 0; nd < 2; ++nd) {
        uint32_t b0, b1, b2, b3;
        const int yr = (lane & 7) + ((lane >> 3) & 1) * 8;
        const int ycol = nd * 16 + ((lane >> 4) & 1) * 8;
        ldsm_x4_t(Ys + yr * L::kYRow + ycol * 2, b0, b1, b2, b3);
        mma_bf16_16816(xo[2 * nd], ta, b0, b1);
        mma_bf16_16816(xo[2 * nd + 1], ta, b2, b3);
      }
      // X_I -> shared, in place over R_I (operand of later block rows; W also of Qt);
      // U'_I also -> the U'^T staging tile (row = value index, column = token)
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        const int col = nt * 8 + c2;
        *reinterpret_cast<uint32_t *>(Xp + boxed(64, 16 * I + g8, xcol + col)) = pack_bf16(xo[nt][0], xo[nt][1]);
        *reinterpret_cast<uint32_t *>(Xp + boxed(64, 16 * I + g8 + 8, xcol + col)) = pack_bf16(xo[nt][2], xo[nt][3]);
        if (!is_w) {
          const int v = cbase + col, t = 16 * I + g8;
          uint8_t *u0 = sm + L::oUt + v * 128 + (t & 7) * 2, *u1 = u0 + 128;
          *reinterpret_cast<bf16_t *>(u0 + (((t >> 3) ^ (v & 7)) << 4)) = f_to_bf16(xo[nt][0]);
          *reinterpret_cast<bf16_t *>(u1 + (((t >> 3) ^ ((v + 1) & 7)) << 4)) = f_to_bf16(xo[nt][1]);
          *reinterpret_cast<bf16_t *>(u0 + ((((t + 8) >> 3) ^ (v & 7)) << 4)) = f_to_bf16(xo[nt][2]);
          *reinterpret_cast<bf16_t *>(u1 + ((((t + 8) >> 3) ^ ((v + 1) & 7)) << 4)) = f_to_bf16(xo[nt][3]);
        }
      }
      __syncwarp();
    }
  }

  // ---- step 4: Qt = diag(gamma) Q - P W (the state-free part of the output map), in place over Q;
  // warp w owns columns 16w .. 16w+15 of Qt, all 64 rows.  P is lower triangular, so the
  // (row tile, key tile) products above the diagonal are skipped. ----
  tc::fence_proxy_async_smem();  // U'^T is final
  __syncthreads();
  {
    const int g8 = lane >> 2, c2 = (lane & 3) * 2;
    const int kcol = warp * 16;
    float acc[4][2][4];
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) acc[mt][nt][0] = acc[mt][nt][1] = acc[mt][nt][2] = acc[mt][nt][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      uint32_t b0, b1, b2, b3;
      const int irow = 16 * ks + (lane & 7) + ((lane >> 3) & 1) * 8;
      const int dcol = kcol + ((lane >> 4) & 1) * 8;
      ldsm_x4_t(Xs + (dcol >> 6) * 8192 + sw128(irow, (dcol & 63) >> 3), b0, b1, b2, b3);
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        if (ks > mt) continue;
        uint32_t a[4];
        ldsm_x4(Ps + sw128(16 * mt + (lane & 7) + ((lane >> 3) & 1) * 8, ks * 2 + (lane >> 4)), a[0], a[1], a[2], a[3]);
        mma_bf16_16816(acc[mt][0], a, b0, b1);
        mma_bf16_16816(acc[mt][1], a, b2, b3);
      }
    }
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int t = 16 * mt + g8 + 8 * h2;
        const float gm = Eg[t];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const int k = kcol + nt * 8 + c2;
          uint32_t *qp = reinterpret_cast<uint32_t *>(sm + L::oQ + boxed(64, t, k));
          const uint32_t qv = *qp;
          *qp = pack_bf16(fmaf(gm, bf16_lo(qv), -acc[mt][nt][2 * h2]), fmaf(gm, bf16_hi(qv), -acc[mt][nt][2 * h2 + 1]));
        }
      }
  }
  if (threadIdx.x == 0) {
    tma_store_2d(&p.tm_u, smem_u32(sm + L::oUt), 0, 2 * wrow);
    bulk_commit();
  }
  tc::fence_proxy_async_smem();  // Qt is final
  __syncthreads();
  // ---- step 5: -W_e = -diag(e) W in place (W is no longer read) and its TMA store; the
  // record is flagged once all of its stores have completed ----
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int q = threadIdx.x + j * kPT;  // 16-byte chunk of the two W boxes
    const int r = (q >> 3) & 63;
    uint4 *w4 = reinterpret_cast<uint4 *>(Xp + (q >> 9) * 8192 + r * 128 + (q & 7) * 16);
    const uint4 v = *w4;
    const float s = -Ee[r];
    *w4 = make_uint4(pack_bf16(s * bf16_lo(v.x), s * bf16_hi(v.x)), pack_bf16(s * bf16_lo(v.y), s * bf16_hi(v.y)),
                     pack_bf16(s * bf16_lo(v.z), s * bf16_hi(v.z)), pack_bf16(s * bf16_lo(v.w), s * bf16_hi(v.w)));
  }
  if (threadIdx.x == 0) {
    tma_store_2d(&p.tm_qt, qb, 0, wrow);
    tma_store_2d(&p.tm_qt, qb + 8192, 64, wrow);
    bulk_commit();
  }
  tc::fence_proxy_async_smem();
  __syncthreads();
  if (threadIdx.x == 0) {
    tma_store_2d(&p.tm_w, kb, 0, wrow);
    tma_store_2d(&p.tm_w, kb + 8192, 64, wrow);
    bulk_commit();
    bulk_wait_all();
    asm volatile("fence.proxy.async.global;\n" ::: "memory");
    asm volatile("st.release.gpu.global.u32 [%0], %1;\n" ::"l"(p.ws.flag + rec), "r"(1u) : "memory");
  }
}

// ============================================================================
// gdn_scan: the state scan on the 5th-generation tensor cores, one CTA per
// (sequence, value head).  A chunk's update is affine in the state:
//     S_{c+1} = gamma_C S_c - S_c M_c + B_c,   M_c = W^T diag(e) K,   B_c = U'^T diag(e) K,
// because the scalar gates commute with the rank-one factors, so the chunk's product of
// exp(g_t) (I - beta_t k_t k_t^T) is gamma_C times the ungated product (I - M_c / gamma_C).
// The output is O_c = scale (Qt S_c^T + P U') with Qt = diag(gamma) Q - P W from gdn_prep.
// The state is held transposed, S^T (d_k x d_v, fp32), in tensor memory (lane = key index n,
// column = value index v), so that -M_c^T can be the MMA's A operand from tensor memory.
// Per chunk c:
//   MMA M     (one chunk ahead)  Mt = K^T (-W_e) = -M_c^T,   W_e = diag(e) W
//   convert   (side warps)       Mt -> bf16 pairs in place (columns 0..63), Kh^T = (diag(e) K)^T as
//                                bf16 pairs (columns 64..95): A = [ -M_c^T | Kh^T ], K = 128 + 64
//   pass      (chain warps)      S^T -> bf16 copy in shared memory (MN-major), gamma_C S^T -> TMEM
//   MMA S                        S^T += A [ S^T_bf16 ; U' ]                 (the sequential chain)
//   MMA O     (off the chain)    O^T = S Qt^T + U'^T P^T  -> out pass: o = scale O
// Only pass -> MMA S is sequential from chunk to chunk.
// Warps 0-7: pass and out pass (two per TMEM lane quarter, half of the columns each);
// warps 8-11: conversion (one per lane quarter); warp 12: MMA issue; warp 13: TMA issue.
// ============================================================================
constexpr int kSThreads = 14 * 32;

struct ScanParams {
  CUtensorMap tm_k;               // input K, 4-D (d, heads, T, B), box (64, 1, 64, 1)
  CUtensorMap tm_w, tm_qt, tm_p;  // workspace -W_e, Qt [rows][128] and P [rows][64], box (64, 64)
  CUtensorMap tm_u;               // workspace U'^T [rows][64], box (64, 128)
  GdnWs ws;
  const float *state_in;
  float *state_out;
  bf16_t *o;
  int B, T, n_chunks;
  Heads h;
  float scale;
  unsigned *status;
};

struct ScanSmem {
  // ring A (2 slots): -W_e and K of a chunk, used one chunk ahead (MMA M, conversion)
  static constexpr int kASlot = 32768, oA = 0, aW = 0, aK = 16384;
  // ring B (3 slots): U'^T, Qt and P of a chunk (MMA S, MMA O)
  static constexpr int kBSlot = 40960, oB = oA + 2 * kASlot, bU = 0, bQ = 16384, bP = 32768;
  static constexpr int oS = oB + 3 * kBSlot;  // bf16 S^T [128 k][128 v], MN-major: 2 boxes of 64 v
  static constexpr int oE = oS + 32768;       // fp32 e[2][64] (ring A), gamma[3][64] (ring B)
  static constexpr int oBar = oE + 5 * 256;
  static constexpr int kTotal = oBar + 256 + 1024;
};
static_assert(ScanSmem::kTotal <= 232448, "shared memory budget");

// bounded wait for gdn_prep's ready flag of one record, then order the async-proxy (TMA) reads after it
__device__ bool wait_record(const unsigned *flag, unsigned *status) {
  auto ready = [&]() {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];\n" : "=r"(v) : "l"(flag) : "memory");
    return v != 0u;
  };
  bool ok = ready();
  if (!ok) {
    const uint64_t t0 = global_ns();
    for (uint32_t i = 1;; ++i) {
      __nanosleep(32);
      if (ready()) {
        ok = true;
        break;
      }
      if ((i & 63u) == 0) {
        const uint64_t dt = global_ns() - t0;
        if ((dt > HH_WAIT_PEER_NS && status && (*reinterpret_cast<volatile unsigned *>(status) & kStatusTimeout)) ||
            dt > HH_WAIT_NS) {
          if (status) atomicOr(status, kStatusTimeout);
          break;
        }
      }
    }
  }
  asm volatile("fence.proxy.async.global;\n" ::: "memory");
  return ok;
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__global__ void __launch_bounds__(kSThreads, 1) gdn_scan_kernel(const __grid_constant__ ScanParams p) {
  using L = ScanSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::oBar);
  uint64_t *fullA = bars, *fullB = bars + 2, *mdone = bars + 5, *mready = bars + 7, *passd = bars + 9,
           *chaind = bars + 10, *odoneS = bars + 11, *odone = bars + 12, *ofree = bars + 14, *fin = bars + 16,
           *bfree = bars + 17;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 20);
  float *eA = reinterpret_cast<float *>(sm + L::oE);  // [2][64]
  float *gB = eA + 128;                                // [3][64]
  const uint32_t sA = smem_u32(sm + L::oA), sB = smem_u32(sm + L::oB), sS = smem_u32(sm + L::oS);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hi = blockIdx.x, b = blockIdx.y;
  const int vh = p.h.vh(hi), qh = p.h.qh(hi);
  const size_t rec0 = ((size_t)b * p.h.n_heads + hi) * p.n_chunks;
  const size_t st_base = ((size_t)b * p.h.v_heads + vh) * kDK * kDK;
  const int n = p.n_chunks;
  // tensor memory columns: S^T, two M buffers (128 each), two O buffers (64 each)
  constexpr uint32_t cS = 0, cM = 128, cO = 384;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&fullA[i], 1);
      mbar_init(&mdone[i], 1);
      mbar_init(&mready[i], 4);
      mbar_init(&odone[i], 1);
      mbar_init(&ofree[i], 8);
    }
    for (int i = 0; i < 3; ++i) {
      mbar_init(&fullB[i], 1);
      mbar_init(&bfree[i], 1);
    }
    mbar_init(passd, 8);
    mbar_init(chaind, 1);
    mbar_init(odoneS, 1);
    mbar_init(fin, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(smem_u32(tmem_slot), 512);
    tc::tmem_relinquish();
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 12) {
    // ---------------- MMA issue: the warp runs the loop, one elected lane issues ----------------
    // Descriptors are hoisted; a k step or a ring slot only adds to the 16-byte address field.
    const uint64_t dK = tc::desc_mnmajor_sw128(sA + L::aK, 8192, 1024);
    const uint64_t dW = tc::desc_mnmajor_sw128(sA + L::aW, 8192, 1024);
    const uint64_t dS = tc::desc_mnmajor_sw128(sS, 16384, 1024);  // B of MMA S, A of MMA O
    const uint64_t dU = tc::desc_kmajor_sw128(sB + L::bU);
    const uint64_t dQ = tc::desc_kmajor_sw128(sB + L::bQ);
    const uint64_t dP = tc::desc_kmajor_sw128(sB + L::bP);
    constexpr uint32_t idM = tc::idesc_bf16_f32(128, 128, 1, 1);   // K^T, -W_e: both MN-major
    constexpr uint32_t idS1 = tc::idesc_bf16_f32(128, 128, 0, 1);  // A in TMEM, S^T_bf16 MN-major
    constexpr uint32_t idS2 = tc::idesc_bf16_f32(128, 128, 0, 0);  // A in TMEM, U'^T K-major
    constexpr uint32_t idO1 = tc::idesc_bf16_f32(128, 64, 1, 0);   // S (MN-major from S^T), Qt K-major
    constexpr uint32_t idO2 = tc::idesc_bf16_f32(128, 64, 0, 0);   // U'^T, P: both K-major
    auto wait_all = [&](uint64_t *bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, p.status));
    };
    auto mmaM = [&](int c) -> bool {
      const int s = c & 1;
      if (!wait_all(&fullA[s], (c >> 1) & 1)) return false;
      tc::fence_after();
      {
        const uint32_t o = (uint32_t)(s * L::kASlot) >> 4;
#pragma unroll
        for (int ks = 0; ks < kC / 16; ++ks)
          tc::mma_ss_w(tbase + cM + s * 128, dK + o + ks * 128, dW + o + ks * 128, idM, ks ? 1u : 0u);
        tc::commit_w(&mdone[s]);
      }
      return true;
    };
    bool ok = n > 0 && mmaM(0);
    for (int c = 0; c < n && ok; ++c) {
      const int s2 = c & 1, s3 = c % 3;
      // M of the next chunk, into the buffer MMA S of chunk c - 1 has finished reading
      if (c >= 1 && !wait_all(chaind, (c - 1) & 1)) break;
      if (c + 1 < n && !mmaM(c + 1)) break;
      // MMA S (the chain): S^T += [-M_c^T | Kh^T] [S^T_bf16 ; U']
      if (!wait_all(&mready[s2], (c >> 1) & 1)) break;
      if (!wait_all(passd, c & 1)) break;
      if (!wait_all(&fullB[s3], (c / 3) & 1)) break;
      tc::fence_after();
      const uint32_t ob = (uint32_t)(s3 * L::kBSlot) >> 4;
      {
        const uint32_t aM = tbase + cM + s2 * 128;
#pragma unroll
        for (int ks = 0; ks < kDK / 16; ++ks) tc::mma_ts_w(tbase + cS, aM + ks * 8, dS + ks * 128, idS1, 1u);
#pragma unroll
        for (int ks = 0; ks < kC / 16; ++ks) tc::mma_ts_w(tbase + cS, aM + 64 + ks * 8, dU + ob + ks * 2, idS2, 1u);
        tc::commit_w(chaind);
      }
      // MMA O of chunk c, into the buffer the out pass of chunk c - 2 has drained
      if (c >= 2 && !wait_all(&ofree[s2], ((c - 2) >> 1) & 1)) break;
      tc::fence_after();
      {
        const uint32_t dO = tbase + cO + s2 * 64;
#pragma unroll
        for (int ks = 0; ks < kDK / 16; ++ks) {
          const int k0 = ks * 16;
          tc::mma_ss_w(dO, dS + ks * 128, dQ + ob + (uint32_t)(((k0 >> 6) * 8192 + (k0 & 63) * 2) >> 4), idO1, ks ? 1u : 0u);
        }
        tc::commit_w(odoneS);
#pragma unroll
        for (int ks = 0; ks < kC / 16; ++ks) tc::mma_ss_w(dO, dU + ob + ks * 2, dP + ob + ks * 2, idO2, 1u);
        tc::commit_w(&odone[s2]);
        tc::commit_w(&bfree[s3]);
      }
    }
    tc::commit_w(fin);
    mbar_wait(fin, 0, p.status);
  } else if (warp == 13) {
    // ---------------- TMA issue (one thread) ----------------
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_w);
      tma_prefetch_desc(&p.tm_qt);
      tma_prefetch_desc(&p.tm_p);
      tma_prefetch_desc(&p.tm_u);
      int lastA = -1, lastB = -1;  // the last chunk loaded into ring A / ring B
      for (int c = 0; c < n; ++c) {
        // ring A slot: free once chunk c - 2 is converted; the record must have been written
        if (c >= 2 && !mbar_wait(&mready[c & 1], ((c - 2) >> 1) & 1, p.status)) break;
        if (!wait_record(p.ws.flag + rec0 + c, p.status)) break;
        {
          const int s = c & 1;
          mbar_arrive_expect_tx(&fullA[s], 2 * 16384 + 256);
          const uint32_t dst = sA + s * L::kASlot;
          const int row = (int)((rec0 + c) * kC);
          tma_load_2d(dst + L::aW, &p.tm_w, &fullA[s], 0, row);
          tma_load_2d(dst + L::aW + 8192, &p.tm_w, &fullA[s], 64, row);
          tma_load_4d(dst + L::aK, &p.tm_k, &fullA[s], 0, qh, c * kC, b);
          tma_load_4d(dst + L::aK + 8192, &p.tm_k, &fullA[s], 64, qh, c * kC, b);
          bulk_load(smem_u32(eA + s * 64), p.ws.fc + (rec0 + c) * 128 + 64, 256, &fullA[s]);
          lastA = c;
        }
        // ring B slot: free once MMA O of chunk c - 3 has completed
        if (c >= 3 && !mbar_wait(&bfree[c % 3], ((c - 3) / 3) & 1, p.status)) break;
        {
          const int s = c % 3;
          mbar_arrive_expect_tx(&fullB[s], 2 * 16384 + 8192 + 256);
          const uint32_t dst = sB + s * L::kBSlot;
          const int row = (int)((rec0 + c) * kC);
          tma_load_2d(dst + L::bU, &p.tm_u, &fullB[s], 0, 2 * row);
          tma_load_2d(dst + L::bQ, &p.tm_qt, &fullB[s], 0, row);
          tma_load_2d(dst + L::bQ + 8192, &p.tm_qt, &fullB[s], 64, row);
          tma_load_2d(dst + L::bP, &p.tm_p, &fullB[s], 0, row);
          bulk_load(smem_u32(gB + s * 64), p.ws.fc + (rec0 + c) * 128, 256, &fullB[s]);
          lastB = c;
        }
      }
      // every load issued above has landed before the CTA can exit (bounded; complete on the
      // normal path, where the consumers waited for each of them)
      for (int c = max(lastA - 1, 0); c <= lastA; ++c) mbar_wait(&fullA[c & 1], (c >> 1) & 1, p.status);
      for (int c = max(lastB - 2, 0); c <= lastB; ++c) mbar_wait(&fullB[c % 3], (c / 3) & 1, p.status);
    }
    __syncwarp();
  } else if (warp >= 8) {
    // ---------------- conversion: -M_c^T and Kh^T -> bf16 A operand of MMA S ----------------
    const int q4 = warp & 3;
    const int nrow = q4 * 32 + lane;  // key index n = TMEM lane
    const uint32_t tl = tbase + ((uint32_t)(q4 * 32) << 16);
    for (int c = 0; c < n; ++c) {
      const int s = c & 1;
      const bool w = mbar_wait(&fullA[s], (c >> 1) & 1, p.status) && mbar_wait(&mdone[s], (c >> 1) & 1, p.status);
      if (!__all_sync(0xffffffffu, w)) break;
      tc::fence_after();
      const uint32_t tm = tl + cM + s * 128;
      // in place: fp32 columns 64h .. 64h+63 -> bf16 pairs in columns 32h .. 32h+31 (read before written)
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        uint32_t r0[32], r1[32], pk[32];
        tc::ld32(tm + h * 64, r0);
        tc::ld32(tm + h * 64 + 32, r1);
        tc::wait_ld();
        tc::regfence(r0);
        tc::regfence(r1);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          pk[i] = pack_bf16(__uint_as_float(r0[2 * i]), __uint_as_float(r0[2 * i + 1]));
          pk[16 + i] = pack_bf16(__uint_as_float(r1[2 * i]), __uint_as_float(r1[2 * i + 1]));
        }
        tc::st32u(tm + h * 32, pk);
      }
      {  // Kh^T row n: column n of the K tile scaled by e_t, pairs of tokens
        const uint8_t *kt = sm + L::oA + s * L::kASlot + L::aK + (nrow >> 6) * 8192 + (nrow & 7) * 2;
        const int cchunk = (nrow & 63) >> 3;
        const float *e = eA + s * 64;
        uint32_t pk[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int t = 2 * j;
          const float k0 = bf16_to_f(*reinterpret_cast<const bf16_t *>(kt + sw128(t, cchunk)));
          const float k1 = bf16_to_f(*reinterpret_cast<const bf16_t *>(kt + sw128(t + 1, cchunk)));
          pk[j] = pack_bf16(k0 * e[t], k1 * e[t + 1]);
        }
        tc::st32u(tm + 64, pk);
      }
      tc::wait_st();
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&mready[s]);
    }
  } else {
    // ---------------- chain pass and out pass: warps 0-7 ----------------
    const int q4 = warp & 3, half = warp >> 2;
    const int nrow = q4 * 32 + lane;  // S^T row (key index n); O^T row (value index v)
    const uint32_t tl = tbase + ((uint32_t)(q4 * 32) << 16);
    const uint32_t srow = sS + half * 16384 + nrow * 128;
    auto out_pass = [&](int c) -> bool {
      const int s2 = c & 1;
      const bool w = mbar_wait(&odone[s2], (c >> 1) & 1, p.status);
      if (!__all_sync(0xffffffffu, w)) return false;
      tc::fence_after();
      uint32_t ov[32];
      tc::ld32(tl + cO + s2 * 64 + half * 32, ov);
      tc::wait_ld();
      tc::regfence(ov);
      const int t0 = c * kC + half * 32, nv = min(32, p.T - t0);
      bf16_t *dst = p.o + (((size_t)b * p.T + t0) * p.h.v_heads + vh) * kDK + nrow;
      const size_t tstride = (size_t)p.h.v_heads * kDK;
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (i < nv) dst[i * tstride] = f_to_bf16(p.scale * __uint_as_float(ov[i]));
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ofree[s2]);
      return true;
    };
    bool ok = true;
    for (int c = 0; c < n; ++c) {
      const int s3 = c % 3;
      {
        bool w = c == 0 || mbar_wait(chaind, (c - 1) & 1, p.status);
        w = w && mbar_wait(&fullB[s3], (c / 3) & 1, p.status);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        tc::fence_after();
      }
      const float gC = gB[s3 * 64 + kC - 1];
      uint32_t pk[32];
      // this thread's 64 columns (values 64*half ..) of S^T_c: bf16 copy kept, gamma_C S^T_c -> TMEM
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int v0 = half * 64 + h * 32;
        float f[32];
        if (c == 0) {
#pragma unroll
          for (int i = 0; i < 32; ++i) f[i] = p.state_in ? p.state_in[st_base + (size_t)(v0 + i) * kDK + nrow] : 0.f;
        } else {
          uint32_t r[32];
          tc::ld32(tl + cS + v0, r);
          tc::wait_ld();
          tc::regfence(r);
#pragma unroll
          for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(r[i]);
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[h * 16 + i] = pack_bf16(f[2 * i], f[2 * i + 1]);
#pragma unroll
        for (int i = 0; i < 32; ++i) f[i] *= gC;
        tc::st32(tl + cS + v0, f);
      }
      {  // the shared copy is overwritten once MMA O of chunk c - 1 has read it
        const bool w = c == 0 || mbar_wait(odoneS, (c - 1) & 1, p.status);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) sts128(srow + ((j ^ (nrow & 7)) << 4), pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
      tc::wait_st();
      tc::fence_proxy_async_smem();
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(passd);
      if (c > 0 && !out_pass(c - 1)) {
        ok = false;
        break;
      }
    }
    if (ok && n > 0) {
      const bool w = mbar_wait(chaind, (n - 1) & 1, p.status);
      if (__all_sync(0xffffffffu, w)) {
        tc::fence_after();
        if (p.state_out) {
#pragma unroll 1
          for (int h = 0; h < 2; ++h) {
            const int v0 = half * 64 + h * 32;
            uint32_t r[32];
            tc::ld32(tl + cS + v0, r);
            tc::wait_ld();
            tc::regfence(r);
#pragma unroll
            for (int i = 0; i < 32; ++i) p.state_out[st_base + (size_t)(v0 + i) * kDK + nrow] = __uint_as_float(r[i]);
          }
        }
        out_pass(n - 1);
      }
    }
  }
  tc::fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after();
    tc::tmem_dealloc(tbase, 512);
  }
}

// RMS fusion pass over the rows of the mapped heads (used when d_v was split):
// y = x / sqrt(mean(x^2) + eps) per (token, head), in place.  One warp per row.
__global__ void gdn_rms_rows_kernel(bf16_t *o, int B, int T, Heads h, float eps) {
  const long long rowid = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const long long n_rows = (long long)B * T * h.n_heads;
  if (rowid >= n_rows) return;
  const int hi = (int)(rowid % h.n_heads);
  const long long bt = rowid / h.n_heads;
  bf16_t *row = o + (bt * h.v_heads + h.vh(hi)) * kDK + lane * 4;
  uint2 v = *reinterpret_cast<uint2 *>(row);
  const float x0 = bf16_lo(v.x), x1 = bf16_hi(v.x), x2 = bf16_lo(v.y), x3 = bf16_hi(v.y);
  const float ss = warp_sum(x0 * x0 + x1 * x1 + x2 * x2 + x3 * x3);
  const float r = rsqrtf(ss / (float)kDK + eps);
  *reinterpret_cast<uint2 *>(row) = make_uint2(pack_bf16(x0 * r, x1 * r), pack_bf16(x2 * r, x3 * r));
}

// T == 0: the state passes through unchanged
__global__ void gdn_state_copy_kernel(const float *__restrict__ in, float *__restrict__ out, Heads h) {
  const int hi = blockIdx.x, b = blockIdx.y;
  const size_t base = ((size_t)b * h.v_heads + h.vh(hi)) * kDK * kDK;
  for (int i = threadIdx.x; i < kDK * kDK; i += blockDim.x) out[base + i] = in ? in[base + i] : 0.f;
}

}  // namespace
size_t gdn_workspace_bytes(int B, int T, int n_heads) {
  const size_t n_chunks = ((size_t)T + kC - 1) / kC;
  return (size_t)B * n_heads * n_chunks * (kWBytes + kUBytes + kPBytes + kQBytes + kFBytes + sizeof(unsigned));
}

namespace {
// Library-owned streams per device: gdn_prep on `lo`, the scan on `hi` (highest
// priority), so that the scan's CTAs (one per sequence and head, waiting for each
// chunk's record) take SMs as gdn_prep's first CTAs drain, while gdn_prep fills the
// rest producing the records in chunk order.  gdn_prep is launched first: where
// launches are serialised (a profiler, CUDA_LAUNCH_BLOCKING) it simply completes
// before the scan starts.
struct PrepStream {
  cudaStream_t lo = nullptr, hi = nullptr;
  cudaEvent_t fork = nullptr, join_lo = nullptr, join_hi = nullptr;
};
std::mutex g_prep_mu;
PrepStream g_prep[128];
}  // namespace

namespace {
cudaError_t launch_rms_rows(const GdnChunkArgs &a, const Heads &h, cudaStream_t s) {
  const long long n_rows = (long long)a.B * a.T * a.n_heads;
  gdn_rms_rows_kernel<<<(unsigned)((n_rows + 7) / 8), 256, 0, s>>>(a.o, a.B, a.T, h, a.eps);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_gdn_chunk(const GdnChunkArgs &a, cudaStream_t s) {
  if (a.B == 0 || a.n_heads == 0) return cudaSuccess;
  Heads h;
  memset(&h, 0, sizeof(h));
  h.n_heads = a.n_heads;
  h.group = a.group;
  h.qk_heads = a.qk_heads;
  h.v_heads = a.v_heads;
  h.use_map = a.use_map;
  memcpy(h.map, a.map, sizeof(h.map));
  if (a.T == 0) {
    if (!a.state_out) return cudaSuccess;
    gdn_state_copy_kernel<<<dim3(a.n_heads, a.B), 256, 0, s>>>(a.state_in, a.state_out, h);
    return cudaGetLastError();
  }
  const int n_chunks = (a.T + kC - 1) / kC;
  if (n_chunks > 65535 || a.B > 65535) {
    set_error("gdn_chunk_fwd: T above 4194240 tokens or B above 65535");
    return cudaErrorInvalidValue;
  }
  const GdnWs ws = carve(a.workspace, a.B, a.n_heads, n_chunks);
  unsigned *status = device_status_ptr();

  // ---- inputs' tensor maps ----
  CUtensorMap tq, tk, tv, tw, tp, tu, tqt;
  const uint32_t box4[4] = {64, 1, (uint32_t)kC, 1};
  const uint64_t dq[4] = {(uint64_t)kDK, (uint64_t)a.qk_heads, (uint64_t)a.T, (uint64_t)a.B};
  const uint64_t sq[3] = {(uint64_t)kDK * 2, (uint64_t)a.qk_heads * kDK * 2, (uint64_t)a.T * a.qk_heads * kDK * 2};
  const uint64_t dv[4] = {(uint64_t)kDK, (uint64_t)a.v_heads, (uint64_t)a.T, (uint64_t)a.B};
  const uint64_t sv[3] = {(uint64_t)kDK * 2, (uint64_t)a.v_heads * kDK * 2, (uint64_t)a.T * a.v_heads * kDK * 2};
  const uint64_t rows = (uint64_t)a.B * a.n_heads * n_chunks * kC;
  const uint64_t dw[2] = {(uint64_t)kDK, rows}, sw[1] = {(uint64_t)kDK * 2};
  const uint64_t dp[2] = {(uint64_t)kC, rows}, sp[1] = {(uint64_t)kC * 2};
  const uint32_t box2[2] = {64, (uint32_t)kC};
  const uint64_t du[2] = {(uint64_t)kC, rows * 2}, su[1] = {(uint64_t)kC * 2};
  const uint32_t boxu[2] = {(uint32_t)kC, (uint32_t)kDK};
  if (encode_tmap(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.q, dq, sq, box4, CU_TENSOR_MAP_SWIZZLE_128B) ||
      encode_tmap(&tu, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws.up, du, su, boxu, CU_TENSOR_MAP_SWIZZLE_128B) ||
      encode_tmap(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.k, dq, sq, box4, CU_TENSOR_MAP_SWIZZLE_128B) ||
      encode_tmap(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.v, dv, sv, box4, CU_TENSOR_MAP_SWIZZLE_128B) ||
      encode_tmap(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws.wn, dw, sw, box2, CU_TENSOR_MAP_SWIZZLE_128B) ||
      encode_tmap(&tqt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws.qt, dw, sw, box2, CU_TENSOR_MAP_SWIZZLE_128B) ||
      encode_tmap(&tp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws.pm, dp, sp, box2, CU_TENSOR_MAP_SWIZZLE_128B)) {
    set_error("gdn_chunk_fwd: cuTensorMapEncodeTiled failed");
    return cudaErrorInvalidValue;
  }

  // ---- gdn_prep: chunk-local products, all chunks in parallel ----
  PrepParams pp;
  memset(&pp, 0, sizeof(pp));
  pp.tm_q = tq;
  pp.tm_k = tk;
  pp.tm_v = tv;
  pp.tm_w = tw;
  pp.tm_u = tu;
  pp.tm_p = tp;
  pp.tm_qt = tqt;
  pp.g = a.g;
  pp.beta = a.beta;
  pp.ws = ws;
  pp.B = a.B;
  pp.T = a.T;
  pp.n_chunks = n_chunks;
  pp.h = h;
  pp.status = status;
  cudaError_t e = cudaFuncSetAttribute(gdn_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, PrepSmem::kTotal);
  if (e != cudaSuccess) return e;

  // ---- gdn_scan: the state chain on the tensor cores, one CTA per (sequence, head) ----
  ScanParams st;
  memset(&st, 0, sizeof(st));
  st.tm_k = tk;
  st.tm_w = tw;
  st.tm_qt = tqt;
  st.tm_p = tp;
  st.tm_u = tu;
  st.ws = ws;
  st.state_in = a.state_in;
  st.state_out = a.state_out;
  st.o = a.o;
  st.B = a.B;
  st.T = a.T;
  st.n_chunks = n_chunks;
  st.h = h;
  st.scale = a.scale;
  st.status = status;
  e = cudaFuncSetAttribute(gdn_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, ScanSmem::kTotal);
  if (e != cudaSuccess) return e;

  // ---- launch: flags cleared, then gdn_prep and the scan on the library's two streams,
  // joined back into the caller's stream.  The scan's CTAs (one SM each) wait for
  // gdn_prep, so they run beside it only while they take at most half of the SMs;
  // otherwise both run one after the other on the caller's stream. ----
  {
    int dev = 0, n_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
    if ((e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const size_t rec = (size_t)a.B * a.n_heads * n_chunks;
    if ((e = cudaMemsetAsync(ws.flag, 0, rec * sizeof(unsigned), s)) != cudaSuccess) return e;
    if (2LL * a.B * a.n_heads > (long long)n_sm) {
      gdn_prep_kernel<<<dim3(a.n_heads, n_chunks, a.B), kPThreads, PrepSmem::kTotal, s>>>(pp);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
      gdn_scan_kernel<<<dim3(a.n_heads, a.B), kSThreads, ScanSmem::kTotal, s>>>(st);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
      return a.rms ? launch_rms_rows(a, h, s) : cudaSuccess;
    }
    std::lock_guard<std::mutex> lock(g_prep_mu);
    PrepStream &ps = g_prep[dev];
    if (!ps.lo) {
      int lo_pri = 0, hi_pri = 0;
      if ((e = cudaDeviceGetStreamPriorityRange(&lo_pri, &hi_pri)) != cudaSuccess ||
          (e = cudaStreamCreateWithPriority(&ps.hi, cudaStreamNonBlocking, hi_pri)) != cudaSuccess ||
          (e = cudaStreamCreateWithFlags(&ps.lo, cudaStreamNonBlocking)) != cudaSuccess ||
          (e = cudaEventCreateWithFlags(&ps.fork, cudaEventDisableTiming)) != cudaSuccess ||
          (e = cudaEventCreateWithFlags(&ps.join_lo, cudaEventDisableTiming)) != cudaSuccess ||
          (e = cudaEventCreateWithFlags(&ps.join_hi, cudaEventDisableTiming)) != cudaSuccess)
        return e;
    }
    if ((e = cudaEventRecord(ps.fork, s)) != cudaSuccess || (e = cudaStreamWaitEvent(ps.lo, ps.fork, 0)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(ps.hi, ps.fork, 0)) != cudaSuccess)
      return e;
    gdn_prep_kernel<<<dim3(a.n_heads, n_chunks, a.B), kPThreads, PrepSmem::kTotal, ps.lo>>>(pp);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    gdn_scan_kernel<<<dim3(a.n_heads, a.B), kSThreads, ScanSmem::kTotal, ps.hi>>>(st);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = cudaEventRecord(ps.join_lo, ps.lo)) != cudaSuccess || (e = cudaEventRecord(ps.join_hi, ps.hi)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(s, ps.join_lo, 0)) != cudaSuccess || (e = cudaStreamWaitEvent(s, ps.join_hi, 0)) != cudaSuccess)
      return e;
  }
  return a.rms ? launch_rms_rows(a, h, s) : cudaSuccess;
}
}  // namespace hh
