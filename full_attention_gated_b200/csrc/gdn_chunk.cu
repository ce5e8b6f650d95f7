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
// (These identities are checked on the CPU against the token-by-token oracle.)
//
// Two kernels, so that only the state-dependent products sit on the
// sequential chain over chunks:
//   gdn_prep   parallel over (chunk, value head): K K^T, Q K^T, the blocked fp32
//              triangular inverse, -W, U', P and the decay factors, written to a
//              caller-provided workspace (bf16 matrices, fp32 factors);
//   gdn_scan   one CTA per (sequence, value head, d_v slice) runs the chain: per
//              chunk U = U' - W S^T, O = scale(gamma Q S^T + P U), S update.  State
//              rows evolve independently, so d_v is split over up to 4 CTAs to fill
//              the GPU.  The fp32 state master stays in MMA accumulator registers
//              for the whole sequence, a bf16 copy in shared memory feeds the MMAs.
// Both stream their tiles with TMA (128-byte swizzle) and use warp-level bf16
// MMAs with fp32 accumulation.  A last partial chunk is padded with k = 0,
// beta = 0, g = 0 tokens, which leave the state unchanged and whose outputs are
// not written.  The head-level hybrid layer's RMS fusion is applied in the scan
// when a CTA holds whole rows, otherwise by a small row pass afterwards.
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace hh {

namespace {

constexpr int kC = 64;    // chunk length
constexpr int kDK = 128;  // key (and value) dim

// workspace record per (sequence, value head, chunk)
constexpr size_t kWBytes = (size_t)kC * kDK * 2;  // -W   [64][128] bf16
constexpr size_t kUBytes = (size_t)kC * kDK * 2;  // U'^T [128][64] bf16 (d_v rows, token columns)
constexpr size_t kPBytes = (size_t)kC * kC * 2;   // P    [64][64]  bf16
constexpr size_t kFBytes = (size_t)2 * kC * 4;    // gamma[64], exp(G_C - G)[64] fp32

struct GdnWs {
  bf16_t *wn, *up, *pm;  // [B, Hn, n_chunks] x (-W [64][128] | U'^T [128][64] | P [64][64])
  float *fc;             // [B, Hn, n_chunks, 2, 64]
};

GdnWs carve(void *ws, int B, int Hn, int n_chunks) {
  const size_t rec = (size_t)B * Hn * n_chunks;
  uint8_t *p = reinterpret_cast<uint8_t *>(ws);
  GdnWs w;
  w.wn = reinterpret_cast<bf16_t *>(p);
  w.up = reinterpret_cast<bf16_t *>(p + rec * kWBytes);
  w.pm = reinterpret_cast<bf16_t *>(p + rec * (kWBytes + kUBytes));
  w.fc = reinterpret_cast<float *>(p + rec * (kWBytes + kUBytes + kPBytes));
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
// gdn_prep: one CTA per (chunk, head, sequence), 8 MMA warps; thread 0 issues TMA.
// W and U' come from a block forward substitution on (I + A) X = R with
// R = [diag(beta gamma) K | diag(beta) V] and 16-row blocks:
//     X_I = (I + A_II)^-1 (R_I - sum_{J<I} A_IJ X_J),   W = X[:, :128], U' = X[:, 128:]
// The four 16 x 16 diagonal inverses are formed in fp32 by forward substitution;
// every other product is a warp MMA (bf16 operands, fp32 accumulation).  Warp w
// owns columns 32w .. 32w+31 of X through all four block rows, so the solve
// needs no CTA-wide synchronisation.
// ============================================================================
constexpr int kPW = 8;            // warps
constexpr int kPT = kPW * 32;     // threads
constexpr int kPThreads = kPT;

struct PrepParams {
  CUtensorMap tm_q, tm_k, tm_v;  // 4-D (d, heads, T, B), box (64, 1, 64, 1)
  const float *g, *beta;
  GdnWs ws;
  int B, T, n_chunks;
  Heads h;
  unsigned *status;
};

struct PrepSmem {
  static constexpr int oQ = 0, oK = 16384, oV = 32768;  // TMA tiles [64][128] bf16 (2 boxes each)
  static constexpr int oX = 49152;                       // X bf16 [64][256] (4 boxes of 64 columns)
  static constexpr int oAb = oX + 32768;                 // -A off-diagonal blocks, bf16 [64][64] (1 box)
  static constexpr int oAd = oAb + 8192;                 // A diagonal blocks fp32 [4][16][16]
  static constexpr int oTd = oAd + 4096;                 // (I + A_II)^-1 fp32 [4][16][16]
  static constexpr int oY = oTd + 4096;                  // per-warp bf16 [16][32] scratch
  static constexpr int oSmall = oY + kPW * 1024;         // G, beta, gamma [64] each, barrier
  static constexpr int kTotal = oSmall + 3 * 256 + 16 + 1024;
};

__global__ void __launch_bounds__(kPThreads, 2) gdn_prep_kernel(const __grid_constant__ PrepParams p) {
  using L = PrepSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float *Ad = reinterpret_cast<float *>(sm + L::oAd);
  float *Td = reinterpret_cast<float *>(sm + L::oTd);
  float *Gs = reinterpret_cast<float *>(sm + L::oSmall);
  float *Bs = Gs + 64, *Eg = Bs + 64;
  uint64_t *full = reinterpret_cast<uint64_t *>(Eg + 64);
  const uint32_t qb = smem_u32(sm + L::oQ), kb = smem_u32(sm + L::oK), vb = smem_u32(sm + L::oV),
                 Xs = smem_u32(sm + L::oX), Abs = smem_u32(sm + L::oAb);
  uint8_t *Xp = sm + L::oX, *Abp = sm + L::oAb;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x, hi = blockIdx.y, b = blockIdx.z;
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
    p.ws.fc[rec * 128 + 2 * lane] = expf(g_lo);
    p.ws.fc[rec * 128 + 2 * lane + 1] = expf(run);
    p.ws.fc[rec * 128 + 64 + 2 * lane] = expf(GC - g_lo);
    p.ws.fc[rec * 128 + 64 + 2 * lane + 1] = expf(GC - run);
  }
  __syncthreads();
  const bool waited = mbar_wait(full, 0, p.status);
  if (__syncthreads_or(!waited)) return;  // CTA-uniform

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
    bf16_t *P = p.ws.pm + rec * (kC * kC);
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
        *reinterpret_cast<uint32_t *>(P + t * kC + i) = pack_bf16(d0 * qk[j][2 * h2], d1 * qk[j][2 * h2 + 1]);
      }
  }
  __syncthreads();

  // ---- step 2: the four diagonal inverses (I + A_II)^-1, fp32, one column per thread ----
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
  __syncthreads();

  // ---- step 3: block forward substitution; warp w owns columns 32w .. 32w+31 of X ----
  {
    const bool is_w = warp < 4;                      // columns 0..127: W (from K), 128..255: U' (from V)
    const uint8_t *src = sm + (is_w ? L::oK : L::oV);
    const int cbase = (warp & 3) * 32;               // column inside the K or V tile
    const int xcol = warp * 32;                      // column inside X
    uint8_t *Yp = sm + L::oY + warp * 1024;          // [16][32] bf16, 64-byte rows
    const uint32_t Ys = smem_u32(Yp);
    bf16_t *dst = (is_w ? p.ws.wn : p.ws.up) + rec * (kC * kDK) + cbase;
    const float sg = is_w ? -1.f : 1.f;              // the workspace keeps -W
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
        *reinterpret_cast<uint32_t *>(Yp + g8 * 64 + (nt * 8 + c2) * 2) = pack_bf16(acc[nt][0], acc[nt][1]);
        *reinterpret_cast<uint32_t *>(Yp + (g8 + 8) * 64 + (nt * 8 + c2) * 2) = pack_bf16(acc[nt][2], acc[nt][3]);
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
        ldsm_x4_t(Ys + yr * 64 + ycol * 2, b0, b1, b2, b3);
        mma_bf16_16816(xo[2 * nd], ta, b0, b1);
        mma_bf16_16816(xo[2 * nd + 1], ta, b2, b3);
      }
      // X_I -> shared (operand of later block rows) and -> workspace
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        const int col = nt * 8 + c2;
        const uint32_t lo = pack_bf16(xo[nt][0], xo[nt][1]), hi2 = pack_bf16(xo[nt][2], xo[nt][3]);
        if (I < 3) {
          *reinterpret_cast<uint32_t *>(Xp + boxed(64, 16 * I + g8, xcol + col)) = lo;
          *reinterpret_cast<uint32_t *>(Xp + boxed(64, 16 * I + g8 + 8, xcol + col)) = hi2;
        }
        if (is_w) {
          *reinterpret_cast<uint32_t *>(dst + (16 * I + g8) * kDK + col) = pack_bf16(sg * xo[nt][0], sg * xo[nt][1]);
          *reinterpret_cast<uint32_t *>(dst + (16 * I + g8 + 8) * kDK + col) = pack_bf16(sg * xo[nt][2], sg * xo[nt][3]);
        } else {  // U' transposed: row = d_v, column = token
          bf16_t *ut = p.ws.up + rec * (kC * kDK) + (size_t)(cbase + col) * kC + 16 * I + g8;
          ut[0] = f_to_bf16(xo[nt][0]);
          ut[kC] = f_to_bf16(xo[nt][1]);
          ut[8] = f_to_bf16(xo[nt][2]);
          ut[kC + 8] = f_to_bf16(xo[nt][3]);
        }
      }
      __syncwarp();
    }
  }
}

// ============================================================================
// gdn_scan_tc: the state scan on the 5th-generation tensor cores.  One CTA per
// (sequence, value head).  The fp32 state S (d_v x d_k) lives in tensor memory,
// lane = row of S.  Per chunk c (z = c mod 2 selects double-buffered columns):
//   MMA U:   Y   = S (-W)^T                        (M = 128 rows of S, N = 64 tokens)
//   MMA Z:   Z_z = S Q^T                           (off the chain)
//   pass 1:  U^T = U'^T + Y, Uh^T = U^T diag(exp(G_C - G)) -> shared (bf16),
//            S <- gamma_C S                        (in tensor memory)
//   MMA S:   S  += Uh^T K
//   MMA V:   V_z = U^T P^T                         (off the chain)
//   pass 2a: bf16 copy of S -> shared (operand of the next chunk)
//   pass 2b: o_t = scale (gamma_t Z_z + V_z)_t     (overlaps the next chunk's MMAs)
// Only MMA U -> pass 1 -> MMA S -> pass 2a is sequential from chunk to chunk.
// Eight pass warps: two per TMEM lane quarter, each taking half of the columns.
// Thread 0 of warp 8 issues the TMA loads and the MMAs.
// ============================================================================
constexpr int kTSThreads = 288;

struct ScanTcParams {
  CUtensorMap tm_q, tm_k;  // inputs, 4-D (d, heads, T, B), box (64, 1, 64, 1)
  CUtensorMap tm_w, tm_p;  // workspace -W [rows][128] and P [rows][64], box (64, 64)
  CUtensorMap tm_u;        // workspace U'^T [rows][64], box (64, 128), 128-byte swizzle
  GdnWs ws;
  const float *state_in;
  float *state_out;
  bf16_t *o;
  int B, T, n_chunks;
  Heads h;
  float scale;
  unsigned *status;
};

struct ScanTcSmem {
  // stage: -W, Q, K (2 swizzled boxes each), P (1 box), U'^T [128][64] (1 swizzled box), factors [2][64] fp32
  static constexpr int sW = 0, sQ = 16384, sK = 32768, sP = 49152, sU = 57344, sF = 73728;
  static constexpr int kStageBytes = sF + 512;
  static constexpr int kStage = 75776;  // 1024-aligned stride
  static constexpr int oS = 2 * kStage;           // bf16 S [128][128], K-major (2 boxes of 128 rows)
  static constexpr int oUt = oS + 32768;          // bf16 U^T [128][64], K-major (1 box)
  static constexpr int oUh = oUt + 16384;         // bf16 Uh^T [128][64]
  static constexpr int oBar = oUh + 16384;
  static constexpr int kTotal = oBar + 128 + 1024;
  static_assert(kStage >= kStageBytes && (kStage % 1024) == 0, "stage stride");
};

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__global__ void __launch_bounds__(kTSThreads, 1) gdn_scan_tc_kernel(const __grid_constant__ ScanTcParams p) {
  using L = ScanTcSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(sm + L::oBar);  // [2]
  uint64_t *mmaU = full + 2, *mmaS = full + 3, *mmaV = full + 4, *pass1 = full + 5, *pass2 = full + 6, *fin = full + 7;
  uint64_t *outdone = full + 8;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(full + 9);
  const uint32_t ring = smem_u32(sm), sS = smem_u32(sm + L::oS), sUt = smem_u32(sm + L::oUt),
                 sUh = smem_u32(sm + L::oUh);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hi = blockIdx.x, b = blockIdx.y;
  const int vh = p.h.vh(hi), qh = p.h.qh(hi);
  const size_t rec0 = ((size_t)b * p.h.n_heads + hi) * p.n_chunks;
  const size_t st_base = ((size_t)b * p.h.v_heads + vh) * kDK * kDK;
  // tensor memory columns
  constexpr uint32_t cS = 0, cY = 128, cZ = 192, cV = 320;  // Z, V: two 64-column buffers each

  auto issue = [&](int c) {
    const int s = c & 1;
    mbar_arrive_expect_tx(&full[s], L::kStageBytes);
    const uint32_t st = ring + s * L::kStage;
    const int row = (int)((rec0 + c) * kC);
    tma_load_2d(st + L::sW, &p.tm_w, &full[s], 0, row);
    tma_load_2d(st + L::sW + 8192, &p.tm_w, &full[s], 64, row);
    tma_load_2d(st + L::sP, &p.tm_p, &full[s], 0, row);
    tma_load_2d(st + L::sU, &p.tm_u, &full[s], 0, 2 * row);
    bulk_load(st + L::sF, p.ws.fc + (rec0 + c) * 128, 512, &full[s]);
    for (int bx = 0; bx < 2; ++bx) {
      tma_load_4d(st + L::sQ + bx * 8192, &p.tm_q, &full[s], bx * 64, qh, c * kC, b);
      tma_load_4d(st + L::sK + bx * 8192, &p.tm_k, &full[s], bx * 64, qh, c * kC, b);
    }
  };

  if (threadIdx.x == 0) {
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    mbar_init(mmaU, 1);
    mbar_init(mmaS, 1);
    mbar_init(mmaV, 1);
    mbar_init(pass1, 8);
    mbar_init(pass2, 8);
    mbar_init(fin, 1);
    mbar_init(outdone, 8);
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

  if (warp == 8) {
    // ---------------- TMA + MMA issue (one thread) ----------------
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_w);
      tma_prefetch_desc(&p.tm_p);
      tma_prefetch_desc(&p.tm_u);
      for (int c = 0; c < 2 && c < p.n_chunks; ++c) issue(c);
      constexpr uint32_t id64 = tc::idesc_bf16_f32(128, 64, 0, 0);  // N = 64 tokens, K-major B
      constexpr uint32_t idS = tc::idesc_bf16_f32(128, 128, 0, 1);  // N = 128 (d_k), MN-major B (K tile)
      for (int c = 0; c < p.n_chunks; ++c) {
        const int s = c & 1;
        const uint32_t z = (uint32_t)(c & 1) * 64;
        if (!mbar_wait(pass2, c & 1, p.status)) break;  // bf16 S of this chunk is in shared memory
        if (!mbar_wait(&full[s], (c >> 1) & 1, p.status)) break;
        tc::fence_after();
        const uint32_t st = ring + s * L::kStage;
#pragma unroll
        for (int ks = 0; ks < kDK / 16; ++ks) {
          const int k0 = ks * 16;
          tc::mma_ss(tbase + cY, tc::desc_kmajor_sw128(sS + (k0 >> 6) * 16384 + (k0 & 63) * 2),
                     tc::desc_kmajor_sw128(st + L::sW + (k0 >> 6) * 8192 + (k0 & 63) * 2), id64, ks ? 1u : 0u);
        }
        tc::commit(mmaU);
#pragma unroll
        for (int ks = 0; ks < kDK / 16; ++ks) {
          const int k0 = ks * 16;
          tc::mma_ss(tbase + cZ + z, tc::desc_kmajor_sw128(sS + (k0 >> 6) * 16384 + (k0 & 63) * 2),
                     tc::desc_kmajor_sw128(st + L::sQ + (k0 >> 6) * 8192 + (k0 & 63) * 2), id64, ks ? 1u : 0u);
        }
        // the stage of chunk c-1 is free once its outputs are written (MMA V(c-1) done, factors read)
        if (c >= 1) {
          if (!mbar_wait(outdone, (c - 1) & 1, p.status)) break;
          if (c + 1 < p.n_chunks) issue(c + 1);
        }
        if (!mbar_wait(pass1, c & 1, p.status)) break;
        tc::fence_after();
#pragma unroll
        for (int kk = 0; kk < kC / 16; ++kk)
          tc::mma_ss(tbase + cS, tc::desc_kmajor_sw128(sUh + kk * 32),
                     tc::desc_mnmajor_sw128(st + L::sK + kk * 16 * 128, 8192, 1024), idS, 1u);
        tc::commit(mmaS);
#pragma unroll
        for (int kk = 0; kk < kC / 16; ++kk)
          tc::mma_ss(tbase + cV + z, tc::desc_kmajor_sw128(sUt + kk * 32), tc::desc_kmajor_sw128(st + L::sP + kk * 32), id64,
                     kk ? 1u : 0u);
        tc::commit(mmaV);
      }
      tc::commit(fin);
      mbar_wait(fin, 0, p.status);
    }
    __syncwarp();
  } else {
    // ---------------- passes: warps 0-7, rows 32*(w%4) + lane of S, column half w/4 ----------------
    const int q4 = warp & 3, half = warp >> 2;
    const int r = q4 * 32 + lane;
    const uint32_t tl = tbase + ((uint32_t)(q4 * 32) << 16);
    // setup: this thread's half row of S (64 columns) -> tensor memory and the bf16 copy
#pragma unroll 1
    for (int c2 = 0; c2 < 2; ++c2) {
      const int k0 = half * 64 + c2 * 32;
      float v[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = p.state_in ? p.state_in[st_base + (size_t)r * kDK + k0 + i] : 0.f;
      tc::st32(tl + cS + k0, v);
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        const int kc = k0 + ch * 8;
        sts128(sS + (kc >> 6) * 16384 + r * 128 + ((((kc & 63) >> 3) ^ (r & 7)) << 4), pack_bf16(v[ch * 8], v[ch * 8 + 1]),
               pack_bf16(v[ch * 8 + 2], v[ch * 8 + 3]), pack_bf16(v[ch * 8 + 4], v[ch * 8 + 5]),
               pack_bf16(v[ch * 8 + 6], v[ch * 8 + 7]));
      }
    }
    tc::wait_st();
    tc::fence_proxy_async_smem();
    tc::fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(pass2);

    // The state is kept as S = lam * St: the per-chunk decay gamma_C is folded into lam and
    // into the scale of Uh, and St is renormalised in tensor memory only when lam < 2^-64
    // (St then stays far inside the fp32 / bf16 exponent range).
    float lam = 1.f;
    for (int c = 0; c < p.n_chunks; ++c) {
      const int s = c & 1;
      const uint32_t z = (uint32_t)(c & 1) * 64;
      const int t0 = c * kC, nvalid = min(kC, p.T - t0);
      const uint8_t *stp = sm + s * L::kStage;
      const float *F = reinterpret_cast<const float *>(stp + L::sF);
      const float lam_c = lam;  // S = lam_c * St during this chunk's first MMAs
      // ---- pass 1: tokens 32*half .. +31 of U ----
      const bool w1 = mbar_wait(mmaU, c & 1, p.status);
      if (!__all_sync(0xffffffffu, w1)) break;
      tc::fence_after();
      {
        uint32_t y[32];
        tc::ld32(tl + cY + half * 32, y);
        float lam_new = lam_c * F[63];
        float coef;
        if (lam_new < 5.421010862427522e-20f) {  // 2^-64: renormalise St (this thread's 64 columns)
          uint32_t sv[2][32];
          tc::ld32(tl + cS + half * 64, sv[0]);
          tc::ld32(tl + cS + half * 64 + 32, sv[1]);
          tc::wait_ld();
          tc::regfence(sv[0]);
          tc::regfence(sv[1]);
#pragma unroll
          for (int c2 = 0; c2 < 2; ++c2) {
            float f[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(sv[c2][i]) * lam_new;
            tc::st32(tl + cS + half * 64 + c2 * 32, f);
          }
          lam_new = 1.f;
          coef = 1.f;
        } else {
          coef = 1.f / lam_new;
        }
        lam = lam_new;
        tc::wait_ld();
        tc::regfence(y);
        const uint8_t *urow = stp + L::sU + r * 128;  // 128-byte swizzled row of U'^T
        const float4 *f4 = reinterpret_cast<const float4 *>(F + 64 + half * 32);
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const uint4 uu = *reinterpret_cast<const uint4 *>(urow + (((half * 4 + ch) ^ (r & 7)) << 4));
          const float4 fa = f4[2 * ch], fb = f4[2 * ch + 1];
          const uint32_t uw[4] = {uu.x, uu.y, uu.z, uu.w};
          const float fv[8] = {fa.x, fa.y, fa.z, fa.w, fb.x, fb.y, fb.z, fb.w};
          uint32_t pu[4], ph[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int tt = ch * 8 + 2 * e;
            const float u0 = fmaf(lam_c, __uint_as_float(y[tt]), bf16_lo(uw[e]));
            const float u1 = fmaf(lam_c, __uint_as_float(y[tt + 1]), bf16_hi(uw[e]));
            pu[e] = pack_bf16(u0, u1);
            ph[e] = pack_bf16(u0 * fv[2 * e] * coef, u1 * fv[2 * e + 1] * coef);
          }
          const uint32_t off = r * 128 + (((half * 4 + ch) ^ (r & 7)) << 4);
          sts128(sUt + off, pu[0], pu[1], pu[2], pu[3]);
          sts128(sUh + off, ph[0], ph[1], ph[2], ph[3]);
        }
        tc::wait_st();
      }
      tc::fence_proxy_async_smem();
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(pass1);
      // ---- pass 2a: bf16 copy of the updated St (this thread's 64 columns) ----
      const bool w2 = mbar_wait(mmaS, c & 1, p.status);
      if (!__all_sync(0xffffffffu, w2)) break;
      tc::fence_after();
      {
        uint32_t sv[2][32];
        tc::ld32(tl + cS + half * 64, sv[0]);
        tc::ld32(tl + cS + half * 64 + 32, sv[1]);
        tc::wait_ld();
        tc::regfence(sv[0]);
        tc::regfence(sv[1]);
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2)
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            const int kc = half * 64 + c2 * 32 + ch * 8;
            const uint32_t *v = sv[c2] + ch * 8;
            sts128(sS + (kc >> 6) * 16384 + r * 128 + ((((kc & 63) >> 3) ^ (r & 7)) << 4),
                   pack_bf16(__uint_as_float(v[0]), __uint_as_float(v[1])),
                   pack_bf16(__uint_as_float(v[2]), __uint_as_float(v[3])),
                   pack_bf16(__uint_as_float(v[4]), __uint_as_float(v[5])),
                   pack_bf16(__uint_as_float(v[6]), __uint_as_float(v[7])));
          }
        tc::fence_proxy_async_smem();
        tc::fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(pass2);
        if (c + 1 == p.n_chunks && p.state_out) {
          float *so = p.state_out + st_base + (size_t)r * kDK + half * 64;
#pragma unroll
          for (int c2 = 0; c2 < 2; ++c2)
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4 *>(so + c2 * 32 + i) =
                  make_float4(lam * __uint_as_float(sv[c2][i]), lam * __uint_as_float(sv[c2][i + 1]),
                              lam * __uint_as_float(sv[c2][i + 2]), lam * __uint_as_float(sv[c2][i + 3]));
        }
      }
      // ---- pass 2b: outputs of tokens 32*half .. +31 (overlaps the next chunk's MMAs) ----
      const bool w3 = mbar_wait(mmaV, c & 1, p.status);
      if (!__all_sync(0xffffffffu, w3)) break;
      tc::fence_after();
      {
        uint32_t zv[32], vv[32];
        tc::ld32(tl + cZ + z + half * 32, zv);
        tc::ld32(tl + cV + z + half * 32, vv);
        tc::wait_ld();
        tc::regfence(zv);
        tc::regfence(vv);
        bf16_t *dst = p.o + (((size_t)b * p.T + t0 + half * 32) * p.h.v_heads + vh) * kDK + r;
        const size_t tstride = (size_t)p.h.v_heads * kDK;
        const float4 *g4 = reinterpret_cast<const float4 *>(F + half * 32);
        const float zs = p.scale * lam_c;
#pragma unroll
        for (int q8 = 0; q8 < 8; ++q8) {
          const float4 gg = g4[q8];
          const float gv[4] = {gg.x, gg.y, gg.z, gg.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = q8 * 4 + e;
            if (half * 32 + i < nvalid)
              dst[i * tstride] = f_to_bf16(fmaf(zs * gv[e], __uint_as_float(zv[i]), p.scale * __uint_as_float(vv[i])));
          }
        }
      }
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(outdone);
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
  return (size_t)B * n_heads * n_chunks * (kWBytes + kUBytes + kPBytes + kFBytes);
}

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
  const GdnWs ws = carve(a.workspace, a.B, a.n_heads, n_chunks);
  unsigned *status = device_status_ptr();

  // ---- inputs' tensor maps ----
  CUtensorMap tq, tk, tv, tw, tp, tu;
  const uint32_t box4[4] = {64, 1, (uint32_t)kC, 1};
  const uint64_t dq[4] = {(uint64_t)kDK, (uint64_t)a.qk_heads, (uint64_t)a.T, (uint64_t)a.B};
  const uint64_t sq[3] = {(uint64_t)kDK * 2, (uint64_t)a.qk_heads * kDK * 2, (uint64_t)a.T * a.qk_heads * kDK * 2};
  const uint64_t dv[4] = {(uint64_t)kDK, (uint64_t)a.v_heads, (uint64_t)a.T, (uint64_t)a.B};
  const uint64_t sv[3] = {(uint64_t)kDK * 2, (uint64_t)a.v_heads * kDK * 2, (uint64_t)a.T * a.v_heads * kDK * 2};
  const uint64_t rows = (uint64_t)a.B * a.n_heads * n_chunks * kC;
  const uint64_t dw[2] = {(uint64_t)kDK, rows}, sw[1] = {(uint64_t)kDK * 2};
  const uint64_t dp[2] = {(uint64_t)kC, rows}, sp[1] = {(uint64_t)kC * 2};
  const uint32_t box2[2] = {64, (uint32_t)kC};
  if (encode_tmap(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.q, dq, sq, box4, CU_TENSOR_MAP_SWIZZLE_128B) ||
      encode_tmap(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.k, dq, sq, box4, CU_TENSOR_MAP_SWIZZLE_128B) ||
      encode_tmap(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.v, dv, sv, box4, CU_TENSOR_MAP_SWIZZLE_128B) ||
      encode_tmap(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws.wn, dw, sw, box2, CU_TENSOR_MAP_SWIZZLE_128B) ||
      encode_tmap(&tp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws.pm, dp, sp, box2, CU_TENSOR_MAP_SWIZZLE_128B)) {
    set_error("gdn_chunk_fwd: cuTensorMapEncodeTiled failed");
    return cudaErrorInvalidValue;
  }

  // ---- phase 1: chunk-local products, all chunks in parallel ----
  PrepParams pp;
  memset(&pp, 0, sizeof(pp));
  pp.tm_q = tq;
  pp.tm_k = tk;
  pp.tm_v = tv;
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
  gdn_prep_kernel<<<dim3(n_chunks, a.n_heads, a.B), kPThreads, PrepSmem::kTotal, s>>>(pp);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  // ---- phase 2: the state scan on the tensor cores, one CTA per (sequence, head) ----
  {
    const uint64_t du[2] = {(uint64_t)kC, rows * 2}, su[1] = {(uint64_t)kC * 2};
    const uint32_t boxu[2] = {(uint32_t)kC, (uint32_t)kDK};
    if (encode_tmap(&tu, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws.up, du, su, boxu, CU_TENSOR_MAP_SWIZZLE_128B)) {
      set_error("gdn_chunk_fwd: cuTensorMapEncodeTiled failed (U')");
      return cudaErrorInvalidValue;
    }
  }
  ScanTcParams st;
  memset(&st, 0, sizeof(st));
  st.tm_q = tq;
  st.tm_k = tk;
  st.tm_w = tw;
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
  e = cudaFuncSetAttribute(gdn_scan_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, ScanTcSmem::kTotal);
  if (e != cudaSuccess) return e;
  gdn_scan_tc_kernel<<<dim3(a.n_heads, a.B), kTSThreads, ScanTcSmem::kTotal, s>>>(st);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (a.rms) {
    const long long n_rows = (long long)a.B * a.T * a.n_heads;
    gdn_rms_rows_kernel<<<(unsigned)((n_rows + 7) / 8), 256, 0, s>>>(a.o, a.B, a.T, h, a.eps);
    e = cudaGetLastError();
  }
  return e;
}
}  // namespace hh
