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
//   gdn_prep   parallel over (value head, chunk): K K^T and Q K^T, the triangular
//              inverse T = (I + A)^-1, W = T diag(beta gamma) K, U' = T diag(beta) V,
//              P and Qt on the 5th-generation tensor cores, written to a caller-
//              provided workspace (bf16 matrices, fp32 decay factors), each record
//              flagged once complete;
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
constexpr size_t kWBytes = (size_t)kC * kDK * 2;  // -W_e^T = -(diag(e) W)^T [128][64] bf16 (key rows, token columns)
constexpr size_t kUBytes = (size_t)kC * kDK * 2;  // U'^T [128][64] bf16 (d_v rows, token columns)
constexpr size_t kPBytes = (size_t)kC * kC * 2;   // P    [64][64]  bf16
constexpr size_t kQBytes = (size_t)kC * kDK * 2;  // Qt^T = (diag(gamma) Q - P W)^T [128][64] bf16
constexpr size_t kFBytes = (size_t)2 * kC * 4;    // gamma[64], e = exp(G_C - G)[64] fp32

struct GdnWs {
  bf16_t *wn, *up, *pm, *qt;  // [B, Hn, n_chunks] x (-W_e^T | U'^T | P | Qt^T)
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

struct Heads {
  int n_heads, group, qk_heads, v_heads, use_map;
  int map[kMaxMappedHeads];
  __device__ __forceinline__ int vh(int i) const { return use_map ? map[i] : i; }
  __device__ __forceinline__ int qh(int i) const { return use_map ? map[i] : i / group; }
};

// ============================================================================
// gdn_prep: one CTA per (head, chunk, sequence), heads fastest so that the records of
// chunk c complete before those of chunk c + 1.  Every product is a 5th-generation
// tensor-core MMA (tcgen05, accumulators in tensor memory, operands staged by TMA);
// the 64 x 64 unit lower-triangular inverse T = (I + A)^-1 is formed in fp32 on the
// CUDA cores, so that only its final entries are rounded to bf16.
//   MMA S1   [K ; Q] K^T  (M = 128: rows 0..63 K K^T, rows 64..127 Q K^T)
//   masks    A_ti = beta_t exp(G_t - G_i) k_t.k_i (i < t), P_ti = exp(G_t - G_i) q_t.k_i (i <= t)
//   inverse  the four 16 x 16 diagonal blocks by forward substitution, then the six
//            blocks below them, T_IJ = -T_II sum_{J <= K < I} A_IK T_KJ, diagonal by diagonal
//   MMA WU   W^T = K^T (T diag(beta gamma))^T,  U'^T = V^T (T diag(beta))^T
//   MMA D    D = W^T P^T  (W^T converted to bf16 in tensor memory: the A operand)
//   record   -W_e^T = -W^T diag(e), U'^T, P and Qt^T = Q^T diag(gamma) - D, all bf16,
//            transposed so that each tensor-memory lane writes one 128-byte row
// 8 warps: warp 0 issues the MMAs (one elected lane), thread 0 the TMA loads, thread 32 the
// TMA stores of the record and, once they have completed, its ready flag.
// ============================================================================
constexpr int kPW = 8;         // warps
constexpr int kPThreads = kPW * 32;

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
  // TMA tiles, 64 rows x 128 bytes per box.  K and Q boxes interleave so that rows 0..63 (K)
  // and 64..127 (Q) of each 64-column box form the M = 128 A operand [K ; Q] of MMA S1.
  static constexpr int oK0 = 0, oQ0 = 8192, oK1 = 16384, oQ1 = 24576;
  static constexpr int oV = 32768;              // V [64][128]: 2 boxes; later the U'^T staging tile
  static constexpr int oP = 49152;              // P [64 t][64 i] bf16
  static constexpr int oTw = 57344;             // T diag(beta gamma) [64 t][64 i] bf16; Tw|Tu later Qt^T
  static constexpr int oTu = 65536;             // T diag(beta) [64 t][64 i] bf16
  static constexpr int oA = 73728;              // A: the 10 lower 16 x 16 blocks, fp32; A|T later -W_e^T
  static constexpr int oT = oA + 10 * 1024;     // T: the 10 lower blocks, fp32
  static constexpr int oY = oT + 10 * 1024;     // Y: the 6 blocks below the diagonal, fp32
  static constexpr int oSmall = oY + 6 * 1024;  // G, beta, gamma, e, beta gamma [64] fp32; barriers; TMEM slot
  static constexpr int kTotal = oSmall + 5 * 256 + 64 + 1024;
};
static_assert(PrepSmem::oA + 16384 <= PrepSmem::oSmall, "-W_e^T staging fits over A | T | Y");
static_assert(2 * PrepSmem::kTotal <= 232448, "two CTAs per SM");

// lower 16 x 16 blocks of a 64 x 64 triangular matrix: (I, J), J <= I
__device__ __forceinline__ int lblk(int I, int J) { return I * (I + 1) / 2 + J; }
// blocks strictly below the diagonal: (I, J), J < I
__device__ __forceinline__ int oblk(int I, int J) { return I * (I - 1) / 2 + J; }

constexpr float kLog2eF = 1.4426950408889634f;

// bf16 element (t, i) of a [64][64] 128-byte-swizzled tile
__device__ __forceinline__ uint32_t sw_el(int t, int i) { return sw128(t, i >> 3) + (uint32_t)(i & 7) * 2u; }

__global__ void __launch_bounds__(kPThreads, 2) gdn_prep_kernel(const __grid_constant__ PrepParams p) {
  using L = PrepSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  float *Ab = reinterpret_cast<float *>(sm + L::oA);
  float *Tb = reinterpret_cast<float *>(sm + L::oT);
  float *Yb = reinterpret_cast<float *>(sm + L::oY);
  float *Gs = reinterpret_cast<float *>(sm + L::oSmall);
  float *Bs = Gs + 64, *Eg = Bs + 64, *Ee = Eg + 64, *BG = Ee + 64;  // Gs holds G log2(e)
  uint64_t *bars = reinterpret_cast<uint64_t *>(BG + 64);
  uint64_t *full = bars, *s1done = bars + 1, *wudone = bars + 2, *ddone = bars + 3, *fin = bars + 4;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 6);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hi = blockIdx.x, c = blockIdx.y, b = blockIdx.z;  // heads fastest: chunks complete in order
  const int vh = p.h.vh(hi), qh = p.h.qh(hi);
  const int t0 = c * kC, nvalid = min(kC, p.T - t0);
  const size_t rec = ((size_t)b * p.h.n_heads + hi) * p.n_chunks + c;
  const int wrow = (int)(rec * kC);  // first workspace row of this record (P); 2 * wrow for the [128][64] tiles

  if (threadIdx.x == 0) {
    for (int i = 0; i < 5; ++i) mbar_init(&bars[i], 1);
    fence_barrier_init();
    mbar_arrive_expect_tx(full, 6 * 8192);
    tma_load_4d(sb + L::oK0, &p.tm_k, full, 0, qh, t0, b);
    tma_load_4d(sb + L::oK1, &p.tm_k, full, 64, qh, t0, b);
    tma_load_4d(sb + L::oQ0, &p.tm_q, full, 0, qh, t0, b);
    tma_load_4d(sb + L::oQ1, &p.tm_q, full, 64, qh, t0, b);
    tma_load_4d(sb + L::oV, &p.tm_v, full, 0, vh, t0, b);
    tma_load_4d(sb + L::oV + 8192, &p.tm_v, full, 64, vh, t0, b);
  }
  if (warp == 0) {
    tc::tmem_alloc(smem_u32(tmem_slot), 128);
    tc::tmem_relinquish();
  }
  // gates -> G (in-chunk cumulative log decay), gamma = exp(G), e = exp(G_C - G), beta; padded tokens: g = beta = 0
  if (warp == 1) {
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
    const float GC = __shfl_sync(0xffffffffu, run, 31);
    const float gam0 = expf(g_lo), gam1 = expf(run), e0 = expf(GC - g_lo), e1 = expf(GC - run);
    Gs[2 * lane] = g_lo * kLog2eF;  // the masks take exp(G_t - G_i) as exp2 of the scaled difference
    Gs[2 * lane + 1] = run * kLog2eF;
    Eg[2 * lane] = gam0;
    Eg[2 * lane + 1] = gam1;
    Ee[2 * lane] = e0;
    Ee[2 * lane + 1] = e1;
    Bs[2 * lane] = bv[0];
    Bs[2 * lane + 1] = bv[1];
    BG[2 * lane] = bv[0] * gam0;
    BG[2 * lane + 1] = bv[1] * gam1;
    // decay factors for the scan: gamma_t and exp(G_C - G_t)
    *reinterpret_cast<float2 *>(p.ws.fc + rec * 128 + 2 * lane) = make_float2(gam0, gam1);
    *reinterpret_cast<float2 *>(p.ws.fc + rec * 128 + 64 + 2 * lane) = make_float2(e0, e1);
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tbase = *tmem_slot;
  // tensor memory: S1 / U'^T / D in columns 0..63, W^T in 64..127 (its bf16 copy in 64..95)
  constexpr uint32_t cS = 0, cW = 64;

  // ---- MMA S1 = [K ; Q] K^T ----
  bool ok = true;
  if (warp == 0) {
    ok = __all_sync(0xffffffffu, mbar_wait(full, 0, p.status));
    if (ok) {
      tc::fence_after();
      const uint64_t d0 = tc::desc_kmajor_sw128(sb + L::oK0), d1 = tc::desc_kmajor_sw128(sb + L::oK1);
      constexpr uint32_t id = tc::idesc_bf16_f32(128, 64, 0, 0);
#pragma unroll
      for (int ks = 0; ks < kDK / 16; ++ks) {
        const uint64_t d = (ks < 4 ? d0 : d1) + (uint32_t)(ks & 3) * 2u;
        tc::mma_ss_w(tbase + cS, d, d, id, ks ? 1u : 0u);
      }
      tc::commit_w(s1done);
    }
  }

  // ---- masks: warp w reads TMEM lane quarter w % 4 (quarters 0-1: K K^T rows -> A, fp32 blocks;
  // quarters 2-3: Q K^T rows -> P, bf16) and the 32 columns 32 (w / 4) .. + 31 of its rows.
  // exp(G_t - G_i) is formed only where i <= t (elsewhere the difference is positive) ----
  {
    const bool w = mbar_wait(s1done, 0, p.status);
    if (__all_sync(0xffffffffu, w)) {
      tc::fence_after();
      const int q4 = warp & 3, ch = warp >> 2;  // column half: keys i = 32 ch .. 32 ch + 31
      uint32_t r0[32];
      tc::ld32(tbase + ((uint32_t)(q4 * 32) << 16) + cS + ch * 32, r0);
      tc::wait_ld();
      tc::regfence(r0);
      const int t = (q4 & 1) * 32 + lane;
      const float Gt = Gs[t];
      if (q4 < 2) {
        const float bt = Bs[t];
        const int I = t >> 4, r = t & 15;
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int J = 2 * ch + jj;  // 16-column block of A
          if (J <= I) {
            float a[16];
#pragma unroll
            for (int m = 0; m < 16; ++m) {
              const int i = 16 * J + m;
              a[m] = i < t ? bt * exp2f(Gt - Gs[i]) * __uint_as_float(r0[16 * jj + m]) : 0.f;
            }
            float4 *dst = reinterpret_cast<float4 *>(Ab + lblk(I, J) * 256 + r * 16);
#pragma unroll
            for (int q = 0; q < 4; ++q) dst[q] = make_float4(a[4 * q], a[4 * q + 1], a[4 * q + 2], a[4 * q + 3]);
          }
        }
      } else {
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int i = 32 * ch + 2 * j;
          const float q0 = __uint_as_float(r0[2 * j]), q1 = __uint_as_float(r0[2 * j + 1]);
          pk[j] = pack_bf16(i <= t ? exp2f(Gt - Gs[i]) * q0 : 0.f, i + 1 <= t ? exp2f(Gt - Gs[i + 1]) * q1 : 0.f);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j)
          *reinterpret_cast<uint4 *>(sm + L::oP + sw128(t, 4 * ch + j)) =
              make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
      }
    } else {
      ok = false;
    }
  }
  tc::fence_before();
  tc::fence_proxy_async_smem();  // P: TMA store source and MMA D operand
  if (__syncthreads_or(!ok)) goto drain;
  tc::fence_after();
  // every record store is issued by thread 32 (warp 1), which waits for all of them before it flags the record
  if (threadIdx.x == 32) {
    tma_store_2d(&p.tm_p, sb + L::oP, 0, wrow);
    bulk_commit();
  }

  // ---- T = (I + A)^-1 in fp32, 16 x 16 blocks ----
  {
    const int tid = threadIdx.x;
    // diagonal blocks: thread (I, cc) forms column cc of (I + A_II)^-1 by forward substitution
    // (entries above the diagonal stay 0: multiplying by them changes nothing).  The other
    // threads zero the blocks of Tw / Tu above the diagonal.
    if (tid < 64) {
      const int I = tid >> 4, cc = tid & 15;
      const float *a = Ab + lblk(I, I) * 256;
      float x[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) x[r] = r == cc ? 1.f : 0.f;
#pragma unroll
      for (int r = 0; r < 16; ++r)
#pragma unroll
        for (int u = r + 1; u < 16; ++u) x[u] = fmaf(-a[u * 16 + r], x[r], x[u]);
      float *tb = Tb + lblk(I, I) * 256;
      const int i = 16 * I + cc;
      const float sw = BG[i], su = Bs[i];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        tb[r * 16 + cc] = x[r];
        *reinterpret_cast<bf16_t *>(sm + L::oTw + sw_el(16 * I + r, i)) = f_to_bf16(x[r] * sw);
        *reinterpret_cast<bf16_t *>(sm + L::oTu + sw_el(16 * I + r, i)) = f_to_bf16(x[r] * su);
      }
    } else {
      // rows 0..47 of each tile have blocks above the diagonal: row t (block row I = t / 16) is zero
      // from column 16 (I + 1) on, i.e. 16-byte chunks 2 (I + 1) .. 7
      const int k = tid - 64;
      if (k < 96) {
        const int t = k % 48, I = t >> 4;
        uint8_t *row = sm + (k < 48 ? L::oTw : L::oTu);
        for (int c8 = 2 * (I + 1); c8 < 8; ++c8) *reinterpret_cast<uint4 *>(row + sw128(t, c8)) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    __syncthreads();
    const int r = tid >> 4, cc = tid & 15;  // element (r, cc) of a 16 x 16 block
    // row r of block X times column cc of block Y (16 x 16 fp32 blocks), two partial sums
    auto rowcol = [&](const float *X, const float *Y) {
      const float4 *x4 = reinterpret_cast<const float4 *>(X + r * 16);
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 xv = x4[q];
        s0 = fmaf(xv.x, Y[(4 * q) * 16 + cc], s0);
        s1 = fmaf(xv.y, Y[(4 * q + 1) * 16 + cc], s1);
        s0 = fmaf(xv.z, Y[(4 * q + 2) * 16 + cc], s0);
        s1 = fmaf(xv.w, Y[(4 * q + 3) * 16 + cc], s1);
      }
      return s0 + s1;
    };
    // Y_IJ = A_IJ T_JJ for the six blocks below the diagonal
#pragma unroll
    for (int I = 1; I < 4; ++I)
#pragma unroll
      for (int J = 0; J < I; ++J) Yb[oblk(I, J) * 256 + r * 16 + cc] = rowcol(Ab + lblk(I, J) * 256, Tb + lblk(J, J) * 256);
    __syncthreads();
    // T_IJ = -T_II Y_IJ (with Y_IJ complete), written with its bf16 copies
    auto finish = [&](int I, int J) {
      const float tv = -rowcol(Tb + lblk(I, I) * 256, Yb + oblk(I, J) * 256);
      Tb[lblk(I, J) * 256 + r * 16 + cc] = tv;
      const int t = 16 * I + r, i = 16 * J + cc;
      *reinterpret_cast<bf16_t *>(sm + L::oTw + sw_el(t, i)) = f_to_bf16(tv * BG[i]);
      *reinterpret_cast<bf16_t *>(sm + L::oTu + sw_el(t, i)) = f_to_bf16(tv * Bs[i]);
    };
    // Y_IJ += A_IK T_KJ
    auto accumulate = [&](int I, int K, int J) {
      Yb[oblk(I, J) * 256 + r * 16 + cc] += rowcol(Ab + lblk(I, K) * 256, Tb + lblk(K, J) * 256);
    };
    // Two levels of the 2 x 2 block inverse: within each 32-row half (T_10, T_32, and T_21 with
    // them), then the lower-left 32 x 32 block,
    //     -[T_22 0; T_32 T_33] [Y_20 + A_21 T_10, Y_21; Y_30 + A_31 T_10, Y_31]
    auto store_T = [&](int I, int J, float tv) {
      Tb[lblk(I, J) * 256 + r * 16 + cc] = tv;
      const int t = 16 * I + r, i = 16 * J + cc;
      *reinterpret_cast<bf16_t *>(sm + L::oTw + sw_el(t, i)) = f_to_bf16(tv * BG[i]);
      *reinterpret_cast<bf16_t *>(sm + L::oTu + sw_el(t, i)) = f_to_bf16(tv * Bs[i]);
    };
    finish(1, 0);
    finish(2, 1);
    finish(3, 2);
    __syncthreads();
    accumulate(2, 1, 0);  // Y_20 = A_20 T_00 + A_21 T_10
    accumulate(3, 1, 0);  // Y_30 = A_30 T_00 + A_31 T_10
    store_T(3, 1, -(rowcol(Tb + lblk(3, 2) * 256, Yb + oblk(2, 1) * 256) + rowcol(Tb + lblk(3, 3) * 256, Yb + oblk(3, 1) * 256)));
    __syncthreads();
    finish(2, 0);         // T_20 = -T_22 Y_20
    store_T(3, 0, -(rowcol(Tb + lblk(3, 2) * 256, Yb + oblk(2, 0) * 256) + rowcol(Tb + lblk(3, 3) * 256, Yb + oblk(3, 0) * 256)));
  }
  tc::fence_proxy_async_smem();  // Tw, Tu: MMA operands
  __syncthreads();

  // ---- MMA WU: W^T = K^T Tw^T -> columns 64..127, U'^T = V^T Tu^T -> columns 0..63 ----
  if (warp == 0) {
    tc::fence_after();
    const uint64_t dKt = tc::desc_mnmajor_sw128(sb + L::oK0, L::oK1 - L::oK0, 1024);
    const uint64_t dVt = tc::desc_mnmajor_sw128(sb + L::oV, 8192, 1024);
    const uint64_t dTw = tc::desc_kmajor_sw128(sb + L::oTw), dTu = tc::desc_kmajor_sw128(sb + L::oTu);
    constexpr uint32_t id = tc::idesc_bf16_f32(128, 64, 1, 0);
#pragma unroll
    for (int ks = 0; ks < kC / 16; ++ks) tc::mma_ss_w(tbase + cW, dKt + ks * 128, dTw + ks * 2, id, ks ? 1u : 0u);
#pragma unroll
    for (int ks = 0; ks < kC / 16; ++ks) tc::mma_ss_w(tbase + cS, dVt + ks * 128, dTu + ks * 2, id, ks ? 1u : 0u);
    tc::commit_w(wudone);
  }
  // ---- passes: W^T -> bf16 in place (A of MMA D) and -W_e^T; U'^T -> bf16 (staging tiles) ----
  {
    const bool w = mbar_wait(wudone, 0, p.status);
    ok = __all_sync(0xffffffffu, w);
    if (ok) {
      tc::fence_after();
      const int q4 = warp & 3, row = q4 * 32 + lane;
      const uint32_t tl = tbase + ((uint32_t)(q4 * 32) << 16);
      uint32_t r0[32], r1[32], pk[32];
      tc::ld32(tl + (warp < 4 ? cW : cS), r0);
      tc::ld32(tl + (warp < 4 ? cW : cS) + 32, r1);
      tc::wait_ld();
      tc::regfence(r0);
      tc::regfence(r1);
      if (warp < 4) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          pk[j] = pack_bf16(__uint_as_float(r0[2 * j]), __uint_as_float(r0[2 * j + 1]));
          pk[16 + j] = pack_bf16(__uint_as_float(r1[2 * j]), __uint_as_float(r1[2 * j + 1]));
        }
        tc::st32u(tl + cW, pk);
        tc::wait_st();  // pk is reused below
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          pk[j] = pack_bf16(-Ee[2 * j] * __uint_as_float(r0[2 * j]), -Ee[2 * j + 1] * __uint_as_float(r0[2 * j + 1]));
          pk[16 + j] = pack_bf16(-Ee[32 + 2 * j] * __uint_as_float(r1[2 * j]),
                                 -Ee[33 + 2 * j] * __uint_as_float(r1[2 * j + 1]));
        }
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          pk[j] = pack_bf16(__uint_as_float(r0[2 * j]), __uint_as_float(r0[2 * j + 1]));
          pk[16 + j] = pack_bf16(__uint_as_float(r1[2 * j]), __uint_as_float(r1[2 * j + 1]));
        }
      }
      uint8_t *dst = sm + (warp < 4 ? L::oA : L::oV) + row * 128;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        *reinterpret_cast<uint4 *>(dst + ((j ^ (row & 7)) << 4)) = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
    }
  }
  tc::fence_before();
  tc::fence_proxy_async_smem();
  if (__syncthreads_or(!ok)) goto drain;
  tc::fence_after();
  // ---- MMA D = W^T P^T -> columns 0..63; the -W_e^T and U'^T records leave ----
  if (warp == 0) {
    const uint64_t dP = tc::desc_kmajor_sw128(sb + L::oP);
    constexpr uint32_t id = tc::idesc_bf16_f32(128, 64, 0, 0);
#pragma unroll
    for (int ks = 0; ks < kC / 16; ++ks) tc::mma_ts_w(tbase + cS, tbase + cW + ks * 8, dP + ks * 2, id, ks ? 1u : 0u);
    tc::commit_w(ddone);
  } else if (threadIdx.x == 32) {
    tma_store_2d(&p.tm_w, sb + L::oA, 0, 2 * wrow);
    tma_store_2d(&p.tm_u, sb + L::oV, 0, 2 * wrow);
    bulk_commit();
  }
  // ---- Qt^T = Q^T diag(gamma) - D: warp w takes rows 32 (w % 4) .., token half w / 4 ----
  {
    const bool w = mbar_wait(ddone, 0, p.status);
    ok = __all_sync(0xffffffffu, w);
    if (ok) {
      tc::fence_after();
      const int q4 = warp & 3, half = warp >> 2, d = q4 * 32 + lane;
      uint32_t r0[32], pk[16];
      tc::ld32(tbase + ((uint32_t)(q4 * 32) << 16) + cS + half * 32, r0);
      tc::wait_ld();
      tc::regfence(r0);
      const uint8_t *qcol = sm + (d < 64 ? L::oQ0 : L::oQ1) + (d & 7) * 2;
      const int dc = (d & 63) >> 3;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int t = half * 32 + 2 * j;
        const float q0 = bf16_to_f(*reinterpret_cast<const bf16_t *>(qcol + sw128(t, dc)));
        const float q1 = bf16_to_f(*reinterpret_cast<const bf16_t *>(qcol + sw128(t + 1, dc)));
        pk[j] = pack_bf16(fmaf(Eg[t], q0, -__uint_as_float(r0[2 * j])), fmaf(Eg[t + 1], q1, -__uint_as_float(r0[2 * j + 1])));
      }
      uint8_t *dst = sm + L::oTw + d * 128;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int ch = half * 4 + j;
        *reinterpret_cast<uint4 *>(dst + ((ch ^ (d & 7)) << 4)) = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
      }
    }
  }
  tc::fence_before();
  tc::fence_proxy_async_smem();
  if (__syncthreads_or(!ok)) goto drain;
  if (threadIdx.x == 32) {
    tma_store_2d(&p.tm_qt, sb + L::oTw, 0, 2 * wrow);
    bulk_commit();
    bulk_wait_all();
    asm volatile("fence.proxy.async.global;\n" ::: "memory");
    asm volatile("st.release.gpu.global.u32 [%0], %1;\n" ::"l"(p.ws.flag + rec), "r"(1u) : "memory");
  }

drain:
  // every MMA issued above has completed and every load has landed before tensor memory is
  // released and the CTA exits (bounded; already true on the normal path)
  if (warp == 0) {
    tc::commit_w(fin);
    mbar_wait(fin, 0, p.status);
    if (lane == 0) mbar_wait(full, 0, p.status);
  }
  if (threadIdx.x == 32) bulk_wait_all();
  tc::fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after();
    tc::tmem_dealloc(tbase, 128);
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
  CUtensorMap tm_p;               // workspace P [rows][64], box (64, 64)
  CUtensorMap tm_w, tm_u, tm_qt;  // workspace -W_e^T, U'^T, Qt^T [2 rows][64], box (64, 128)
  GdnWs ws;
  const float *state_in;
  float *state_out;
  bf16_t *o;
  int B, T, n_chunks;
  Heads h;
  float scale;
  int rms;    // 1: each output row (token, head) leaves RMS-normalised, y = o / sqrt(mean(o^2) + eps)
  float eps;
  float *chunk_states;  // nullable: [B, n_heads, n_chunks, d_k, d_v] fp32, S^T at the start of every chunk
  unsigned *status;
};

// kRms (the head-level hybrid layer's delta-rule heads): each output row leaves RMS-normalised.
// That normalisation divides by the row's norm, so it scales up the absolute error of rows whose
// norm is small; for them the state enters the output product as two bf16 terms, S = S_hi + S_lo
// (the second copy, S_lo^T, takes the place of one ring-B slot).
template <bool kRms>
struct ScanSmem {
  static constexpr int kBSlots = kRms ? 2 : 3;
  // ring A (2 slots): -W_e^T and K of a chunk, used one chunk ahead (MMA M, conversion)
  static constexpr int kASlot = 32768, oA = 0, aW = 0, aK = 16384;
  // ring B (kBSlots slots): U'^T, Qt^T and P of a chunk (MMA S, MMA O)
  static constexpr int kBSlot = 40960, oB = oA + 2 * kASlot, bU = 0, bQ = 16384, bP = 32768;
  static constexpr int oS = oB + kBSlots * kBSlot;  // bf16 S^T [128 k][128 v], MN-major: 2 boxes of 64 v
  static constexpr int oSlo = oS + 32768;           // kRms: bf16 (S^T - S^T_hi), same layout
  static constexpr int oE = oSlo + (kRms ? 32768 : 0);  // fp32 e[2][64] (ring A), gamma[3][64] (ring B)
  static constexpr int oBar = oE + 5 * 256;
  static constexpr int oR = oBar + 256;        // RMS partial sums [2 chunk parities][2 token halves][4 lane quarters][32]
  static constexpr int kTotal = oR + 2048 + 1024;
};
static_assert(ScanSmem<false>::kTotal <= 232448 && ScanSmem<true>::kTotal <= 232448, "shared memory budget");

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

template <bool kRms>
__global__ void __launch_bounds__(kSThreads, 1) gdn_scan_kernel(const __grid_constant__ ScanParams p) {
  using L = ScanSmem<kRms>;
  constexpr int kB = L::kBSlots;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::oBar);
  uint64_t *fullA = bars, *fullB = bars + 2, *mdone = bars + 5, *mready = bars + 7, *passd = bars + 9,
           *chaind = bars + 10, *odoneS = bars + 11, *odone = bars + 12, *ofree = bars + 14, *fin = bars + 16,
           *bfree = bars + 17;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 20);
  uint64_t *rmsbar = bars + 22;  // [2 chunk parities][2 token halves], 4 arrivals (one per lane quarter)
  float *rms_part = reinterpret_cast<float *>(sm + L::oR);
  float *eA = reinterpret_cast<float *>(sm + L::oE);  // [2][64]
  float *gB = eA + 128;                                // [kB][64]
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
    for (int i = 0; i < kB; ++i) {
      mbar_init(&fullB[i], 1);
      mbar_init(&bfree[i], 1);
    }
    for (int i = 0; i < 4; ++i) mbar_init(&rmsbar[i], 4);
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
    const uint64_t dW = tc::desc_kmajor_sw128(sA + L::aW);                  // -W_e^T: key rows, token columns
    const uint64_t dS = tc::desc_mnmajor_sw128(sS, 16384, 1024);  // B of MMA S, A of MMA O
    const uint64_t dU = tc::desc_kmajor_sw128(sB + L::bU);
    const uint64_t dQ = tc::desc_mnmajor_sw128(sB + L::bQ, 8192, 1024);     // Qt^T: key rows, token columns
    const uint64_t dP = tc::desc_kmajor_sw128(sB + L::bP);
    constexpr uint32_t idM = tc::idesc_bf16_f32(128, 128, 1, 0);   // K^T MN-major, -W_e from -W_e^T K-major
    constexpr uint32_t idS1 = tc::idesc_bf16_f32(128, 128, 0, 1);  // A in TMEM, S^T_bf16 MN-major
    constexpr uint32_t idS2 = tc::idesc_bf16_f32(128, 128, 0, 0);  // A in TMEM, U'^T K-major
    constexpr uint32_t idO1 = tc::idesc_bf16_f32(128, 64, 1, 1);   // S (MN-major from S^T), Qt from Qt^T MN-major
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
          tc::mma_ss_w(tbase + cM + s * 128, dK + o + ks * 128, dW + o + ks * 2, idM, ks ? 1u : 0u);
        tc::commit_w(&mdone[s]);
      }
      return true;
    };
    bool ok = n > 0 && mmaM(0);
    for (int c = 0; c < n && ok; ++c) {
      const int s2 = c & 1, s3 = c % kB;
      // M of the next chunk, into the buffer MMA S of chunk c - 1 has finished reading
      if (c >= 1 && !wait_all(chaind, (c - 1) & 1)) break;
      if (c + 1 < n && !mmaM(c + 1)) break;
      // MMA S (the chain): S^T += [-M_c^T | Kh^T] [S^T_bf16 ; U']
      if (!wait_all(&mready[s2], (c >> 1) & 1)) break;
      if (!wait_all(passd, c & 1)) break;
      if (!wait_all(&fullB[s3], (c / kB) & 1)) break;
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
        for (int ks = 0; ks < kDK / 16; ++ks) tc::mma_ss_w(dO, dS + ks * 128, dQ + ob + ks * 128, idO1, ks ? 1u : 0u);
        if (kRms) {
          const uint64_t dSlo = tc::desc_mnmajor_sw128(sS + (L::oSlo - L::oS), 16384, 1024);
#pragma unroll
          for (int ks = 0; ks < kDK / 16; ++ks) tc::mma_ss_w(dO, dSlo + ks * 128, dQ + ob + ks * 128, idO1, 1u);
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
          tma_load_2d(dst + L::aW, &p.tm_w, &fullA[s], 0, 2 * row);
          tma_load_4d(dst + L::aK, &p.tm_k, &fullA[s], 0, qh, c * kC, b);
          tma_load_4d(dst + L::aK + 8192, &p.tm_k, &fullA[s], 64, qh, c * kC, b);
          bulk_load(smem_u32(eA + s * 64), p.ws.fc + (rec0 + c) * 128 + 64, 256, &fullA[s]);
          lastA = c;
        }
        // ring B slot: free once MMA O of chunk c - 3 has completed
        if (c >= kB && !mbar_wait(&bfree[c % kB], ((c - kB) / kB) & 1, p.status)) break;
        {
          const int s = c % kB;
          mbar_arrive_expect_tx(&fullB[s], 2 * 16384 + 8192 + 256);
          const uint32_t dst = sB + s * L::kBSlot;
          const int row = (int)((rec0 + c) * kC);
          tma_load_2d(dst + L::bU, &p.tm_u, &fullB[s], 0, 2 * row);
          tma_load_2d(dst + L::bQ, &p.tm_qt, &fullB[s], 0, 2 * row);
          tma_load_2d(dst + L::bP, &p.tm_p, &fullB[s], 0, row);
          bulk_load(smem_u32(gB + s * 64), p.ws.fc + (rec0 + c) * 128, 256, &fullB[s]);
          lastB = c;
        }
      }
      // every load issued above has landed before the CTA can exit (bounded; complete on the
      // normal path, where the consumers waited for each of them)
      for (int c = max(lastA - 1, 0); c <= lastA; ++c) mbar_wait(&fullA[c & 1], (c >> 1) & 1, p.status);
      for (int c = max(lastB - (kB - 1), 0); c <= lastB; ++c) mbar_wait(&fullB[c % kB], (c / kB) & 1, p.status);
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
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ofree[s2]);  // the O buffer is free once read
      const int t0 = c * kC + half * 32, nv = min(32, p.T - t0);
      bf16_t *dst = p.o + (((size_t)b * p.T + t0) * p.h.v_heads + vh) * kDK + nrow;
      const size_t tstride = (size_t)p.h.v_heads * kDK;
      float x[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) x[i] = p.scale * __uint_as_float(ov[i]);
      if (kRms) {
        // Sum of squares over the 128 values of each token: a butterfly over the warp leaves lane l
        // with its 32 values' share for token l; the four lane quarters then add their shares.
        float a[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) a[i] = x[i] * x[i];
#pragma unroll
        for (int o = 16, n = 16; o >= 1; o >>= 1, n >>= 1) {
          const bool up = (lane & o) != 0;
#pragma unroll
          for (int j = 0; j < n; ++j) {
            const float send = up ? a[j] : a[j + n], keep = up ? a[j + n] : a[j];
            a[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
          }
        }
        float *part = rms_part + ((c & 1) * 2 + half) * 128;
        part[q4 * 32 + lane] = a[0];
        __syncwarp();
        uint64_t *rb = &rmsbar[(c & 1) * 2 + half];
        if (lane == 0) mbar_arrive(rb);
        const bool w2 = mbar_wait(rb, (c >> 1) & 1, p.status);
        if (!__all_sync(0xffffffffu, w2)) return false;
        const float ss = part[lane] + part[32 + lane] + part[64 + lane] + part[96 + lane];
        const float inv = rsqrtf(ss * (1.f / kDK) + p.eps);
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] *= __shfl_sync(0xffffffffu, inv, i);
      }
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (i < nv) dst[i * tstride] = f_to_bf16(x[i]);
      return true;
    };
    bool ok = true;
    for (int c = 0; c < n; ++c) {
      const int s3 = c % kB;
      {
        bool w = c == 0 || mbar_wait(chaind, (c - 1) & 1, p.status);
        w = w && mbar_wait(&fullB[s3], (c / kB) & 1, p.status);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        tc::fence_after();
      }
      const float gC = gB[s3 * 64 + kC - 1];
      uint32_t pk[32], plo[kRms ? 32 : 1];
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
        if (p.chunk_states) {  // the state at the chunk's start, for a backward pass: S^T row n
          float4 *cs = reinterpret_cast<float4 *>(p.chunk_states + ((rec0 + c) * kDK + nrow) * kDK + v0);
#pragma unroll
          for (int i = 0; i < 8; ++i) cs[i] = make_float4(f[4 * i], f[4 * i + 1], f[4 * i + 2], f[4 * i + 3]);
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[h * 16 + i] = pack_bf16(f[2 * i], f[2 * i + 1]);
        if (kRms) {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            plo[h * 16 + i] = pack_bf16(f[2 * i] - bf16_lo(pk[h * 16 + i]), f[2 * i + 1] - bf16_hi(pk[h * 16 + i]));
        }
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
      if (kRms) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          sts128(srow + (L::oSlo - L::oS) + ((j ^ (nrow & 7)) << 4), plo[4 * j], plo[4 * j + 1], plo[4 * j + 2], plo[4 * j + 3]);
      }
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
  const uint64_t dp[2] = {(uint64_t)kC, rows}, sp[1] = {(uint64_t)kC * 2};
  const uint32_t box2[2] = {64, (uint32_t)kC};
  const uint64_t du[2] = {(uint64_t)kC, rows * 2}, su[1] = {(uint64_t)kC * 2};
  const uint32_t boxu[2] = {(uint32_t)kC, (uint32_t)kDK};
  if (encode_tmap(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.q, dq, sq, box4, CU_TENSOR_MAP_SWIZZLE_128B) ||
      encode_tmap(&tu, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws.up, du, su, boxu, CU_TENSOR_MAP_SWIZZLE_128B) ||
      encode_tmap(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.k, dq, sq, box4, CU_TENSOR_MAP_SWIZZLE_128B) ||
      encode_tmap(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.v, dv, sv, box4, CU_TENSOR_MAP_SWIZZLE_128B) ||
      encode_tmap(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws.wn, du, su, boxu, CU_TENSOR_MAP_SWIZZLE_128B) ||
      encode_tmap(&tqt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws.qt, du, su, boxu, CU_TENSOR_MAP_SWIZZLE_128B) ||
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
  st.rms = a.rms;
  st.eps = a.eps;
  st.chunk_states = a.chunk_states;
  st.status = status;
  auto scan_kernel = a.rms ? gdn_scan_kernel<true> : gdn_scan_kernel<false>;
  const int scan_smem = a.rms ? ScanSmem<true>::kTotal : ScanSmem<false>::kTotal;
  e = cudaFuncSetAttribute(scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, scan_smem);
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
      scan_kernel<<<dim3(a.n_heads, a.B), kSThreads, scan_smem, s>>>(st);
      return cudaGetLastError();
    }
    std::lock_guard<std::mutex> lock(g_prep_mu);
    PrepStream &ps = g_prep[dev];
    if (!ps.lo) {
      int lo_pri = 0, hi_pri = 0;
      // the scan at the highest priority (its CTAs start at once); gdn_prep one step below it, above
      // the caller's work: records must stay ahead of the scan when other kernels (the head-level
      // hybrid's softmax heads) share the GPU, or the sequential scan waits on them
      if ((e = cudaDeviceGetStreamPriorityRange(&lo_pri, &hi_pri)) != cudaSuccess ||
          (e = cudaStreamCreateWithPriority(&ps.hi, cudaStreamNonBlocking, hi_pri)) != cudaSuccess ||
          (e = cudaStreamCreateWithPriority(&ps.lo, cudaStreamNonBlocking, hi_pri < lo_pri ? hi_pri + 1 : lo_pri)) !=
              cudaSuccess ||
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
    scan_kernel<<<dim3(a.n_heads, a.B), kSThreads, scan_smem, ps.hi>>>(st);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = cudaEventRecord(ps.join_lo, ps.lo)) != cudaSuccess || (e = cudaEventRecord(ps.join_hi, ps.hi)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(s, ps.join_lo, 0)) != cudaSuccess || (e = cudaStreamWaitEvent(s, ps.join_hi, 0)) != cudaSuccess)
      return e;
  }
  return cudaSuccess;
}
}  // namespace hh
