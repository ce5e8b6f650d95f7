// attn_fwd_tc.cu -- causal grouped-query softmax attention (prefill) at head dim 128
// on the 5th-generation tensor cores (tcgen05, accumulators in tensor memory).
//
// What is computed is the same as in attn_fwd.cu: per query head and position,
//   o_t = sum_{j<=t} exp(s_tj - m_t) v_j / sum_j exp(s_tj - m_t),  s_tj = scale q_t.k_j,
// then o_t *= sigmoid(G_t) for a gated layer, or the per-head RMS fusion of the
// head-level hybrid layer.  The FA heads of the HydraHead layer use head dim 128;
// the d = 256 attention layers run on CTA pairs (attn_fwd_tc2.cu).
//
// CTA = one tile of 128 query rows of one head, eighteen warps:
//   warp 0      TMA producer: Q once, then K and V of every 128-key tile through a
//               ring of four 32 KiB stages, 128-byte swizzle, rows past T zero-filled;
//   warp 1      allocates tensor memory and runs the MMA loop as a whole warp, one lane
//               chosen by elect.sync issuing (the descriptors stay warp-uniform):
//               S = Q K^T (M=128, N=128, bf16 K-major operands) and O += P V (M=128,
//               N=128, V MN-major, P read from tensor memory);
//   warps 2-17  softmax in two groups of eight warps that take the key tiles in turn
//               (group 0 the even tiles, group 1 the odd ones).  Each group has its own
//               S buffer (128 columns) and P buffer (64 columns of bf16 pairs) in tensor
//               memory, next to the 128-column O accumulator: 512 columns in all.  In a
//               group, two warps share each TMEM lane quarter, 64 key columns each, and
//               exchange their row maxima as fp16 rounded up.
// Because the groups alternate, the exponentials of one tile overlap the loads,
// maximum and handoffs of the next, and the tensor pipe is fed by both.  The online
// softmax keeps one reference maximum per row (lazy rescaling: it moves only when a
// tile's maximum exceeds it by more than 2^8).  The reference is handed from group to
// group through a two-slot ring in shared memory right after each tile's maximum is
// known; each group keeps its own partial row sum relative to the reference it last
// used and rescales it when the reference moves; the group that moves it also
// rescales O in tensor memory, after O += P V of the previous tile has completed.  At
// the end the four partial sums of a row are added, O is read from tensor memory,
// divided by the row sum, gated or RMS-normalised, and stored.
// Query tiles are scheduled longest first (causal), heads of one kv group next to
// each other (K/V reuse in L2).
#include <cuda_fp16.h>
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace hh {

namespace {

constexpr int TD = 128;  // head dim
constexpr int TBM = 128, TBN = 128;
constexpr int kTStage = 32768;  // one 128-key x 128-d tile of K or V
constexpr int kTRing = 4;
constexpr int kTThreads = 576;  // producer, MMA, 16 softmax warps
constexpr float kTLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.0f;

struct TcParams {
  CUtensorMap tm_q, tm_k, tm_v;  // 4-D (d, heads, T, B); box (64, 1, 128, 1)
  const bf16_t *gate;
  bf16_t *o;
  int B, T, n_heads, group, q_heads, kv_heads;
  int use_map;
  int map[kMaxMappedHeads];
  float scale_log2;
  int causal, rms;
  float eps;
  int n_qblocks;
  unsigned *status;
};

struct TcL {
  static constexpr int kQ = TBM * TD * 2;  // Q tile
  static constexpr int kP = 2048;          // final row sums / squares [4][128] fp32
  static constexpr int oQ = 0, oP = kQ, oRing = kQ + kP, oBar = oRing + kTRing * kTStage;
  // full/empty ring barriers, qfull, sfull[2], sfree[2], pfull[2], pvdone[2], mfull[2], fin
  static constexpr int kBars = 2 * kTRing + 12;
  static constexpr int oX = oBar + kBars * 8 + 16;  // row maxima [2 groups][2 warps][128] fp16
  static constexpr int oM = oX + 1024;              // reference maxima ring [2][128] fp32
  static constexpr int kTotal = oM + 1024 + 1024;
  static constexpr uint32_t kTmemCols = 512;
  // O (128 columns), S of group 0 and 1 (128 each), P of group 0 and 1 (64 each, bf16 pairs)
  static constexpr uint32_t kOCol = 0, kSCol = 128, kPCol = 384;
  static_assert(kTotal <= 232448, "shared memory budget");
};

// the two warps of one group and TMEM lane quarter (64 threads) meet and AND their
// predicates, so a wait that gave up in one of them ends both together
__device__ __forceinline__ bool pair_bar_and(int id, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, %2, 64, p;\n"
      " selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id)
      : "memory");
  return r != 0;
}
// the four softmax warps of a TMEM lane quarter (128 threads), for the epilogue
__device__ __forceinline__ void quad_bar(int id) { asm volatile("bar.sync %0, 128;\n" ::"r"(id) : "memory"); }
__device__ __forceinline__ bool quad_bar_and(int id, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, %2, 128, p;\n"
      " selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// Positions of the K and V tiles in the load ring, in the order the MMAs consume them:
// K0, K1, then for each tile j: K(j+2), V(j).  A position p reuses the slot of p - kTRing,
// which is K(j) for K(j+2) and V(j-2) for V(j) (kTRing = 4), so a K tile never waits for
// a V tile to be consumed.  Positions of tiles past the end are skipped by both sides.
__device__ __forceinline__ int pos_k(int j) { return j < 2 ? j : 2 * j - 2; }
__device__ __forceinline__ int pos_v(int j) { return 2 * j + 3; }

__global__ void __launch_bounds__(kTThreads, 1) attn_fwd_tc_kernel(const __grid_constant__ TcParams p) {
  using L = TcL;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(sm + L::oBar);
  uint64_t *empty = full + kTRing;
  uint64_t *qfull = full + 2 * kTRing;
  uint64_t *sfull = qfull + 1;   // [2] S of the group's tile is in tensor memory
  uint64_t *sfree = qfull + 3;   // [2] the group has read its S (8 warps)
  uint64_t *pfull = qfull + 5;   // [2] the group's P is in tensor memory (8 warps)
  uint64_t *pvdone = qfull + 7;  // [2] O += P V of the group's tile completed
  uint64_t *mfull = qfull + 9;   // [2] reference maxima of a tile are in the ring (4 warps)
  uint64_t *fin = qfull + 11;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::oBar + L::kBars * 8);
  const uint32_t sQ = smem_u32(sm + L::oQ), sRing = smem_u32(sm + L::oRing);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per_q = p.n_heads * p.B;
  const int idx = blockIdx.x;
  const int qblk = p.causal ? (p.n_qblocks - 1 - idx / per_q) : idx / per_q;
  const int rem = idx % per_q;
  const int hi = rem % p.n_heads, b = rem / p.n_heads;
  const int qh = p.use_map ? p.map[hi] : hi;
  const int kh = p.use_map ? p.map[hi] : hi / p.group;
  const int m0 = qblk * TBM;
  const int kv_end = p.causal ? min(p.T, m0 + TBM) : p.T;
  const int n_tiles = (kv_end + TBN - 1) / TBN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTRing; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(qfull, 1);
    for (int g = 0; g < 2; ++g) {
      mbar_init(&sfull[g], 1);
      mbar_init(&sfree[g], 8);
      mbar_init(&pfull[g], 8);
      mbar_init(&pvdone[g], 1);
      mbar_init(&mfull[g], 4);
    }
    mbar_init(fin, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 0) {
    // ---------------- TMA producer: K and V tiles in the order the MMAs consume them ----------------
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      mbar_arrive_expect_tx(qfull, L::kQ);
      for (int bx = 0; bx < TD / 64; ++bx) tma_load_4d(sQ + bx * (TBM * 128), &p.tm_q, qfull, bx * 64, qh, m0, b);
      // the load sequence K0, K1, then K(j+2), V(j) for j = 0, 1, ...
      int last_pos[kTRing];  // the last position loaded into each slot, -1 if none
#pragma unroll
      for (int s = 0; s < kTRing; ++s) last_pos[s] = -1;
      for (int step = 0; step < 2 * n_tiles + 2; ++step) {
        int j, pos;
        bool is_v;
        if (step < 2) {
          j = step, pos = step, is_v = false;
        } else {
          j = (step - 2) >> 1;
          is_v = (step & 1) != 0;
          if (!is_v) j += 2;
          pos = is_v ? pos_v(j) : pos_k(j);
        }
        if (j >= n_tiles) continue;
        const int s = pos % kTRing;
        if (pos >= kTRing && !mbar_wait(&empty[s], ((pos / kTRing) - 1) & 1, p.status)) break;
        mbar_arrive_expect_tx(&full[s], kTStage);
        const uint32_t dst = sRing + s * kTStage;
        const CUtensorMap *tm = is_v ? &p.tm_v : &p.tm_k;
        for (int bx = 0; bx < TD / 64; ++bx) tma_load_4d(dst + bx * 16384, tm, &full[s], bx * 64, kh, j * TBN, b);
        last_pos[s] = pos;
      }
      // Every load issued above has landed before the CTA can exit: after a wait that gave up,
      // some may never have been consumed.  On the normal path these phases are complete.
      mbar_wait(qfull, 0, p.status);
#pragma unroll
      for (int s = 0; s < kTRing; ++s)
        if (last_pos[s] >= 0) mbar_wait(&full[s], (last_pos[s] / kTRing) & 1, p.status);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issue: the warp runs the loop, one elected lane issues ----------------
    // Descriptor bases are hoisted; a k step or a ring slot only adds to the 16-byte address field.
    const uint32_t tO = tbase + L::kOCol;
    const uint64_t dQ = tc::desc_kmajor_sw128(sQ);
    const uint64_t dK = tc::desc_kmajor_sw128(sRing);
    const uint64_t dV = tc::desc_mnmajor_sw128(sRing, TBN * 128, 1024);
    constexpr uint32_t idS = tc::idesc_bf16_f32(128, TBN, 0, 0);
    constexpr uint32_t idO = tc::idesc_bf16_f32(128, TD, 0, 1);
    auto wait_all = [&](uint64_t *bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, p.status));
    };
    auto issue_S = [&](int j) -> bool {  // S(j) into the S buffer of group j & 1
      const int pos = pos_k(j), s = pos % kTRing;
      if (!wait_all(&full[s], (pos / kTRing) & 1)) return false;
      tc::fence_after();
      const uint32_t tS = tbase + L::kSCol + (uint32_t)(j & 1) * TBN;
      const uint32_t so = (uint32_t)(s * kTStage) >> 4;
#pragma unroll
      for (int kk = 0; kk < TD / 16; ++kk) {
        const uint32_t o = (uint32_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);  // d0 = 16 kk
        tc::mma_ss_w(tS, dQ + o, dK + so + o, idS, kk ? 1u : 0u);
      }
      tc::commit_w(&empty[s]);
      tc::commit_w(&sfull[j & 1]);
      return true;
    };
    auto issue_PV = [&](int j) -> bool {  // O += P(j) V(j), P from the P buffer of group j & 1
      const int pos = pos_v(j), s = pos % kTRing;
      if (!wait_all(&full[s], (pos / kTRing) & 1)) return false;
      tc::fence_after();
      const uint32_t tP = tbase + L::kPCol + (uint32_t)(j & 1) * (TBN / 2);
      const uint32_t so = (uint32_t)(s * kTStage) >> 4;
#pragma unroll
      for (int kk = 0; kk < TBN / 16; ++kk)
        tc::mma_ts_w(tO, tP + kk * 8, dV + so + (uint32_t)((kk * 16 * 128) >> 4), idO, (j | kk) ? 1u : 0u);
      tc::commit_w(&empty[s]);
      tc::commit_w(&pvdone[j & 1]);
      return true;
    };
    bool ok = wait_all(qfull, 0);
    tc::fence_after();
    if (ok) ok = issue_S(0);
    if (ok && n_tiles > 1) ok = issue_S(1);
    for (int j = 0; j < n_tiles && ok; ++j) {
      if (j + 2 < n_tiles) {  // S(j+2) reuses the S buffer of tile j once its group has read it
        if (!wait_all(&sfree[j & 1], (j >> 1) & 1)) break;
        tc::fence_after();
        if (!issue_S(j + 2)) break;
      }
      if (!wait_all(&pfull[j & 1], (j >> 1) & 1)) break;
      tc::fence_after();
      if (!issue_PV(j)) break;
    }
    // every MMA issued above must be complete before the CTA releases tensor memory
    tc::commit_w(fin);
    mbar_wait(fin, 0, p.status);
    __syncwarp();
  } else {
    // ---------------- softmax (two groups, tiles in turn) / correction / epilogue ----------------
    const int sw = warp - 2;            // 0..15
    const int q4 = warp & 3;            // TMEM lane quarter this warp may access
    const int grp = sw >> 3;            // 0: even key tiles, 1: odd key tiles
    const int part = (sw >> 2) & 1;     // which 64 keys of the tile (and 64 columns of O)
    const int k4 = grp * 2 + part;      // 0..3: this warp's quarter of O in the epilogue
    const int row = q4 * 32 + lane;
    const int row_g = m0 + row;
    const uint32_t tl = tbase + ((uint32_t)(q4 * 32) << 16);
    const uint32_t tS = tl + L::kSCol + (uint32_t)grp * TBN + part * 64;
    const uint32_t tP = tl + L::kPCol + (uint32_t)grp * (TBN / 2) + part * 32;
    const uint32_t tOr = tl + L::kOCol + part * 64;  // the 64 O columns this warp rescales
    __half *xmx = reinterpret_cast<__half *>(sm + L::oX);  // [2][2][128]
    float *mref = reinterpret_cast<float *>(sm + L::oM);   // [2][128]
    const int pbar = 1 + grp * 4 + q4;                     // named barriers 1..8
    const float cs = p.scale_log2;
    float m_use = -INFINITY;  // the reference maximum this group's l_run is relative to
    float l_run = 0.f;
    bool ok = true, okw = true;
    for (int j = grp; j < n_tiles; j += 2) {
      const int u = j >> 1;  // use count of this group's S and P buffers
      const bool w1 = mbar_wait(&sfull[grp], u & 1, p.status);
      tc::fence_after();
      const int key0 = j * TBN + part * 64;
      const bool edge = (key0 + 64 > p.T) || (p.causal && key0 + 63 > row_g);
      // pass 1: the row maximum over this warp's 64 keys
      float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t r[32];
        tc::ld32(tS + h * 32, r);
        tc::wait_ld();
        tc::regfence(r);
        if (edge) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int key = key0 + h * 32 + i;
            if (key >= p.T || (p.causal && key > row_g)) r[i] = __float_as_uint(-INFINITY);
          }
        }
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          a0 = fmaxf(a0, __uint_as_float(r[i]));
          a1 = fmaxf(a1, __uint_as_float(r[i + 1]));
          a2 = fmaxf(a2, __uint_as_float(r[i + 2]));
          a3 = fmaxf(a3, __uint_as_float(r[i + 3]));
        }
      }
      xmx[(grp * 2 + part) * 128 + row] = __float2half_ru(fmaxf(fmaxf(a0, a1), fmaxf(a2, a3)));
      if (!pair_bar_and(pbar, w1 && okw)) {
        ok = false;
        break;
      }
      const float mx = fmaxf(__half2float(xmx[(grp * 2) * 128 + row]), __half2float(xmx[(grp * 2 + 1) * 128 + row])) * cs;
      // the reference maximum: the previous tile's (from the other group) or, if this tile's
      // maximum exceeds it by more than 2^8, this tile's
      bool wm = true;
      float m_prev = -INFINITY;
      if (j > 0) {
        wm = mbar_wait(&mfull[(j - 1) & 1], ((j - 1) >> 1) & 1, p.status);
        m_prev = mref[((j - 1) & 1) * 128 + row];
      }
      float m_ref = m_prev;
      bool resc = false;
      if (j == 0) {
        m_ref = mx;
      } else if (mx > m_prev + kRescaleLog2) {
        m_ref = mx;
        resc = true;
      }
      if (part == 0) {
        mref[(j & 1) * 128 + row] = m_ref;
        __syncwarp();
        if (lane == 0) mbar_arrive(&mfull[j & 1]);
      }
      if (m_ref != m_use) {
        l_run = m_use == -INFINITY ? 0.f : l_run * ex2_approx(m_use - m_ref);
        m_use = m_ref;
      }
      const float nb = m_ref == -INFINITY ? 0.f : -m_ref;
      // this group's P buffer is free once O += P V of tile j - 2 has completed
      bool wp = true;
      if (j >= 2) {
        wp = mbar_wait(&pvdone[grp], (u - 1) & 1, p.status);
        tc::fence_after();
      }
      // pass 2: exponentials, row sums, P as bf16 pairs into tensor memory
      float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t r[32];
        tc::ld32(tS + h * 32, r);
        tc::wait_ld();
        tc::regfence(r);
        if (h == 1) {  // the group's S is read: S(j + 2) may overwrite it
          tc::fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sfree[grp]);
        }
        if (edge) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int key = key0 + h * 32 + i;
            if (key >= p.T || (p.causal && key > row_g)) r[i] = __float_as_uint(-INFINITY);
          }
        }
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float e0 = ex2_approx(fmaf(__uint_as_float(r[i]), cs, nb));
          const float e1 = ex2_approx(fmaf(__uint_as_float(r[i + 1]), cs, nb));
          const float e2 = ex2_approx(fmaf(__uint_as_float(r[i + 2]), cs, nb));
          const float e3 = ex2_approx(fmaf(__uint_as_float(r[i + 3]), cs, nb));
          s0 += e0;
          s1 += e1;
          s2 += e2;
          s3 += e3;
          pk[i / 2] = pack_bf16(e0, e1);
          pk[i / 2 + 1] = pack_bf16(e2, e3);
        }
        tc::st16u(tP + h * 16, pk);
      }
      l_run += (s0 + s1) + (s2 + s3);
      tc::wait_st();
      tc::fence_before();
      // O is rescaled by the group that moved the reference, after O += P V of tile j - 1
      bool wo = true;
      if (__any_sync(0xffffffffu, resc)) {
        wo = mbar_wait(&pvdone[(j - 1) & 1], ((j - 1) >> 1) & 1, p.status);
        tc::fence_after();
        const float alpha = resc ? ex2_approx(m_prev - m_ref) : 1.f;
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          uint32_t ov[32];
          tc::ld32(tOr + c * 32, ov);
          tc::wait_ld();
          tc::regfence(ov);
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
          tc::st32u(tOr + c * 32, ov);
        }
        tc::wait_st();
        tc::fence_before();
      }
      okw = wm && wp && wo;
      if (lane == 0) mbar_arrive(&pfull[grp]);
    }
    // epilogue: every partial row sum relative to the last tile's reference, summed over
    // the four warps of the lane quarter (both groups, both halves of the keys)
    float *xsum = reinterpret_cast<float *>(sm + L::oP);  // [4][128]
    const int qbar = 9 + q4;                              // named barriers 9..12
    const uint32_t tO = tl + L::kOCol + k4 * 32;
    // the four warps of a lane quarter belong to both groups, and a pair that gave up a wait
    // left its loop early: every warp reaches this barrier, and all four go on only if none failed
    bool we = false;
    if (ok && n_tiles > 0) {
      const int jl = n_tiles - 1;
      we = mbar_wait(&mfull[jl & 1], (jl >> 1) & 1, p.status);
      const float m_fin = mref[(jl & 1) * 128 + row];
      if (m_fin != m_use) l_run = m_use == -INFINITY ? 0.f : l_run * ex2_approx(m_use - m_fin);
      we = mbar_wait(&pvdone[jl & 1], (jl >> 1) & 1, p.status) && we;  // the last MMA, so all of them
      tc::fence_after();
      xsum[k4 * 128 + row] = l_run;
    }
    ok = quad_bar_and(qbar, ok && we && okw);
    if (ok) {
      const float l_tot = (xsum[row] + xsum[128 + row]) + (xsum[256 + row] + xsum[384 + row]);
      const float inv_l = l_tot > 0.f ? 1.f / l_tot : 0.f;
      const bool valid = row_g < p.T;
      const size_t obase = (((size_t)b * p.T + (valid ? row_g : 0)) * p.q_heads + qh) * TD + k4 * 32;
      const bf16_t *gp = p.gate ? p.gate + obase : nullptr;
      uint32_t ov[32];
      tc::ld32(tO, ov);
      tc::wait_ld();
      tc::regfence(ov);
      float v[32];
#pragma unroll
      for (int i = 0; i < 32; i += 8) {
        uint4 gg = make_uint4(0, 0, 0, 0);
        if (gp && valid) gg = *reinterpret_cast<const uint4 *>(gp + i);
        const uint32_t gw[4] = {gg.x, gg.y, gg.z, gg.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float x = __uint_as_float(ov[i + e]) * inv_l;
          if (gp) x *= 1.f / (1.f + expf(-((e & 1) ? bf16_hi(gw[e >> 1]) : bf16_lo(gw[e >> 1]))));
          v[i + e] = x;
        }
      }
      if (p.rms) {
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) ss += v[i] * v[i];
        quad_bar(qbar);  // all four have read the row sums before the slots are reused
        xsum[k4 * 128 + row] = ss;
        quad_bar(qbar);
        ss = (xsum[row] + xsum[128 + row]) + (xsum[256 + row] + xsum[384 + row]);
        const float rs = rsqrtf(ss / (float)TD + p.eps);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= rs;
      }
      if (valid) {
#pragma unroll
        for (int i = 0; i < 32; i += 8)
          *reinterpret_cast<uint4 *>(p.o + obase + i) = make_uint4(pack_bf16(v[i], v[i + 1]), pack_bf16(v[i + 2], v[i + 3]),
                                                                   pack_bf16(v[i + 4], v[i + 5]), pack_bf16(v[i + 6], v[i + 7]));
      }
    }
  }
  tc::fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after();
    tc::tmem_dealloc(tbase, L::kTmemCols);
  }
}

cudaError_t launch_tc(const TcParams &p, cudaStream_t s) {
  auto kern = attn_fwd_tc_kernel;
  const int smem = TcL::kTotal;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const long long grid = (long long)p.n_qblocks * p.n_heads * p.B;
  kern<<<(unsigned)grid, kTThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd_tc(const AttnFwdArgs &a, cudaStream_t s) {
  if (a.B == 0 || a.T == 0 || a.n_heads == 0) return cudaSuccess;
  if (a.d != TD) {
    set_error("gqa_attn_fwd: the single-CTA kernel is built for head dim 128");
    return cudaErrorInvalidValue;
  }
  TcParams p;
  memset(&p, 0, sizeof(p));
  const uint32_t box[4] = {64, 1, 128, 1};
  const uint64_t dq[4] = {(uint64_t)a.d, (uint64_t)a.q_heads, (uint64_t)a.T, (uint64_t)a.B};
  const uint64_t sq[3] = {(uint64_t)a.d * 2, (uint64_t)a.q_heads * a.d * 2, (uint64_t)a.T * a.q_heads * a.d * 2};
  const uint64_t dk[4] = {(uint64_t)a.d, (uint64_t)a.kv_heads, (uint64_t)a.T, (uint64_t)a.B};
  const uint64_t sk[3] = {(uint64_t)a.d * 2, (uint64_t)a.kv_heads * a.d * 2, (uint64_t)a.T * a.kv_heads * a.d * 2};
  if (encode_tmap(&p.tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.q, dq, sq, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
      encode_tmap(&p.tm_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.k, dk, sk, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
      encode_tmap(&p.tm_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.v, dk, sk, box, CU_TENSOR_MAP_SWIZZLE_128B)) {
    set_error("gqa_attn_fwd: cuTensorMapEncodeTiled failed");
    return cudaErrorInvalidValue;
  }
  p.gate = a.gate;
  p.o = a.o;
  p.B = a.B;
  p.T = a.T;
  p.n_heads = a.n_heads;
  p.group = a.group;
  p.q_heads = a.q_heads;
  p.kv_heads = a.kv_heads;
  p.use_map = a.use_map;
  memcpy(p.map, a.map, sizeof(p.map));
  p.scale_log2 = a.scale * kTLog2e;
  p.causal = a.causal;
  p.rms = a.rms;
  p.eps = a.eps;
  p.n_qblocks = (a.T + TBM - 1) / TBM;
  p.status = device_status_ptr();
  return launch_tc(p, s);
}

}  // namespace hh
