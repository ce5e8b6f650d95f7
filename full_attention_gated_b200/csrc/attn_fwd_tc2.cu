// attn_fwd_tc2.cu -- causal grouped-query softmax attention (prefill) on CTA
// pairs: one tcgen05 MMA with M = 256 spans the tensor cores of two SMs.
//
// Same computation as attn_fwd_tc.cu (online softmax flash attention with the
// optional sigmoid gate or the per-head RMS fusion; 24 query heads over 4 KV
// heads at d = 256 in the hybrid stack's attention layers, "The Hybrid
// Attention in Qwen3.8-27B", "Grouped-query attention multiplies on top of
// that"; d = 128 for the FA heads of the HydraHead layer).
//
// A cluster of two CTAs owns 256 query rows of one head; CTA r holds rows
// 128 r .. 128 r + 127 in its own shared memory (Q) and tensor memory (S, P, O).
//   S = Q K^T : M = 256 (128 rows per CTA), N = 128 keys; each CTA holds 64 of
//               the 128 keys of a K tile (the B operand is split along N);
//   O += P V  : M = 256, N = d; each CTA holds d/2 columns of the V tile.
// So each CTA streams only half of every K/V tile, and the 4 x 32 KiB ring of a
// CTA holds two whole KV tiles in flight.  Roles per CTA: warp 0 issues the TMA
// loads (both CTAs' loads complete on the leader CTA's barriers), warp 1 owns
// tensor memory and, in the leader CTA only, runs the MMA loop as a whole warp
// with one elected lane issuing, so the descriptors stay warp-uniform
// (completions are multicast to both CTAs); warps 2-17 run the softmax of the
// CTA's 128 rows, four warps per TMEM lane quarter (a quarter of the key columns
// each), and one warp of each four reports to the leader's barriers.  P goes to
// tensor memory as bf16 pairs and is the A operand of O += P V, so the P tile
// costs no shared-memory bandwidth (stores or MMA operand reads).
#include <cuda_fp16.h>
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace hh {

namespace {

constexpr int PBM = 128;  // rows per CTA (256 per pair)
constexpr int PBN = 128;  // keys per KV tile
constexpr int kPStage = 32768;
constexpr int kPRing = 4;
constexpr int kPThreads2 = 576;  // producer, MMA, 16 softmax warps
constexpr float kPLog2e = 1.4426950408889634f;
constexpr float kPRescale = 8.0f;

struct PairParams {
  CUtensorMap tm_q, tm_k, tm_v;  // 4-D (d, heads, T, B); boxes (64,1,128,1), (64,1,64,1), (64,1,128,1)
  const bf16_t *gate;
  bf16_t *o;
  int B, T, n_heads, group, q_heads, kv_heads;
  int use_map;
  int map[kMaxMappedHeads];
  float scale_log2;
  int causal, rms;
  float eps;
  int n_qblocks;  // 256-row blocks
  unsigned *status;
};

template <int D>
struct PairL {
  static constexpr int kQ = PBM * D * 2;          // this CTA's Q rows
  static constexpr int kP = 2048;                 // final row sums [4][128] fp32 (P itself is in TMEM)
  static constexpr int kKB = (PBN / 2) * D * 2;   // this CTA's half of a K tile (64 keys)
  static constexpr int kVB = PBN * (D / 2) * 2;   // this CTA's half of a V tile (d/2 columns)
  static constexpr int oQ = 0, oP = kQ, oRing = kQ + kP, oBar = oRing + kPRing * kPStage;
  static constexpr int kBars = 2 * kPRing + 6;
  static constexpr int oX = oBar + kBars * 8 + 16;  // row-maximum exchange [4][128] fp16
  static constexpr int kTotal = oX + 1024 + 1024;
  static constexpr uint32_t kTmemCols = 512;
  // O (d columns), S (128 columns), P as bf16 pairs (64 columns): the A operand of O += P V
  static constexpr uint32_t kOCol = 0, kSCol = D, kPCol = D + PBN;
  static_assert(kKB <= kPStage && kVB <= kPStage, "stage size");
  static_assert(kTotal <= 232448, "shared memory budget");
};

// the four softmax warps of a TMEM lane quarter (128 threads)
__device__ __forceinline__ void quad_bar(int id) { asm volatile("bar.sync %0, 128;\n" ::"r"(id) : "memory"); }
// ... meeting and ANDing their predicates, so a wait that gave up in one warp ends all four together
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
__device__ __forceinline__ float ex2a(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// bounded wait with cluster-scope acquire (arrivals may come from the peer CTA)
__device__ __forceinline__ bool wait_cl(uint64_t *bar, uint32_t parity, unsigned *status) {
  const uint32_t a = smem_u32(bar);
  if (tc2::try_wait_cluster(a, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    if (tc2::try_wait_cluster(a, parity)) return true;
    if ((i & 255u) == 0) {
      const uint64_t dt = global_ns() - t0;
      if (dt > HH_WAIT_PEER_NS && status && (*reinterpret_cast<volatile unsigned *>(status) & kStatusTimeout))
        return false;
      if (dt > HH_WAIT_NS) {
        if (status) atomicOr(status, kStatusTimeout);
        return false;
      }
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kPThreads2, 1) attn_fwd_pair_kernel(const __grid_constant__ PairParams p) {
  using L = PairL<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(sm + L::oBar);
  uint64_t *empty = full + kPRing;
  uint64_t *qfull = full + 2 * kPRing;
  uint64_t *sfull = qfull + 1, *sfree = qfull + 2, *pfull = qfull + 3, *odone = qfull + 4, *fin = qfull + 5;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::oBar + L::kBars * 8);
  const uint32_t sQ = smem_u32(sm + L::oQ), sRing = smem_u32(sm + L::oRing);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = tc2::cluster_rank();
  const bool leader = rank == 0;
  const int per_q = p.n_heads * p.B;
  const int cid = blockIdx.x >> 1;  // cluster index
  const int qblk = p.causal ? (p.n_qblocks - 1 - cid / per_q) : cid / per_q;
  const int rem = cid % per_q;
  const int hi = rem % p.n_heads, b = rem / p.n_heads;
  const int qh = p.use_map ? p.map[hi] : hi;
  const int kh = p.use_map ? p.map[hi] : hi / p.group;
  const int m0 = qblk * 2 * PBM;          // first row of the pair
  const int r0 = m0 + (int)rank * PBM;    // first row of this CTA
  const int kv_end = p.causal ? min(p.T, m0 + 2 * PBM) : p.T;
  const int n_tiles = (kv_end + PBN - 1) / PBN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPRing; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(qfull, 1);
    mbar_init(sfull, 1);
    mbar_init(sfree, 8);  // one arrival per TMEM lane quarter (four warps) x 2 CTAs
    mbar_init(pfull, 8);
    mbar_init(odone, 1);
    mbar_init(fin, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tc2::tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tc2::tmem_relinquish();
  }
  tc::fence_before();
  tc2::cluster_sync();  // barriers of both CTAs initialised, tensor memory allocated
  tc::fence_after();
  const uint32_t tbase = *tmem_slot;
  // leader's barriers as seen from this CTA
  const uint32_t full_l = tc2::map_rank(smem_u32(full), 0);
  const uint32_t qfull_l = tc2::map_rank(smem_u32(qfull), 0);
  const uint32_t sfree_l = tc2::map_rank(smem_u32(sfree), 0);
  const uint32_t pfull_l = tc2::map_rank(smem_u32(pfull), 0);

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs) ----------------
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      if (leader) mbar_arrive_expect_tx(qfull, 2 * L::kQ);
      for (int bx = 0; bx < D / 64; ++bx)
        tc2::tma_load_4d_pair(sQ + bx * (PBM * 128), &p.tm_q, qfull_l, bx * 64, qh, r0, b);
      bool ok = true;
      int last_item = -1;
      for (int item = 0; item < 2 * n_tiles && ok; ++item) {
        const int s = item % kPRing, j = item >> 1;
        if (item >= kPRing && !mbar_wait(&empty[s], ((item / kPRing) - 1) & 1, p.status)) {
          ok = false;
          break;
        }
        const uint32_t dst = sRing + s * kPStage;
        const uint32_t bar = full_l + s * 8;
        if ((item & 1) == 0) {  // K: this CTA's 64 keys of tile j, all d
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * L::kKB);
          for (int bx = 0; bx < D / 64; ++bx)
            tc2::tma_load_4d_pair(dst + bx * 8192, &p.tm_k, bar, bx * 64, kh, j * PBN + (int)rank * (PBN / 2), b);
        } else {  // V: all 128 keys of tile j, this CTA's d/2 columns
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * L::kVB);
          for (int bx = 0; bx < D / 128; ++bx)
            tc2::tma_load_4d_pair(dst + bx * 16384, &p.tm_v, bar, (int)rank * (D / 2) + bx * 64, kh, j * PBN, b);
        }
        last_item = item;
      }
      // The loads of both CTAs complete on the leader's barriers, so the leader waits (bounded)
      // for the last phase of each stage before the final cluster barrier, which the peer
      // cannot pass earlier: no load issued above is still landing when either CTA exits.  On
      // the normal path these phases are complete.
      if (leader) {
        wait_cl(qfull, 0, p.status);
        for (int item = max(last_item - kPRing + 1, 0); item <= last_item; ++item)
          wait_cl(&full[item % kPRing], (item / kPRing) & 1, p.status);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issue (leader CTA): the warp runs the loop, one elected lane issues ----
    // Descriptor bases are hoisted; a k step or a ring slot only adds to the 16-byte address field.
    if (leader) {
      const uint32_t tS = tbase + L::kSCol, tO = tbase + L::kOCol;
      const uint64_t dQ = tc::desc_kmajor_sw128(sQ);
      const uint64_t dK = tc::desc_kmajor_sw128(sRing);
      const uint64_t dV = tc::desc_mnmajor_sw128(sRing, PBN * 128, 1024);
      constexpr uint32_t idS = tc::idesc_bf16_f32(256, PBN, 0, 0);
      constexpr uint32_t idO = tc::idesc_bf16_f32(256, D, 0, 1);
      constexpr uint16_t both = 0x3;
      auto wait_all = [&](uint64_t *bar, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, wait_cl(bar, parity, p.status));
      };
      bool ok = wait_all(qfull, 0);
      tc::fence_after();
      auto issue_S = [&](int j) -> bool {
        const int item = 2 * j, s = item % kPRing;
        if (!wait_all(&full[s], (item / kPRing) & 1)) return false;
        tc::fence_after();
        const uint32_t so = (uint32_t)(s * kPStage) >> 4;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t oa = (uint32_t)(((ks >> 2) * (PBM * 128) + (ks & 3) * 32) >> 4);  // d0 = 16 ks
          const uint32_t ob = (uint32_t)(((ks >> 2) * 8192 + (ks & 3) * 32) >> 4);
          tc2::mma_ss_w(tS, dQ + oa, dK + so + ob, idS, ks ? 1u : 0u);
        }
        tc2::commit_mc_w(&empty[s], both);
        tc2::commit_mc_w(sfull, both);
        return true;
      };
      auto issue_PV = [&](int j) -> bool {
        const int item = 2 * j + 1, s = item % kPRing;
        if (!wait_all(&full[s], (item / kPRing) & 1)) return false;
        tc::fence_after();
        const uint32_t so = (uint32_t)(s * kPStage) >> 4;
#pragma unroll
        for (int kk = 0; kk < PBN / 16; ++kk)
          tc2::mma_ts_w(tO, tbase + L::kPCol + kk * 8, dV + so + (uint32_t)((kk * 16 * 128) >> 4), idO,
                        (j | kk) ? 1u : 0u);
        tc2::commit_mc_w(&empty[s], both);
        tc2::commit_mc_w(odone, both);
        return true;
      };
      if (ok) ok = issue_S(0);
      for (int j = 0; j < n_tiles && ok; ++j) {
        if (j + 1 < n_tiles) {
          if (!wait_all(sfree, j & 1)) break;
          tc::fence_after();
          if (!issue_S(j + 1)) break;
        }
        if (!wait_all(pfull, j & 1)) break;
        tc::fence_after();
        if (!issue_PV(j)) break;
      }
      tc2::commit_mc_w(fin, 0x1);  // this CTA only; same cta_group as the MMAs it tracks
      mbar_wait(fin, 0, p.status);
    }
    __syncwarp();
  } else {
    // ---------------- softmax / correction / epilogue: this CTA's 128 rows ----------------
    // four warps per TMEM lane quarter, each owning 32 of the 128 key columns (and d/4 of O);
    // row maxima are exchanged as fp16 rounded up (every warp of the row reads the same four
    // values, so all agree on the maximum), the final row sums in fp32 through the P tile
    const int sw = warp - 2;
    const int q4 = warp & 3;
    const int part = sw >> 2;  // 0..3
    const int row = q4 * 32 + lane;
    const int row_g = r0 + row;
    const uint32_t tl = tbase + ((uint32_t)(q4 * 32) << 16);
    const uint32_t tS = tl + L::kSCol + part * 32, tO = tl + L::kOCol + part * (D / 4);
    __half *xmx = reinterpret_cast<__half *>(sm + L::oX);  // [4][128]
    const float cs = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const bool w1 = wait_cl(sfull, j & 1, p.status);
      tc::fence_after();
      uint32_t r[32];
      tc::ld32(tS, r);
      tc::wait_ld();
      tc::regfence(r);
      const int key0 = j * PBN + part * 32;
      if ((key0 + 32 > p.T) || (p.causal && key0 + 31 > row_g)) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int key = key0 + i;
          if (key >= p.T || (p.causal && key > row_g)) r[i] = __float_as_uint(-INFINITY);
        }
      }
      float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        a0 = fmaxf(a0, __uint_as_float(r[i]));
        a1 = fmaxf(a1, __uint_as_float(r[i + 1]));
        a2 = fmaxf(a2, __uint_as_float(r[i + 2]));
        a3 = fmaxf(a3, __uint_as_float(r[i + 3]));
      }
      xmx[part * 128 + row] = __float2half_ru(fmaxf(fmaxf(a0, a1), fmaxf(a2, a3)));
      tc::fence_before();  // the four warps' S loads completed before the quad barrier
      if (!quad_bar_and(1 + q4, w1)) {
        ok = false;
        break;
      }
      const float mx = fmaxf(fmaxf(__half2float(xmx[row]), __half2float(xmx[128 + row])),
                             fmaxf(__half2float(xmx[256 + row]), __half2float(xmx[384 + row]))) * cs;
      if (part == 0 && lane == 0) {
        if (leader) mbar_arrive(sfree);
        else tc2::remote_arrive(sfree_l);
      }

      float alpha = 1.f;
      bool resc = false;
      if (j == 0) {
        m_run = mx;
      } else if (mx > m_run + kPRescale) {
        alpha = ex2a(m_run - mx);
        m_run = mx;
        resc = true;
      }
      const float nb = m_run == -INFINITY ? 0.f : -m_run;
      float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        const float e0 = ex2a(fmaf(__uint_as_float(r[i]), cs, nb));
        const float e1 = ex2a(fmaf(__uint_as_float(r[i + 1]), cs, nb));
        const float e2 = ex2a(fmaf(__uint_as_float(r[i + 2]), cs, nb));
        const float e3 = ex2a(fmaf(__uint_as_float(r[i + 3]), cs, nb));
        s0 += e0;
        s1 += e1;
        s2 += e2;
        s3 += e3;
        pk[i / 2] = pack_bf16(e0, e1);
        pk[i / 2 + 1] = pack_bf16(e2, e3);
      }
      l_run = l_run * alpha + ((s0 + s1) + (s2 + s3));
      bool w2 = true;
      if (j > 0) {
        w2 = wait_cl(odone, (j - 1) & 1, p.status);
        tc::fence_after();
      }
      if (__any_sync(0xffffffffu, resc)) {
#pragma unroll 1
        for (int c = 0; c < D / 128; ++c) {
          uint32_t ov[32];
          tc::ld32(tO + c * 32, ov);
          tc::wait_ld();
          tc::regfence(ov);
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
          tc::st32u(tO + c * 32, ov);
        }
        tc::wait_st();
      }
      // this warp's 32 keys of the P row -> 16 columns of P in tensor memory (bf16 pairs)
      tc::st16u(tl + L::kPCol + part * 16, pk);
      tc::wait_st();
      tc::fence_before();
      if (!quad_bar_and(5 + q4, w2)) {
        ok = false;
        break;
      }
      if (part == 0 && lane == 0) {
        if (leader) mbar_arrive(pfull);
        else tc2::remote_arrive(pfull_l);
      }
    }
    float *xsum = reinterpret_cast<float *>(sm + L::oP);  // [4][128] fp32 final row sums
    if (ok && n_tiles > 0) {
      const bool w3 = wait_cl(odone, (n_tiles - 1) & 1, p.status);
      tc::fence_after();
      xsum[part * 128 + row] = l_run;
      ok = quad_bar_and(1 + q4, w3);
    }
    if (ok && n_tiles > 0) {
      const float l_tot = (xsum[row] + xsum[128 + row]) + (xsum[256 + row] + xsum[384 + row]);
      const float inv_l = l_tot > 0.f ? 1.f / l_tot : 0.f;
      const bool valid = row_g < p.T;
      const size_t obase = (((size_t)b * p.T + (valid ? row_g : 0)) * p.q_heads + qh) * D + part * (D / 4);
      const bf16_t *gp = p.gate ? p.gate + obase : nullptr;
      float rs = 1.f;
      if (p.rms) {
        float ss = 0.f;
#pragma unroll 1
        for (int c = 0; c < D / 128; ++c) {
          uint32_t ov[32];
          tc::ld32(tO + c * 32, ov);
          tc::wait_ld();
          tc::regfence(ov);
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint4 gg = make_uint4(0, 0, 0, 0);
            if (gp && valid) gg = *reinterpret_cast<const uint4 *>(gp + c * 32 + i);
            const uint32_t gw[4] = {gg.x, gg.y, gg.z, gg.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              float v = __uint_as_float(ov[i + e]) * inv_l;
              if (gp) v *= 1.f / (1.f + expf(-((e & 1) ? bf16_hi(gw[e >> 1]) : bf16_lo(gw[e >> 1]))));
              ss += v * v;
            }
          }
        }
        quad_bar(1 + q4);  // all four have read the row sums before the slots are reused
        xsum[part * 128 + row] = ss;
        quad_bar(1 + q4);
        ss = (xsum[row] + xsum[128 + row]) + (xsum[256 + row] + xsum[384 + row]);
        rs = rsqrtf(ss / (float)D + p.eps);
      }
#pragma unroll 1
      for (int c = 0; c < D / 128; ++c) {
        uint32_t ov[32];
        tc::ld32(tO + c * 32, ov);
        tc::wait_ld();
        tc::regfence(ov);
#pragma unroll
        for (int i = 0; i < 32; i += 8) {
          uint4 gg = make_uint4(0, 0, 0, 0);
          if (gp && valid) gg = *reinterpret_cast<const uint4 *>(gp + c * 32 + i);
          const uint32_t gw[4] = {gg.x, gg.y, gg.z, gg.w};
          float v[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            v[e] = __uint_as_float(ov[i + e]) * inv_l;
            if (gp) v[e] *= 1.f / (1.f + expf(-((e & 1) ? bf16_hi(gw[e >> 1]) : bf16_lo(gw[e >> 1]))));
            v[e] *= rs;
          }
          if (valid)
            *reinterpret_cast<uint4 *>(p.o + obase + c * 32 + i) =
                make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7]));
        }
      }
    }
  }
  tc::fence_before();
  tc2::cluster_sync();  // every MMA done (leader waited on `fin`), every TMEM read done in both CTAs
  if (warp == 1) {
    tc::fence_after();
    tc2::tmem_dealloc(tbase, L::kTmemCols);
  }
}

template <int D>
cudaError_t launch_pair(const PairParams &p, cudaStream_t s) {
  auto kern = attn_fwd_pair_kernel<D>;
  const int smem = PairL<D>::kTotal;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const long long clusters = (long long)p.n_qblocks * p.n_heads * p.B;
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3((unsigned)(2 * clusters), 1, 1);
  cfg.blockDim = dim3(kPThreads2, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd_pair(const AttnFwdArgs &a, cudaStream_t s) {
  if (a.B == 0 || a.T == 0 || a.n_heads == 0) return cudaSuccess;
  PairParams p;
  memset(&p, 0, sizeof(p));
  const uint32_t box_q[4] = {64, 1, (uint32_t)PBM, 1};
  const uint32_t box_k[4] = {64, 1, (uint32_t)(PBN / 2), 1};
  const uint32_t box_v[4] = {64, 1, (uint32_t)PBN, 1};
  const uint64_t dq[4] = {(uint64_t)a.d, (uint64_t)a.q_heads, (uint64_t)a.T, (uint64_t)a.B};
  const uint64_t sq[3] = {(uint64_t)a.d * 2, (uint64_t)a.q_heads * a.d * 2, (uint64_t)a.T * a.q_heads * a.d * 2};
  const uint64_t dk[4] = {(uint64_t)a.d, (uint64_t)a.kv_heads, (uint64_t)a.T, (uint64_t)a.B};
  const uint64_t sk[3] = {(uint64_t)a.d * 2, (uint64_t)a.kv_heads * a.d * 2, (uint64_t)a.T * a.kv_heads * a.d * 2};
  if (encode_tmap(&p.tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.q, dq, sq, box_q, CU_TENSOR_MAP_SWIZZLE_128B) ||
      encode_tmap(&p.tm_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.k, dk, sk, box_k, CU_TENSOR_MAP_SWIZZLE_128B) ||
      encode_tmap(&p.tm_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.v, dk, sk, box_v, CU_TENSOR_MAP_SWIZZLE_128B)) {
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
  p.scale_log2 = a.scale * kPLog2e;
  p.causal = a.causal;
  p.rms = a.rms;
  p.eps = a.eps;
  p.n_qblocks = (a.T + 2 * PBM - 1) / (2 * PBM);
  p.status = device_status_ptr();
  return a.d == 256 ? launch_pair<256>(p, s) : launch_pair<128>(p, s);
}

}  // namespace hh
