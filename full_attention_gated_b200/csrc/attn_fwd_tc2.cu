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
// 128 r .. 128 r + 127 in its own shared memory (Q, P) and tensor memory (S, O).
//   S = Q K^T : M = 256 (128 rows per CTA), N = 128 keys; each CTA holds 64 of
//               the 128 keys of a K tile (the B operand is split along N);
//   O += P V  : M = 256, N = d; each CTA holds d/2 columns of the V tile.
// So each CTA streams only half of every K/V tile, and the 4 x 32 KiB ring of a
// CTA holds two whole KV tiles in flight.  Roles per CTA: warp 0 issues the TMA
// loads (both CTAs' loads complete on the leader CTA's barriers), warp 1 owns
// tensor memory and, in the leader CTA only, issues the MMAs from one thread
// (completions are multicast to both CTAs); warps 2-9 run the softmax of the
// CTA's 128 rows, two warps per TMEM lane quarter (half of the key columns each),
// and one warp of each pair reports to the leader's barriers.
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
constexpr int kPThreads2 = 320;  // producer, MMA, 8 softmax warps
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
  static constexpr int kP = PBM * PBN * 2;        // this CTA's P rows
  static constexpr int kKB = (PBN / 2) * D * 2;   // this CTA's half of a K tile (64 keys)
  static constexpr int kVB = PBN * (D / 2) * 2;   // this CTA's half of a V tile (d/2 columns)
  static constexpr int oQ = 0, oP = kQ, oRing = kQ + kP, oBar = oRing + kPRing * kPStage;
  static constexpr int kBars = 2 * kPRing + 6;
  static constexpr int oX = oBar + kBars * 8 + 16;  // row-statistics exchange [2][128] fp32
  static constexpr int kTotal = oX + 1024 + 1024;
  static constexpr uint32_t kTmemCols = D == 256 ? 512u : 256u;
  static constexpr uint32_t kOCol = 0, kSCol = D;
  static_assert(kKB <= kPStage && kVB <= kPStage, "stage size");
  static_assert(kTotal <= 232448, "shared memory budget");
};

__device__ __forceinline__ void pair_bar2(int id) { asm volatile("bar.sync %0, 64;\n" ::"r"(id) : "memory"); }
// the two warps of a TMEM lane quarter meet and AND their predicates, so a wait that gave up in
// either warp ends both together (neither is left waiting at a later pair barrier)
__device__ __forceinline__ bool pair_bar2_and(int id, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, %2, 64, p;\n"
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
__device__ __forceinline__ void st_shared_v4p(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
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
  const uint32_t sQ = smem_u32(sm + L::oQ), sP = smem_u32(sm + L::oP), sRing = smem_u32(sm + L::oRing);

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
    mbar_init(sfree, 8);  // one arrival per TMEM lane quarter (warp pair) x 2 CTAs
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
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer (leader CTA, one thread) ----------------
    if (leader && lane == 0) {
      const uint32_t tS = tbase + L::kSCol, tO = tbase + L::kOCol;
      constexpr uint32_t idS = tc::idesc_bf16_f32(256, PBN, 0, 0);
      constexpr uint32_t idO = tc::idesc_bf16_f32(256, D, 0, 1);
      constexpr uint16_t both = 0x3;
      bool ok = wait_cl(qfull, 0, p.status);
      tc::fence_after();
      auto issue_S = [&](int j) -> bool {
        const int item = 2 * j, s = item % kPRing;
        if (!wait_cl(&full[s], (item / kPRing) & 1, p.status)) return false;
        tc::fence_after();
        const uint32_t stg = sRing + s * kPStage;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const int d0 = ks * 16;
          const uint64_t ad = tc::desc_kmajor_sw128(sQ + (d0 >> 6) * (PBM * 128) + (d0 & 63) * 2);
          const uint64_t bd = tc::desc_kmajor_sw128(stg + (d0 >> 6) * 8192 + (d0 & 63) * 2);
          tc2::mma_ss(tS, ad, bd, idS, ks ? 1u : 0u);
        }
        tc2::commit_mc(&empty[s], both);
        tc2::commit_mc(sfull, both);
        return true;
      };
      auto issue_PV = [&](int j) -> bool {
        const int item = 2 * j + 1, s = item % kPRing;
        if (!wait_cl(&full[s], (item / kPRing) & 1, p.status)) return false;
        tc::fence_after();
        const uint32_t stg = sRing + s * kPStage;
#pragma unroll
        for (int kk = 0; kk < PBN / 16; ++kk) {
          const int key0 = kk * 16;
          const uint64_t ad = tc::desc_kmajor_sw128(sP + (key0 >> 6) * (PBM * 128) + (key0 & 63) * 2);
          const uint64_t bd = tc::desc_mnmajor_sw128(stg + kk * 16 * 128, PBN * 128, 1024);
          tc2::mma_ss(tO, ad, bd, idO, (j | kk) ? 1u : 0u);
        }
        tc2::commit_mc(&empty[s], both);
        tc2::commit_mc(odone, both);
        return true;
      };
      if (ok) ok = issue_S(0);
      for (int j = 0; j < n_tiles && ok; ++j) {
        if (j + 1 < n_tiles) {
          if (!wait_cl(sfree, j & 1, p.status)) break;
          tc::fence_after();
          if (!issue_S(j + 1)) break;
        }
        if (!wait_cl(pfull, j & 1, p.status)) break;
        tc::fence_after();
        if (!issue_PV(j)) break;
      }
      tc2::commit_mc(fin, 0x1);  // this CTA only; same cta_group as the MMAs it tracks
      mbar_wait(fin, 0, p.status);
    }
    __syncwarp();
  } else {
    // ---------------- softmax / correction / epilogue: this CTA's 128 rows ----------------
    // two warps per TMEM lane quarter, each owning 64 of the 128 key columns (and d/2 of O)
    const int sw = warp - 2;
    const int q4 = warp & 3;
    const int half = sw >> 2;
    const int row = q4 * 32 + lane;
    const int row_g = r0 + row;
    const uint32_t tl = tbase + ((uint32_t)(q4 * 32) << 16);
    const uint32_t tS = tl + L::kSCol + half * (PBN / 2), tO = tl + L::kOCol + half * (D / 2);
    float *xch = reinterpret_cast<float *>(sm + L::oX);
    const float cs = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const bool w1 = wait_cl(sfull, j & 1, p.status);
      tc::fence_after();
      uint32_t r[2][32];
      tc::ld32(tS, r[0]);
      tc::ld32(tS + 32, r[1]);
      tc::wait_ld();
      tc::regfence(r[0]);
      tc::regfence(r[1]);
      const int key0 = j * PBN + half * (PBN / 2);
      if ((key0 + PBN / 2 > p.T) || (p.causal && key0 + PBN / 2 - 1 > row_g)) {
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int key = key0 + c * 32 + i;
            if (key >= p.T || (p.causal && key > row_g)) r[c][i] = __float_as_uint(-INFINITY);
          }
      }
      float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          a0 = fmaxf(a0, __uint_as_float(r[c][i]));
          a1 = fmaxf(a1, __uint_as_float(r[c][i + 1]));
          a2 = fmaxf(a2, __uint_as_float(r[c][i + 2]));
          a3 = fmaxf(a3, __uint_as_float(r[c][i + 3]));
        }
      float mx = fmaxf(fmaxf(a0, a1), fmaxf(a2, a3));
      xch[half * 128 + row] = mx;
      tc::fence_before();  // both warps' S loads completed before the pair barrier
      if (!pair_bar2_and(1 + q4, w1)) {
        ok = false;
        break;
      }
      mx = fmaxf(mx, xch[(1 - half) * 128 + row]) * cs;
      if (half == 0 && lane == 0) {
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
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float e0 = ex2a(fmaf(__uint_as_float(r[c][i]), cs, nb));
          const float e1 = ex2a(fmaf(__uint_as_float(r[c][i + 1]), cs, nb));
          const float e2 = ex2a(fmaf(__uint_as_float(r[c][i + 2]), cs, nb));
          const float e3 = ex2a(fmaf(__uint_as_float(r[c][i + 3]), cs, nb));
          s0 += e0;
          s1 += e1;
          s2 += e2;
          s3 += e3;
          r[c][i] = pack_bf16(e0, e1);
          r[c][i + 2] = pack_bf16(e2, e3);
        }
      l_run = l_run * alpha + ((s0 + s1) + (s2 + s3));
      bool w2 = true;
      if (j > 0) {
        w2 = wait_cl(odone, (j - 1) & 1, p.status);
        tc::fence_after();
      }
      if (__any_sync(0xffffffffu, resc)) {
#pragma unroll 1
        for (int c = 0; c < D / 64; ++c) {
          uint32_t ov[32];
          tc::ld32(tO + c * 32, ov);
          tc::wait_ld();
          tc::regfence(ov);
          float f[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(ov[i]) * alpha;
          tc::st32(tO + c * 32, f);
        }
        tc::wait_st();
      }
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        const int c = ch >> 2, i0 = (ch & 3) * 8;
        const uint32_t addr = sP + half * (PBM * 128) + row * 128 + ((ch ^ (row & 7)) << 4);
        st_shared_v4p(addr, r[c][i0], r[c][i0 + 2], r[c][i0 + 4], r[c][i0 + 6]);
      }
      tc::fence_proxy_async_smem();
      tc::fence_before();
      if (!pair_bar2_and(5 + q4, w2)) {
        ok = false;
        break;
      }
      if (half == 0 && lane == 0) {
        if (leader) mbar_arrive(pfull);
        else tc2::remote_arrive(pfull_l);
      }
    }
    if (ok && n_tiles > 0) {
      const bool w3 = wait_cl(odone, (n_tiles - 1) & 1, p.status);
      tc::fence_after();
      xch[half * 128 + row] = l_run;
      ok = pair_bar2_and(1 + q4, w3);
    }
    if (ok && n_tiles > 0) {
      const float l_tot = l_run + xch[(1 - half) * 128 + row];
      const float inv_l = l_tot > 0.f ? 1.f / l_tot : 0.f;
      const bool valid = row_g < p.T;
      const size_t obase = (((size_t)b * p.T + (valid ? row_g : 0)) * p.q_heads + qh) * D + half * (D / 2);
      const bf16_t *gp = p.gate ? p.gate + obase : nullptr;
      float rs = 1.f;
      if (p.rms) {
        float ss = 0.f;
#pragma unroll 1
        for (int c = 0; c < D / 64; ++c) {
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
        pair_bar2(1 + q4);
        xch[half * 128 + row] = ss;
        pair_bar2(1 + q4);
        ss += xch[(1 - half) * 128 + row];
        rs = rsqrtf(ss / (float)D + p.eps);
      }
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {
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
