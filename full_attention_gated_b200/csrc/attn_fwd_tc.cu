// attn_fwd_tc.cu -- causal grouped-query softmax attention (prefill) on the
// 5th-generation tensor cores (tcgen05, accumulators in tensor memory).
//
// What is computed is the same as in attn_fwd.cu: per query head and position,
//   o_t = sum_{j<=t} exp(s_tj - m_t) v_j / sum_j exp(s_tj - m_t),  s_tj = scale q_t.k_j,
// then o_t *= sigmoid(G_t) for a gated layer, or the per-head RMS fusion of the
// head-level hybrid layer.  The attention layers of the hybrid stack have 24
// query heads over 4 key/value heads at head dim 256 ("The Hybrid Attention in
// Qwen3.8-27B", "Grouped-query attention multiplies on top of that"); the FA heads
// of the HydraHead layer use head dim 128.
//
// CTA = one tile of 128 query rows of one head, ten warps:
//   warp 0      TMA producer: Q once, then K and V of every 128-key tile through a
//               ring of four 32 KiB stages (K in 128-key x 128-d chunks, V in
//               key chunks of 32 KiB), 128-byte swizzle, rows past T zero-filled;
//   warp 1      allocates tensor memory and issues the MMAs from one thread:
//               S = Q K^T (M=128, N=128, bf16 K-major operands) into TMEM and
//               O += P V (M=128, N=d, V MN-major) into a d-column TMEM accumulator;
//   warps 2-9   softmax, two warps per TMEM lane quarter, each owning half of the key
//               columns of its 32 rows (row maxima and sums exchanged through shared
//               memory): mask, running max with lazy rescaling (O in TMEM is only
//               rescaled when the max grows by more than 2^8), exp2, row sums, P as
//               bf16 into shared memory in the UMMA K-major swizzled layout; at the
//               end read O from TMEM, divide by the row sum, apply gate / RMS, store.
// S of tile j+1 is computed while the softmax works on tile j; O += P V of tile j
// runs while the softmax works on tile j+1.  Query tiles are scheduled longest
// first (causal), heads of one kv group next to each other (K/V reuse in L2).
// Dispatched for d = 128; d = 256 runs on CTA pairs (attn_fwd_tc2.cu).
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace hh {

namespace {

constexpr int TBM = 128, TBN = 128;
constexpr int kTStage = 32768;
constexpr int kTRing = 4;
constexpr int kTThreads = 320;  // producer, MMA, 8 softmax warps
constexpr float kTLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.0f;

struct TcParams {
  CUtensorMap tm_q, tm_k, tm_v;  // 4-D (d, heads, T, B); boxes (64,1,128,1), (64,1,128,1), (64,1,VK,1)
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

template <int D>
struct TcL {
  static constexpr int kQ = TBM * D * 2;   // Q tile
  static constexpr int kP = TBM * TBN * 2; // P tile (bf16)
  static constexpr int kKSt = D / 128;     // K stages per KV tile (128 keys x 128 d each)
  static constexpr int kVK = 16384 / D;    // keys per V stage (32 KiB of V)
  static constexpr int kVSt = TBN / kVK;   // V stages per KV tile
  static constexpr int kSPT = kKSt + kVSt; // ring items per KV tile
  static constexpr int oQ = 0, oP = kQ, oRing = kQ + kP, oBar = oRing + kTRing * kTStage;
  static constexpr int kBars = 2 * kTRing + 6;
  static constexpr int oX = oBar + kBars * 8 + 16;  // row-statistics exchange [2][128] fp32
  static constexpr int kTotal = oX + 1024 + 1024;
  static constexpr uint32_t kTmemCols = D == 256 ? 512u : 256u;
  static constexpr uint32_t kOCol = 0, kSCol = D;
  static_assert(kTotal <= 232448, "shared memory budget");
};

// barrier of the two softmax warps that share a TMEM lane quarter (ids 1..4, 64 threads)
__device__ __forceinline__ void pair_bar(int id) { asm volatile("bar.sync %0, 64;\n" ::"r"(id) : "memory"); }
// the two warps of a TMEM lane quarter meet and AND their predicates, so a wait that gave up in
// either warp ends both together (neither is left waiting at a later pair barrier)
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
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

template <int D>
__global__ void __launch_bounds__(kTThreads, 1) attn_fwd_tc_kernel(const __grid_constant__ TcParams p) {
  using L = TcL<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(sm + L::oBar);
  uint64_t *empty = full + kTRing;
  uint64_t *qfull = full + 2 * kTRing;
  uint64_t *sfull = qfull + 1, *sfree = qfull + 2, *pfull = qfull + 3, *odone = qfull + 4, *fin = qfull + 5;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::oBar + L::kBars * 8);
  const uint32_t sQ = smem_u32(sm + L::oQ), sP = smem_u32(sm + L::oP), sRing = smem_u32(sm + L::oRing);

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
    mbar_init(sfull, 1);
    mbar_init(sfree, 4);  // one arrival per TMEM lane quarter (warp pair)
    mbar_init(pfull, 4);
    mbar_init(odone, 1);
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
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      mbar_arrive_expect_tx(qfull, L::kQ);
      for (int bx = 0; bx < D / 64; ++bx) tma_load_4d(sQ + bx * (TBM * 128), &p.tm_q, qfull, bx * 64, qh, m0, b);
      int item = 0;
      bool ok = true;
      for (int j = 0; j < n_tiles && ok; ++j) {
        for (int ks = 0; ks < L::kKSt && ok; ++ks, ++item) {
          const int s = item % kTRing;
          if (item >= kTRing && !mbar_wait(&empty[s], ((item / kTRing) - 1) & 1, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], kTStage);
          const uint32_t dst = sRing + s * kTStage;
          tma_load_4d(dst, &p.tm_k, &full[s], ks * 128, kh, j * TBN, b);
          tma_load_4d(dst + 16384, &p.tm_k, &full[s], ks * 128 + 64, kh, j * TBN, b);
        }
        for (int vs = 0; vs < L::kVSt && ok; ++vs, ++item) {
          const int s = item % kTRing;
          if (item >= kTRing && !mbar_wait(&empty[s], ((item / kTRing) - 1) & 1, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], kTStage);
          const uint32_t dst = sRing + s * kTStage;
          for (int bx = 0; bx < D / 64; ++bx)
            tma_load_4d(dst + bx * (L::kVK * 128), &p.tm_v, &full[s], bx * 64, kh, j * TBN + vs * L::kVK, b);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer (one thread) ----------------
    if (lane == 0) {
      const uint32_t tS = tbase + L::kSCol, tO = tbase + L::kOCol;
      constexpr uint32_t idS = tc::idesc_bf16_f32(128, TBN, 0, 0);
      constexpr uint32_t idO = tc::idesc_bf16_f32(128, D, 0, 1);
      bool ok = mbar_wait(qfull, 0, p.status);
      tc::fence_after();
      auto issue_S = [&](int j) -> bool {
        for (int ks = 0; ks < L::kKSt; ++ks) {
          const int item = j * L::kSPT + ks, s = item % kTRing;
          if (!mbar_wait(&full[s], (item / kTRing) & 1, p.status)) return false;
          tc::fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const int d0 = ks * 128 + kk * 16;
            const uint64_t ad = tc::desc_kmajor_sw128(sQ + (d0 >> 6) * (TBM * 128) + (d0 & 63) * 2);
            const uint64_t bd = tc::desc_kmajor_sw128(sRing + s * kTStage + ((kk * 16) >> 6) * 16384 + ((kk * 16) & 63) * 2);
            tc::mma_ss(tS, ad, bd, idS, (ks | kk) ? 1u : 0u);
          }
          tc::commit(&empty[s]);
        }
        tc::commit(sfull);
        return true;
      };
      auto issue_PV = [&](int j) -> bool {
        for (int vs = 0; vs < L::kVSt; ++vs) {
          const int item = j * L::kSPT + L::kKSt + vs, s = item % kTRing;
          if (!mbar_wait(&full[s], (item / kTRing) & 1, p.status)) return false;
          tc::fence_after();
#pragma unroll
          for (int kk = 0; kk < L::kVK / 16; ++kk) {
            const int key0 = vs * L::kVK + kk * 16;
            const uint64_t ad = tc::desc_kmajor_sw128(sP + (key0 >> 6) * (TBM * 128) + (key0 & 63) * 2);
            const uint64_t bd = tc::desc_mnmajor_sw128(sRing + s * kTStage + kk * 16 * 128, L::kVK * 128, 1024);
            tc::mma_ss(tO, ad, bd, idO, (j | vs | kk) ? 1u : 0u);
          }
          tc::commit(&empty[s]);
        }
        tc::commit(odone);
        return true;
      };
      if (ok) ok = issue_S(0);
      for (int j = 0; j < n_tiles && ok; ++j) {
        if (j + 1 < n_tiles) {
          if (!mbar_wait(sfree, j & 1, p.status)) break;
          tc::fence_after();
          if (!issue_S(j + 1)) break;
        }
        if (!mbar_wait(pfull, j & 1, p.status)) break;
        tc::fence_after();
        if (!issue_PV(j)) break;
      }
      // every MMA issued above must be complete before the CTA releases tensor memory
      tc::commit(fin);
      mbar_wait(fin, 0, p.status);
    }
    __syncwarp();
  } else {
    // ---------------- softmax / correction / epilogue ----------------
    // Two warps per TMEM lane quarter: warp 2+i owns rows 32*q .. 32*q+31 (q = warp % 4)
    // and half h = i / 4 of the columns of S (keys) and of O.  Row maxima are
    // exchanged with the partner warp through shared memory; row sums are kept
    // per half and joined at the end.
    const int sw = warp - 2;
    const int q4 = warp & 3;
    const int half = sw >> 2;
    const int row = q4 * 32 + lane;
    const int row_g = m0 + row;
    const uint32_t tl = tbase + ((uint32_t)(q4 * 32) << 16);
    const uint32_t tS = tl + L::kSCol + half * (TBN / 2), tO = tl + L::kOCol + half * (D / 2);
    float *xch = reinterpret_cast<float *>(sm + L::oX);  // [2 halves][128 rows]
    const float cs = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const bool w1 = mbar_wait(sfull, j & 1, p.status);
      tc::fence_after();
      uint32_t r[2][32];
      tc::ld32(tS, r[0]);
      tc::ld32(tS + 32, r[1]);
      tc::wait_ld();
      tc::regfence(r[0]);
      tc::regfence(r[1]);
      const int key0 = j * TBN + half * (TBN / 2);
      if ((key0 + TBN / 2 > p.T) || (p.causal && key0 + TBN / 2 - 1 > row_g)) {
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
      if (!pair_bar_and(1 + q4, w1)) {
        ok = false;
        break;
      }
      mx = fmaxf(mx, xch[(1 - half) * 128 + row]) * cs;  // row max of the scaled scores (cs > 0)
      // both halves of S are in registers: the next S may overwrite them
      if (half == 0 && lane == 0) mbar_arrive(sfree);

      float alpha = 1.f;
      bool resc = false;
      if (j == 0) {
        m_run = mx;
      } else if (mx > m_run + kRescaleLog2) {
        alpha = ex2_approx(m_run - mx);
        m_run = mx;
        resc = true;
      }
      const float nb = m_run == -INFINITY ? 0.f : -m_run;
      float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float e0 = ex2_approx(fmaf(__uint_as_float(r[c][i]), cs, nb));
          const float e1 = ex2_approx(fmaf(__uint_as_float(r[c][i + 1]), cs, nb));
          const float e2 = ex2_approx(fmaf(__uint_as_float(r[c][i + 2]), cs, nb));
          const float e3 = ex2_approx(fmaf(__uint_as_float(r[c][i + 3]), cs, nb));
          s0 += e0;
          s1 += e1;
          s2 += e2;
          s3 += e3;
          r[c][i] = pack_bf16(e0, e1);
          r[c][i + 2] = pack_bf16(e2, e3);
        }
      l_run = l_run * alpha + ((s0 + s1) + (s2 + s3));
      // O and the P buffer are free once O += P V of the previous tile has completed
      bool w2 = true;
      if (j > 0) {
        w2 = mbar_wait(odone, (j - 1) & 1, p.status);
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
      // this half's 64 keys of the P row -> one 128-byte-swizzled P box (bf16, K-major)
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        const int c = ch >> 2, i0 = (ch & 3) * 8;
        const uint32_t addr = sP + half * (TBM * 128) + row * 128 + ((ch ^ (row & 7)) << 4);
        st_shared_v4(addr, r[c][i0], r[c][i0 + 2], r[c][i0 + 4], r[c][i0 + 6]);
      }
      tc::fence_proxy_async_smem();
      tc::fence_before();
      if (!pair_bar_and(5 + q4, w2)) {
        ok = false;
        break;
      }
      if (half == 0 && lane == 0) mbar_arrive(pfull);
    }
    if (ok && n_tiles > 0) {
      const bool w3 = mbar_wait(odone, (n_tiles - 1) & 1, p.status);
      tc::fence_after();
      xch[half * 128 + row] = l_run;
      ok = pair_bar_and(1 + q4, w3);
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
        pair_bar(1 + q4);  // both halves have read l_tot before the slot is reused
        xch[half * 128 + row] = ss;
        pair_bar(1 + q4);
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
  __syncthreads();
  if (warp == 1) {
    tc::fence_after();
    tc::tmem_dealloc(tbase, L::kTmemCols);
  }
}

template <int D>
cudaError_t launch_tc(const TcParams &p, cudaStream_t s) {
  auto kern = attn_fwd_tc_kernel<D>;
  const int smem = TcL<D>::kTotal;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const long long grid = (long long)p.n_qblocks * p.n_heads * p.B;
  kern<<<(unsigned)grid, kTThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd_tc(const AttnFwdArgs &a, cudaStream_t s) {
  if (a.B == 0 || a.T == 0 || a.n_heads == 0) return cudaSuccess;
  TcParams p;
  memset(&p, 0, sizeof(p));
  const int vk = 16384 / a.d;
  const uint32_t box_q[4] = {64, 1, (uint32_t)TBM, 1};
  const uint32_t box_v[4] = {64, 1, (uint32_t)vk, 1};
  const uint64_t dq[4] = {(uint64_t)a.d, (uint64_t)a.q_heads, (uint64_t)a.T, (uint64_t)a.B};
  const uint64_t sq[3] = {(uint64_t)a.d * 2, (uint64_t)a.q_heads * a.d * 2, (uint64_t)a.T * a.q_heads * a.d * 2};
  const uint64_t dk[4] = {(uint64_t)a.d, (uint64_t)a.kv_heads, (uint64_t)a.T, (uint64_t)a.B};
  const uint64_t sk[3] = {(uint64_t)a.d * 2, (uint64_t)a.kv_heads * a.d * 2, (uint64_t)a.T * a.kv_heads * a.d * 2};
  if (encode_tmap(&p.tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.q, dq, sq, box_q, CU_TENSOR_MAP_SWIZZLE_128B) ||
      encode_tmap(&p.tm_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.k, dk, sk, box_q, CU_TENSOR_MAP_SWIZZLE_128B) ||
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
  p.scale_log2 = a.scale * kTLog2e;
  p.causal = a.causal;
  p.rms = a.rms;
  p.eps = a.eps;
  p.n_qblocks = (a.T + TBM - 1) / TBM;
  p.status = device_status_ptr();
  return a.d == 256 ? launch_tc<256>(p, s) : launch_tc<128>(p, s);
}

}  // namespace hh
