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
// CTA = one tile of 128 query rows of one head, eighteen warps:
//   warp 0      TMA producer: Q once, then K and V of every 128-key tile through a
//               ring of four 32 KiB stages (K in 128-key x 128-d chunks, V in
//               key chunks of 32 KiB), 128-byte swizzle, rows past T zero-filled;
//   warp 1      allocates tensor memory and issues the MMAs from one thread:
//               S = Q K^T (M=128, N=128, bf16 K-major operands) into TMEM and
//               O += P V (M=128, N=d, V MN-major) into a d-column TMEM accumulator;
//   warps 2-17  softmax, four warps per TMEM lane quarter, each owning a quarter of the
//               key columns of its 32 rows (row maxima exchanged as fp16 rounded up, row
//               sums as fp32, through shared memory): mask, running max with lazy
//               rescaling (O in TMEM is only rescaled when the max grows by more than
//               2^8), exp2, row sums, P as bf16 pairs into tensor memory, where it is the
//               A operand of O += P V; at the end read O from TMEM, divide by the row
//               sum, apply gate / RMS, store.
// S of tile j+1 is computed while the softmax works on tile j; O += P V of tile j
// runs while the softmax works on tile j+1.  Query tiles are scheduled longest
// first (causal), heads of one kv group next to each other (K/V reuse in L2).
// Dispatched for d = 128; d = 256 runs on CTA pairs (attn_fwd_tc2.cu).
#include <cuda_fp16.h>
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
constexpr int kTThreads = 576;  // producer, MMA, 16 softmax warps
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
  static constexpr int kP = 2048;          // final row sums [4][128] fp32 (P itself is in TMEM)
  static constexpr int kKSt = D / 128;     // K stages per KV tile (128 keys x 128 d each)
  static constexpr int kVK = 16384 / D;    // keys per V stage (32 KiB of V)
  static constexpr int kVSt = TBN / kVK;   // V stages per KV tile
  static constexpr int kSPT = kKSt + kVSt; // ring items per KV tile
  static constexpr int oQ = 0, oP = kQ, oRing = kQ + kP, oBar = oRing + kTRing * kTStage;
  static constexpr int kBars = 2 * kTRing + 6;
  static constexpr int oX = oBar + kBars * 8 + 16;  // row-maximum exchange [4][128] fp16
  static constexpr int kTotal = oX + 1024 + 1024;
  static constexpr uint32_t kTmemCols = 512;
  // O (d columns), S (128 columns), P as bf16 pairs (64 columns): the A operand of O += P V
  static constexpr uint32_t kOCol = 0, kSCol = D, kPCol = D + TBN;
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
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
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
    mbar_init(sfull, 1);
    mbar_init(sfree, 4);  // one arrival per TMEM lane quarter (four warps)
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
            const uint64_t bd = tc::desc_mnmajor_sw128(sRing + s * kTStage + kk * 16 * 128, L::kVK * 128, 1024);
            tc::mma_ts(tO, tbase + L::kPCol + key0 / 2, bd, idO, (j | vs | kk) ? 1u : 0u);
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
    // four warps per TMEM lane quarter, each owning 32 of the 128 key columns (and d/4 of O);
    // row maxima are exchanged as fp16 rounded up (every warp of the row reads the same four
    // values, so all agree on the maximum), the final row sums in fp32 through the P tile
    const int sw = warp - 2;
    const int q4 = warp & 3;
    const int part = sw >> 2;  // 0..3
    const int row = q4 * 32 + lane;
    const int row_g = m0 + row;
    const uint32_t tl = tbase + ((uint32_t)(q4 * 32) << 16);
    const uint32_t tS = tl + L::kSCol + part * 32, tO = tl + L::kOCol + part * (D / 4);
    __half *xmx = reinterpret_cast<__half *>(sm + L::oX);  // [4][128]
    const float cs = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const bool w1 = mbar_wait(sfull, j & 1, p.status);
      tc::fence_after();
      uint32_t r[32];
      tc::ld32(tS, r);
      tc::wait_ld();
      tc::regfence(r);
      const int key0 = j * TBN + part * 32;
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
      if (part == 0 && lane == 0) mbar_arrive(sfree);

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
      l_run = l_run * alpha + ((s0 + s1) + (s2 + s3));
      bool w2 = true;
      if (j > 0) {
        w2 = mbar_wait(odone, (j - 1) & 1, p.status);
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
      if (part == 0 && lane == 0) mbar_arrive(pfull);
    }
    float *xsum = reinterpret_cast<float *>(sm + L::oP);  // [4][128] fp32 final row sums
    if (ok && n_tiles > 0) {
      const bool w3 = mbar_wait(odone, (n_tiles - 1) & 1, p.status);
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
