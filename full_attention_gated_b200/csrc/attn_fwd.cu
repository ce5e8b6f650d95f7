// attn_fwd.cu -- causal grouped-query softmax attention over a sequence
// (prefill), with the optional sigmoid output gate and the optional per-head
// RMS fusion used by the head-level hybrid layer.
//
// The attention layers of the hybrid stack are ordinary softmax attention with
// 24 query heads over 4 key/value heads at head dim 256 ("The Hybrid Attention
// in Qwen3.8-27B", "Grouped-query attention multiplies on top of that"); in the
// HydraHead layer the FA heads are softmax heads of head dim 128 with their own
// K/V ("HydraHead ...", abstract).  The pages print no kernel; this is a flash
// attention (online softmax, no T x T matrix in memory):
//   o_t = sum_{j<=t} exp(s_tj - m_t) v_j / sum_{j<=t} exp(s_tj - m_t),
//   s_tj = scale q_t . k_j,  then o_t *= sigmoid(G_t) when a gate is given.
//
// This file is the warp-MMA path: CTA = (64-query block, head, sequence); a
// producer warp streams 64-key K/V tiles with TMA (128-byte swizzle) into a
// 2-stage mbarrier ring; four consumer warps each own 16 query rows and run
// S = Q K^T and O += P V as bf16 MMAs with fp32 accumulators and a
// register-resident online softmax (exp2 domain).  Causal blocks are visited
// longest first.
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"

namespace hh {

namespace {

constexpr int kBM = 64, kBN = 64;
constexpr int kStagesF = 2;
constexpr int kCWarps = 4;
constexpr int kThreadsF = (kCWarps + 1) * 32;
constexpr float kLog2eF = 1.4426950408889634f;

struct FwdParams {
  CUtensorMap tm_q, tm_k, tm_v;  // 4-D: (d, heads, T, B)
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
struct FwdSmem {
  static constexpr int kBoxes = D / 64;
  static constexpr int kBoxBytes = 64 * 128;  // 64 rows x 128 bytes
  static constexpr int kTile = kBoxes * kBoxBytes;
  static constexpr int kQ = kTile;  // 64 query rows
  static constexpr int kStage = 2 * kTile;
  static constexpr int kTotal = kQ + kStagesF * kStage + (2 * kStagesF + 1) * 8 + 1024;
};

template <int D>
__global__ void __launch_bounds__(kThreadsF, 1) attn_fwd_mma_kernel(const __grid_constant__ FwdParams p) {
  using L = FwdSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *q_s = smem;
  uint8_t *ring = smem + L::kQ;
  uint64_t *full = reinterpret_cast<uint64_t *>(ring + kStagesF * L::kStage);
  uint64_t *empty = full + kStagesF;
  uint64_t *qbar = empty + kStagesF;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qblk = p.causal ? (p.n_qblocks - 1 - (int)blockIdx.x) : (int)blockIdx.x;
  const int hi = blockIdx.y, b = blockIdx.z;
  const int qh = p.use_map ? p.map[hi] : hi;
  const int kh = p.use_map ? p.map[hi] : hi / p.group;
  const int m0 = qblk * kBM;
  const int kv_end = p.causal ? min(p.T, m0 + kBM) : p.T;
  const int n_tiles = (kv_end + kBN - 1) / kBN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesF; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCWarps);
    }
    mbar_init(qbar, 1);
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kCWarps) {
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      mbar_arrive_expect_tx(qbar, L::kQ);
      for (int bx = 0; bx < L::kBoxes; ++bx)
        tma_load_4d(smem_u32(q_s + bx * L::kBoxBytes), &p.tm_q, qbar, bx * 64, qh, m0, b);
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i % kStagesF;
        if (i >= kStagesF && !mbar_wait(&empty[s], ((i / kStagesF) - 1) & 1, p.status)) break;
        mbar_arrive_expect_tx(&full[s], L::kStage);
        const uint32_t dk = smem_u32(ring + s * L::kStage), dv = dk + L::kTile;
        for (int bx = 0; bx < L::kBoxes; ++bx) {
          tma_load_4d(dk + bx * L::kBoxBytes, &p.tm_k, &full[s], bx * 64, kh, i * kBN, b);
          tma_load_4d(dv + bx * L::kBoxBytes, &p.tm_v, &full[s], bx * 64, kh, i * kBN, b);
        }
      }
    }
    return;
  }

  // ---------------- consumer warps: rows m0 + warp*16 .. +15 ----------------
  constexpr int NO = D / 8;  // output n-tiles
  float o[NO][4];
#pragma unroll
  for (int j = 0; j < NO; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  const uint32_t qbase = smem_u32(q_s);
  const int qrow_lane = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;  // A-operand row address
  const int row_a = m0 + warp * 16 + (lane >> 2);                        // rows of c0/c1 (c2/c3: +8)
  bool ok = mbar_wait(qbar, 0, p.status);

  for (int i = 0; i < n_tiles && ok; ++i) {
    const int s = i % kStagesF;
    if (!mbar_wait(&full[s], (i / kStagesF) & 1, p.status)) { ok = false; break; }
    const uint32_t kb = smem_u32(ring + s * L::kStage), vb = kb + L::kTile;
    float sc[kBN / 8][4];
#pragma unroll
    for (int j = 0; j < kBN / 8; ++j) sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t a[4];
      ldsm_x4(qbase + (ks >> 2) * L::kBoxBytes + sw128(qrow_lane, (ks & 3) * 2 + (lane >> 4)), a[0], a[1], a[2], a[3]);
#pragma unroll
      for (int nj = 0; nj < kBN / 16; ++nj) {
        uint32_t b0, b1, b2, b3;
        const int krow = nj * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
        const int kchunk = (ks & 3) * 2 + ((lane >> 3) & 1);
        ldsm_x4(kb + (ks >> 2) * L::kBoxBytes + sw128(krow, kchunk), b0, b1, b2, b3);
        mma_bf16_16816(sc[2 * nj], a, b0, b1);
        mma_bf16_16816(sc[2 * nj + 1], a, b2, b3);
      }
    }
    // scale + mask (causal diagonal tile, ragged end)
    const int key_base = i * kBN + (lane & 3) * 2;
    const bool need_mask = (i * kBN + kBN > kv_end) || (p.causal && i * kBN + kBN > m0);
#pragma unroll
    for (int j = 0; j < kBN / 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float v = sc[j][e] * p.scale_log2;
        if (need_mask) {
          const int key = key_base + j * 8 + (e & 1);
          const int row = row_a + (e >> 1) * 8;
          if (key >= p.T || (p.causal && key > row)) v = -INFINITY;
        }
        sc[j][e] = v;
      }
    // online softmax per row (two rows per thread: e>>1)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < kBN / 8; ++j) mx = fmaxf(mx, fmaxf(sc[j][2 * r], sc[j][2 * r + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m_run[r], mx);
      const float base = m_new == -INFINITY ? 0.f : m_new;
      const float alpha = exp2f(m_run[r] - base);
      m_run[r] = m_new;
      float ls = 0.f;
#pragma unroll
      for (int j = 0; j < kBN / 8; ++j) {
        sc[j][2 * r] = exp2f(sc[j][2 * r] - base);
        sc[j][2 * r + 1] = exp2f(sc[j][2 * r + 1] - base);
        ls += sc[j][2 * r] + sc[j][2 * r + 1];
      }
      l_run[r] = l_run[r] * alpha + ls;
#pragma unroll
      for (int j = 0; j < NO; ++j) {
        o[j][2 * r] *= alpha;
        o[j][2 * r + 1] *= alpha;
      }
    }
    // O += P V  (P fragments straight from the score accumulators)
#pragma unroll
    for (int kk = 0; kk < kBN / 16; ++kk) {
      uint32_t a[4];
      a[0] = pack_bf16(sc[2 * kk][0], sc[2 * kk][1]);
      a[1] = pack_bf16(sc[2 * kk][2], sc[2 * kk][3]);
      a[2] = pack_bf16(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
      a[3] = pack_bf16(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
      const int vkey = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int nd = 0; nd < D / 16; ++nd) {
        uint32_t b0, b1, b2, b3;
        const int dcol = nd * 16 + ((lane >> 4) & 1) * 8;
        ldsm_x4_t(vb + (dcol >> 6) * L::kBoxBytes + sw128(vkey, (dcol & 63) >> 3), b0, b1, b2, b3);
        mma_bf16_16816(o[2 * nd], a, b0, b1);
        mma_bf16_16816(o[2 * nd + 1], a, b2, b3);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }

  // ---------------- epilogue ----------------
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    float l = l_run[r];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    l_run[r] = l > 0.f ? 1.f / l : 0.f;
  }
  float rs[2] = {1.f, 1.f};
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int row = row_a + r * 8;
    const size_t gbase = (((size_t)b * p.T + (row < p.T ? row : 0)) * p.q_heads + qh) * D;
#pragma unroll
    for (int j = 0; j < NO; ++j) {
      float v0 = o[j][2 * r] * l_run[r], v1 = o[j][2 * r + 1] * l_run[r];
      if (p.gate && row < p.T) {
        const uint32_t gg = *reinterpret_cast<const uint32_t *>(p.gate + gbase + j * 8 + (lane & 3) * 2);
        v0 *= 1.f / (1.f + expf(-bf16_lo(gg)));
        v1 *= 1.f / (1.f + expf(-bf16_hi(gg)));
      }
      o[j][2 * r] = v0;
      o[j][2 * r + 1] = v1;
    }
    if (p.rms) {
      float ss = 0.f;
#pragma unroll
      for (int j = 0; j < NO; ++j) ss += o[j][2 * r] * o[j][2 * r] + o[j][2 * r + 1] * o[j][2 * r + 1];
      ss += __shfl_xor_sync(0xffffffffu, ss, 1);
      ss += __shfl_xor_sync(0xffffffffu, ss, 2);
      rs[r] = rsqrtf(ss / D + p.eps);
    }
    if (row < p.T) {
      bf16_t *dst = p.o + (((size_t)b * p.T + row) * p.q_heads + qh) * D + (lane & 3) * 2;
#pragma unroll
      for (int j = 0; j < NO; ++j)
        *reinterpret_cast<uint32_t *>(dst + j * 8) = pack_bf16(o[j][2 * r] * rs[r], o[j][2 * r + 1] * rs[r]);
    }
  }
}

template <int D>
cudaError_t launch_fwd(const FwdParams &p, cudaStream_t s) {
  auto kern = attn_fwd_mma_kernel<D>;
  const int smem = FwdSmem<D>::kTotal;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.n_qblocks, p.n_heads, p.B);
  kern<<<grid, kThreadsF, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd(const AttnFwdArgs &a, cudaStream_t s) {
  if (a.B == 0 || a.T == 0 || a.n_heads == 0) return cudaSuccess;
  // d = 256: CTA pairs (M = 256 across two SMs, each CTA streams half of every K/V tile, so
  // two tiles stay in flight); d = 128: one CTA per 128 rows (its ring already holds two tiles,
  // and the pair's cross-CTA handshakes cost more than they save): 13.0 vs 14.1 ms at
  // T = 32768 / d = 256 and 4.7 vs 7.0 ms at T = 65536 / d = 128 on B200.
  return a.d == 256 ? launch_attn_fwd_pair(a, s) : launch_attn_fwd_tc(a, s);
  FwdParams p;
  memset(&p, 0, sizeof(p));
  const uint32_t box[4] = {64, 1, (uint32_t)kBM, 1};
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
  p.scale_log2 = a.scale * kLog2eF;
  p.causal = a.causal;
  p.rms = a.rms;
  p.eps = a.eps;
  p.n_qblocks = (a.T + kBM - 1) / kBM;
  p.status = device_status_ptr();
  return a.d == 256 ? launch_fwd<256>(p, s) : launch_fwd<128>(p, s);
}

}  // namespace hh
