// attn_decode.cu -- one new query per sequence against a bf16 KV cache
// (grouped-query attention decode).
//
// Only the attention layers "grow a KV cache", and with 24 query heads over 4
// key/value heads every cached key/value row serves six query heads ("The
// Hybrid Attention in Qwen3.8-27B", sections "Why 27B parameters can carry 262K
// tokens" and "Grouped-query attention multiplies on top of that").  The step
// is a single stream over the cache: every K and V row of a (sequence, kv head)
// is read once from HBM and used for all query heads of its group.
//
// Kernel 1 (split): CTA = (split, kv head, sequence).  A producer warp streams
// 64-key tiles of K and V with TMA (4-D tensor maps, 128-byte swizzle, zero
// fill past the end of the cache) into a 3-stage ring guarded by mbarriers.
// Four consumer warps each take 16 keys of a tile and run warp-level bf16 MMAs
// with the keys as M and the group's query heads as N:
//     S^T[16 keys x 8 heads]  = K[16 x d] Q^T[d x 8]
//     O^T[d x 8 heads]       += V^T[d x 16] P^T[16 x 8]
// with an online (running-max) softmax per head in fp32, exp2 domain.  The CTA
// merges its warps and writes one partial (m, l, o) per query head.
// Kernel 2 (combine): merges the splits of each (sequence, query head) by
// log-sum-exp, divides by the softmax denominator, applies the optional sigmoid
// gate, rounds to bf16.
#include <cuda_fp16.h>
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"

namespace hh {

namespace {

constexpr int kTileKeys = 64;
constexpr int kStages = 3;
constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kPtStride = 24;  // elements per row of the per-warp P^T tile (conflict-free ldmatrix)
constexpr float kLog2e = 1.4426950408889634f;

struct DecodeSplitParams {
  CUtensorMap tm_k, tm_v;  // 4-D: (d, H_kv, T_cache, B)
  const bf16_t *q;
  const int32_t *cache_len;
  float *part_o;   // [B, H_q, n_splits, D]
  float *part_ml;  // [B, H_q, n_splits, 2]
  int B, T_cache, H_q, H_kv, group, n_splits, split_len;
  float scale_log2;
  unsigned *status;
};

template <int D>
struct DecodeSmem {
  static constexpr int kBox = 64;                       // d elements per TMA box (128 bytes)
  static constexpr int kBoxes = D / kBox;               // boxes per tile row
  static constexpr int kBoxBytes = kTileKeys * 128;     // 8 KiB
  static constexpr int kTileBytes = kBoxes * kBoxBytes; // K (or V) tile
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kQStride = D + 8;                // padded Q row (elements)
  static constexpr int kQBytes = 16 * kQStride * 2;
  static constexpr int kPtBytes = kConsumerWarps * 16 * kPtStride * 2;
  static constexpr int kRedBytes = kConsumerWarps * 16 * D * 4 + 2 * kConsumerWarps * 16 * 4;
  static_assert(kRedBytes <= kStages * kStageBytes, "reduction buffer reuses the stage ring");
  static constexpr int kTotal = kStages * kStageBytes + kQBytes + kPtBytes + 2 * kStages * 8 + 1024;
};

template <int D, int NT>
__global__ void __launch_bounds__(kThreads, 1) attn_decode_split_kernel(const __grid_constant__ DecodeSplitParams p) {
  using L = DecodeSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *ring = smem;
  bf16_t *q_s = reinterpret_cast<bf16_t *>(smem + kStages * L::kStageBytes);
  bf16_t *pt_s = reinterpret_cast<bf16_t *>(smem + kStages * L::kStageBytes + L::kQBytes);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kStages * L::kStageBytes + L::kQBytes + L::kPtBytes);
  uint64_t *empty = full + kStages;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  int len = p.cache_len ? p.cache_len[b] : p.T_cache;
  len = len < 0 ? 0 : (len > p.T_cache ? p.T_cache : len);
  const int k_begin = split * p.split_len;
  const int k_end = min(k_begin + p.split_len, len);
  const int n_tiles = k_end > k_begin ? (k_end - k_begin + kTileKeys - 1) / kTileKeys : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    fence_barrier_init();
  }
  // Q of the group -> smem rows [16][D] (rows >= group are zero)
  for (int i = threadIdx.x; i < 16 * (D / 8); i += kThreads) {
    const int hrow = i / (D / 8), c = i % (D / 8);
    uint4 val = make_uint4(0, 0, 0, 0);
    if (hrow < p.group)
      val = *reinterpret_cast<const uint4 *>(p.q + ((size_t)b * p.H_q + kvh * p.group + hrow) * D + c * 8);
    *reinterpret_cast<uint4 *>(q_s + hrow * L::kQStride + c * 8) = val;
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ---------------- producer warp ----------------
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      int last = -1;
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i % kStages;
        if (i >= kStages && !mbar_wait(&empty[s], ((i / kStages) - 1) & 1, p.status)) break;
        last = i;
        mbar_arrive_expect_tx(&full[s], L::kStageBytes);
        const uint32_t dk = smem_u32(ring + s * L::kStageBytes);
        const uint32_t dv = dk + L::kTileBytes;
        const int t0 = k_begin + i * kTileKeys;
        for (int bx = 0; bx < L::kBoxes; ++bx) {
          tma_load_4d(dk + bx * L::kBoxBytes, &p.tm_k, &full[s], bx * 64, kvh, t0, b);
          tma_load_4d(dv + bx * L::kBoxBytes, &p.tm_v, &full[s], bx * 64, kvh, t0, b);
        }
      }
      // every load issued above has landed before the CTA can exit (bounded; complete on the
      // normal path, where the consumers waited for each of them)
      for (int i = max(last - kStages + 1, 0); i <= last; ++i) mbar_wait(&full[i % kStages], (i / kStages) & 1, p.status);
    }
  } else {
    // ---------------- consumer warps ----------------
    // Q^T as B operand fragments, kept in registers: [k-step][n-tile][2]
    uint32_t qb[D / 16][NT][2];
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int row = nt * 8 + (lane & 7);
        const int col = ks * 16 + ((lane >> 3) & 1) * 8;
        ldsm_x2(smem_u32(q_s + row * L::kQStride + col), qb[ks][nt][0], qb[ks][nt][1]);
      }
    float o[D / 16][NT][4];
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) o[mt][nt][0] = o[mt][nt][1] = o[mt][nt][2] = o[mt][nt][3] = 0.f;
    float m_run[NT][2], l_run[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) m_run[nt][0] = m_run[nt][1] = -INFINITY, l_run[nt][0] = l_run[nt][1] = 0.f;

    bf16_t *pt = pt_s + warp * 16 * kPtStride;
    bool ok = true;
    for (int i = 0; i < n_tiles && ok; ++i) {
      const int s = i % kStages;
      if (!mbar_wait(&full[s], (i / kStages) & 1, p.status)) { ok = false; break; }
      const uint32_t kb = smem_u32(ring + s * L::kStageBytes);
      const uint32_t vb = kb + L::kTileBytes;
      // S^T = K Q^T over D
      float sc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
      const int arow = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        uint32_t a[4];
        const int chunk = (ks & 3) * 2 + (lane >> 4);
        ldsm_x4(kb + (ks >> 2) * L::kBoxBytes + sw128(arow, chunk), a[0], a[1], a[2], a[3]);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(sc[nt], a, qb[ks][nt][0], qb[ks][nt][1]);
      }
      // mask keys past the end, scale into the log2 domain
      const int key0 = k_begin + i * kTileKeys + warp * 16 + (lane >> 2);
      const bool v0 = key0 < k_end, v1 = key0 + 8 < k_end;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        sc[nt][0] = v0 ? sc[nt][0] * p.scale_log2 : -INFINITY;
        sc[nt][1] = v0 ? sc[nt][1] * p.scale_log2 : -INFINITY;
        sc[nt][2] = v1 ? sc[nt][2] * p.scale_log2 : -INFINITY;
        sc[nt][3] = v1 ? sc[nt][3] * p.scale_log2 : -INFINITY;
      }
      // online softmax per head column (columns 2*(lane%4) and +1 of each n-tile)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float mx = fmaxf(sc[nt][c], sc[nt][c + 2]);
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
          const float m_new = fmaxf(m_run[nt][c], mx);
          const float base = m_new == -INFINITY ? 0.f : m_new;
          const float alpha = exp2f(m_run[nt][c] - base);
          m_run[nt][c] = m_new;
          const float p0 = exp2f(sc[nt][c] - base), p1 = exp2f(sc[nt][c + 2] - base);
          sc[nt][c] = p0;
          sc[nt][c + 2] = p1;
          l_run[nt][c] = l_run[nt][c] * alpha + p0 + p1;
#pragma unroll
          for (int mt = 0; mt < D / 16; ++mt) {
            o[mt][nt][c] *= alpha;
            o[mt][nt][c + 2] *= alpha;
          }
        }
        // P^T tile for this warp: pt[head][key]
        const int hd = nt * 8 + (lane & 3) * 2, ky = lane >> 2;
        pt[hd * kPtStride + ky] = f_to_bf16(sc[nt][0]);
        pt[(hd + 1) * kPtStride + ky] = f_to_bf16(sc[nt][1]);
        pt[hd * kPtStride + ky + 8] = f_to_bf16(sc[nt][2]);
        pt[(hd + 1) * kPtStride + ky + 8] = f_to_bf16(sc[nt][3]);
      }
      __syncwarp();
      uint32_t pb[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        ldsm_x2(smem_u32(pt + (nt * 8 + (lane & 7)) * kPtStride + ((lane >> 3) & 1) * 8), pb[nt][0], pb[nt][1]);
      // O^T += V^T P^T
      const int vkey = warp * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        uint32_t a[4];
        const int dcol = mt * 16 + ((lane >> 3) & 1) * 8;
        ldsm_x4_t(vb + (dcol >> 6) * L::kBoxBytes + sw128(vkey, (dcol & 63) >> 3), a[0], a[1], a[2], a[3]);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(o[mt][nt], a, pb[nt][0], pb[nt][1]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    // per-warp results -> shared reduction buffer (reuses the stage ring)
    __syncwarp();
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float l = l_run[nt][c];
        l += __shfl_xor_sync(0xffffffffu, l, 4);
        l += __shfl_xor_sync(0xffffffffu, l, 8);
        l += __shfl_xor_sync(0xffffffffu, l, 16);
        l_run[nt][c] = l;
      }
    // wait until every warp is done reading the ring before overwriting it
    asm volatile("bar.sync 1, %0;\n" ::"n"(kConsumerWarps * 32));
    float *red_o = reinterpret_cast<float *>(ring);
    float *red_m = red_o + kConsumerWarps * 16 * D;
    float *red_l = red_m + kConsumerWarps * 16;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int hd = nt * 8 + (lane & 3) * 2;
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        const int dd = mt * 16 + (lane >> 2);
        red_o[(warp * 16 + hd) * D + dd] = o[mt][nt][0];
        red_o[(warp * 16 + hd + 1) * D + dd] = o[mt][nt][1];
        red_o[(warp * 16 + hd) * D + dd + 8] = o[mt][nt][2];
        red_o[(warp * 16 + hd + 1) * D + dd + 8] = o[mt][nt][3];
      }
      if (lane < 4) {
        red_m[warp * 16 + hd] = m_run[nt][0];
        red_m[warp * 16 + hd + 1] = m_run[nt][1];
        red_l[warp * 16 + hd] = l_run[nt][0];
        red_l[warp * 16 + hd + 1] = l_run[nt][1];
      }
    }
    asm volatile("bar.sync 1, %0;\n" ::"n"(kConsumerWarps * 32));
    // merge the warps; write one partial per real query head of the group
    for (int idx = threadIdx.x; idx < p.group * D; idx += kConsumerWarps * 32) {
      const int hd = idx / D, dd = idx % D;
      float mt = -INFINITY;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) mt = fmaxf(mt, red_m[w * 16 + hd]);
      float lt = 0.f, ot = 0.f;
      if (mt != -INFINITY) {
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
          const float f = exp2f(red_m[w * 16 + hd] - mt);
          lt += red_l[w * 16 + hd] * f;
          ot += red_o[(w * 16 + hd) * D + dd] * f;
        }
      }
      const size_t row = ((size_t)b * p.H_q + kvh * p.group + hd) * p.n_splits + split;
      p.part_o[row * D + dd] = ot;
      if (dd == 0) {
        p.part_ml[row * 2 + 0] = mt;
        p.part_ml[row * 2 + 1] = lt;
      }
    }
  }
}

template <int D>
__global__ void __launch_bounds__(D) attn_decode_combine_kernel(const float *__restrict__ part_o,
                                                                const float *__restrict__ part_ml,
                                                                const bf16_t *__restrict__ gate,
                                                                bf16_t *__restrict__ out, int n_splits) {
  const size_t bh = blockIdx.x;  // b * H_q + h
  const int dd = threadIdx.x;
  const float *ml = part_ml + bh * n_splits * 2;
  float M = -INFINITY;
  for (int s = 0; s < n_splits; ++s) M = fmaxf(M, ml[2 * s]);
  float res = 0.f;
  if (M != -INFINITY) {
    float Ls = 0.f, acc = 0.f;
    for (int s = 0; s < n_splits; ++s) {
      const float f = exp2f(ml[2 * s] - M);
      Ls += ml[2 * s + 1] * f;
      acc += part_o[(bh * n_splits + s) * D + dd] * f;
    }
    res = acc / Ls;
    if (gate) res *= 1.f / (1.f + expf(-bf16_to_f(gate[bh * D + dd])));
  }
  out[bh * D + dd] = f_to_bf16(res);
}

template <int D, int NT>
cudaError_t launch_split(const DecodeSplitParams &p, cudaStream_t s) {
  auto kern = attn_decode_split_kernel<D, NT>;
  const int smem = DecodeSmem<D>::kTotal;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.n_splits, p.H_kv, p.B);
  kern<<<grid, kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// q8_0 cache ("The economics of hybrid attention", table in "What a token of
// context costs": 34 KiB per token instead of 64 KiB in f16).  Each block of 32
// consecutive elements of a cached K or V row is 32 int8 values x_i and one
// fp16 scale s, standing for s x_i.  Values and scales are two arrays:
//   values [B, T_cache, H_kv, D] int8,  scales [B, T_cache, H_kv, D/32] fp16.
// The split kernel keeps the structure of the bf16 one (TMA ring of 64-key
// tiles, keys as M, the group's query heads as N, online softmax), with the
// cache dequantised in registers:
//  * S^T = K Q^T: ldmatrix reads the int8 tile as pairs of bytes, so a thread
//    holds 4 consecutive values of a key row; they become fp16 exactly
//    (fp16(1024 + x + 128) - 1152).  A k-step of the MMA contracts its 16
//    columns in any order, so the low pair of the four is taken as the
//    fragment's first column pair and the high pair as its second, and Q's
//    fragments follow the same order.  Each 32-column block's partial scores
//    are multiplied by the key's scale in fp32.
//  * O^T += V^T P^T: the rows of O^T (value columns d) are visited in an order
//    that gives each thread 4 consecutive bytes of a V row per key, and the V
//    scale of (key, block) is folded into P: P'[key][h] = 256 s P[key][h] in
//    fp16 (the factor 256 keeps P' clear of fp16 subnormals; O is divided by
//    it exactly at the end).
// fp16 operands, fp32 accumulation.
// ---------------------------------------------------------------------------
constexpr int kQ8Stages = 3;

struct DecodeQ8Params {
  CUtensorMap tm_kx, tm_vx;  // int8 values, 4-D (D, H_kv, T_cache, B), box (128, 1, 64, 1), 128-byte swizzle
  CUtensorMap tm_ks, tm_vs;  // fp16 scales, 4-D (D/32, H_kv, T_cache, B), box (D/32, 1, 64, 1)
  const bf16_t *q;
  const int32_t *cache_len;
  float *part_o;   // [B, H_q, n_splits, D]
  float *part_ml;  // [B, H_q, n_splits, 2]
  int B, T_cache, H_q, H_kv, group, n_splits, split_len;
  float scale_log2;
  unsigned *status;
};

template <int D>
struct DecodeQ8Smem {
  static constexpr int kBoxBytes = kTileKeys * 128;             // 64 rows x 128 int8
  static constexpr int kBoxes = D / 128;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;         // K (or V) values of a tile
  static constexpr int kScaleBytes = kTileKeys * (D / 32) * 2;  // K (or V) scales of a tile
  static constexpr int kStageBytes = 2 * kTileBytes + 2 * kScaleBytes;
  static constexpr int kPtStride = 20;                          // fp32 P^T rows [head][key], padded
  static constexpr int kPtBytes = kConsumerWarps * 16 * kPtStride * 4;
  static constexpr int kRedBytes = kConsumerWarps * 16 * D * 4 + 2 * kConsumerWarps * 16 * 4;
  static_assert(kRedBytes <= kQ8Stages * kStageBytes, "reduction buffer reuses the stage ring");
  static constexpr int kTotal = kQ8Stages * kStageBytes + kPtBytes + 2 * kQ8Stages * 8 + 1024;
};

// four int8 (one 32-bit word) -> two fp16x2, exactly: low bytes (b0, b1) and high bytes (b2, b3)
__device__ __forceinline__ uint32_t i8x2_lo_f16(uint32_t w) {
  const uint32_t u = w ^ 0x80808080u;  // x + 128 in each byte
  uint32_t h;
  asm("prmt.b32 %0, %1, %2, 0x5140;\n" : "=r"(h) : "r"(u), "r"(0x64646464u));  // fp16 1024 + (x + 128)
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;\n" : "=r"(r) : "r"(h), "r"(0x64806480u));      // - 1152, exact
  return r;
}
__device__ __forceinline__ uint32_t i8x2_hi_f16(uint32_t w) {
  const uint32_t u = w ^ 0x80808080u;
  uint32_t h;
  asm("prmt.b32 %0, %1, %2, 0x5342;\n" : "=r"(h) : "r"(u), "r"(0x64646464u));
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;\n" : "=r"(r) : "r"(h), "r"(0x64806480u));
  return r;
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;\n" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;\n" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ float half_at(const uint4 &v, int i) {  // fp16 element i of 8 packed in a uint4
  const uint32_t w = i < 2 ? v.x : (i < 4 ? v.y : (i < 6 ? v.z : v.w));
  return __half2float(__ushort_as_half((unsigned short)((i & 1) ? (w >> 16) : (w & 0xFFFFu))));
}

template <int D, int NT>
__global__ void __launch_bounds__(kThreads, 2) attn_decode_q8_split_kernel(const __grid_constant__ DecodeQ8Params p) {
  using L = DecodeQ8Smem<D>;
  constexpr int NB = D / 32;  // scale blocks per row
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *ring = smem;
  float *pt_s = reinterpret_cast<float *>(smem + kQ8Stages * L::kStageBytes);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kQ8Stages * L::kStageBytes + L::kPtBytes);
  uint64_t *empty = full + kQ8Stages;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  int len = p.cache_len ? p.cache_len[b] : p.T_cache;
  len = len < 0 ? 0 : (len > p.T_cache ? p.T_cache : len);
  const int k_begin = split * p.split_len;
  const int k_end = min(k_begin + p.split_len, len);
  const int n_tiles = k_end > k_begin ? (k_end - k_begin + kTileKeys - 1) / kTileKeys : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kQ8Stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ---------------- producer warp ----------------
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_kx);
      tma_prefetch_desc(&p.tm_vx);
      tma_prefetch_desc(&p.tm_ks);
      tma_prefetch_desc(&p.tm_vs);
      int last = -1;
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i % kQ8Stages;
        if (i >= kQ8Stages && !mbar_wait(&empty[s], ((i / kQ8Stages) - 1) & 1, p.status)) break;
        last = i;
        mbar_arrive_expect_tx(&full[s], L::kStageBytes);
        const uint32_t dk = smem_u32(ring + s * L::kStageBytes), dv = dk + L::kTileBytes;
        const uint32_t dks = dk + 2 * L::kTileBytes, dvs = dks + L::kScaleBytes;
        const int t0 = k_begin + i * kTileKeys;
        for (int bx = 0; bx < L::kBoxes; ++bx) {
          tma_load_4d(dk + bx * L::kBoxBytes, &p.tm_kx, &full[s], bx * 128, kvh, t0, b);
          tma_load_4d(dv + bx * L::kBoxBytes, &p.tm_vx, &full[s], bx * 128, kvh, t0, b);
        }
        tma_load_4d(dks, &p.tm_ks, &full[s], 0, kvh, t0, b);
        tma_load_4d(dvs, &p.tm_vs, &full[s], 0, kvh, t0, b);
      }
      for (int i = max(last - kQ8Stages + 1, 0); i <= last; ++i)
        mbar_wait(&full[i % kQ8Stages], (i / kQ8Stages) & 1, p.status);
    }
  } else {
    // ---------------- consumer warps: 16 keys of each tile per warp ----------------
    const int g = lane >> 2, c4 = lane & 3;
    // Q^T fragments in fp16, columns of each k-step in the order described above
    uint32_t qb[D / 16][NT][2];
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int h = nt * 8 + g;
        uint2 w = make_uint2(0u, 0u);
        if (h < p.group)
          w = *reinterpret_cast<const uint2 *>(p.q + ((size_t)b * p.H_q + kvh * p.group + h) * D + ks * 16 + 4 * c4);
        qb[ks][nt][0] = pack_f16(bf16_lo(w.x), bf16_hi(w.x));
        qb[ks][nt][1] = pack_f16(bf16_lo(w.y), bf16_hi(w.y));
      }
    float o[D / 16][NT][4];
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) o[mt][nt][0] = o[mt][nt][1] = o[mt][nt][2] = o[mt][nt][3] = 0.f;
    float m_run[NT][2], l_run[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) m_run[nt][0] = m_run[nt][1] = -INFINITY, l_run[nt][0] = l_run[nt][1] = 0.f;

    float *pt = pt_s + warp * 16 * L::kPtStride;
    const int arow = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;  // ldmatrix row of this lane
    bool ok = true;
    for (int i = 0; i < n_tiles && ok; ++i) {
      const int s = i % kQ8Stages;
      if (!mbar_wait(&full[s], (i / kQ8Stages) & 1, p.status)) { ok = false; break; }
      const uint8_t *st = ring + s * L::kStageBytes;
      const uint32_t kb = smem_u32(st);
      const uint8_t *vx = st + L::kTileBytes;
      const uint8_t *ksc = st + 2 * L::kTileBytes, *vsc = ksc + L::kScaleBytes;
      // ---- S^T = K Q^T, block by block of 32 columns, each block scaled by its key's scale ----
      const uint4 sk0 = *reinterpret_cast<const uint4 *>(ksc + (warp * 16 + g) * NB * 2);
      const uint4 sk1 = *reinterpret_cast<const uint4 *>(ksc + (warp * 16 + g + 8) * NB * 2);
      float sc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
      for (int j = 0; j < NB; ++j) {
        uint32_t r0, r1, r2, r3;
        const int ch = 2 * j + (lane >> 4);  // 16-byte chunk of the 256-byte row
        ldsm_x4(kb + (ch >> 3) * L::kBoxBytes + sw128(arow, ch & 7), r0, r1, r2, r3);
        float tmp[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) tmp[nt][0] = tmp[nt][1] = tmp[nt][2] = tmp[nt][3] = 0.f;
        const uint32_t a0[4] = {i8x2_lo_f16(r0), i8x2_lo_f16(r1), i8x2_hi_f16(r0), i8x2_hi_f16(r1)};
        const uint32_t a1[4] = {i8x2_lo_f16(r2), i8x2_lo_f16(r3), i8x2_hi_f16(r2), i8x2_hi_f16(r3)};
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          mma_f16_16816(tmp[nt], a0, qb[2 * j][nt][0], qb[2 * j][nt][1]);
          mma_f16_16816(tmp[nt], a1, qb[2 * j + 1][nt][0], qb[2 * j + 1][nt][1]);
        }
        const float s0 = half_at(sk0, j), s1 = half_at(sk1, j);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          sc[nt][0] = fmaf(s0, tmp[nt][0], sc[nt][0]);
          sc[nt][1] = fmaf(s0, tmp[nt][1], sc[nt][1]);
          sc[nt][2] = fmaf(s1, tmp[nt][2], sc[nt][2]);
          sc[nt][3] = fmaf(s1, tmp[nt][3], sc[nt][3]);
        }
      }
      // mask keys past the end, scale into the log2 domain
      const int key0 = k_begin + i * kTileKeys + warp * 16 + g;
      const bool v0 = key0 < k_end, v1 = key0 + 8 < k_end;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        sc[nt][0] = v0 ? sc[nt][0] * p.scale_log2 : -INFINITY;
        sc[nt][1] = v0 ? sc[nt][1] * p.scale_log2 : -INFINITY;
        sc[nt][2] = v1 ? sc[nt][2] * p.scale_log2 : -INFINITY;
        sc[nt][3] = v1 ? sc[nt][3] * p.scale_log2 : -INFINITY;
      }
      // online softmax per head column; P^T (fp32) to this warp's tile pt[head][key]
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          float mx = fmaxf(sc[nt][cc], sc[nt][cc + 2]);
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
          const float m_new = fmaxf(m_run[nt][cc], mx);
          const float base = m_new == -INFINITY ? 0.f : m_new;
          const float alpha = exp2f(m_run[nt][cc] - base);
          m_run[nt][cc] = m_new;
          const float p0 = exp2f(sc[nt][cc] - base), p1 = exp2f(sc[nt][cc + 2] - base);
          sc[nt][cc] = p0;
          sc[nt][cc + 2] = p1;
          l_run[nt][cc] = l_run[nt][cc] * alpha + p0 + p1;
#pragma unroll
          for (int mt = 0; mt < D / 16; ++mt) {
            o[mt][nt][cc] *= alpha;
            o[mt][nt][cc + 2] *= alpha;
          }
        }
        if (nt == 0 || p.group > 8) {
          const int hd = nt * 8 + c4 * 2;
          pt[hd * L::kPtStride + g] = sc[nt][0];
          pt[(hd + 1) * L::kPtStride + g] = sc[nt][1];
          pt[hd * L::kPtStride + g + 8] = sc[nt][2];
          pt[(hd + 1) * L::kPtStride + g + 8] = sc[nt][3];
        }
      }
      __syncwarp();
      // P^T of keys 2 c4, 2 c4 + 1, 2 c4 + 8, 2 c4 + 9 for head g of each n-tile
      float pv[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const float2 lo = *reinterpret_cast<const float2 *>(pt + (nt * 8 + g) * L::kPtStride + 2 * c4);
        const float2 hi = *reinterpret_cast<const float2 *>(pt + (nt * 8 + g) * L::kPtStride + 2 * c4 + 8);
        pv[nt][0] = 256.f * lo.x;
        pv[nt][1] = 256.f * lo.y;
        pv[nt][2] = 256.f * hi.x;
        pv[nt][3] = 256.f * hi.y;
      }
      // V scales of those four keys
      const int vk = warp * 16 + 2 * c4;
      const uint4 sv0 = *reinterpret_cast<const uint4 *>(vsc + vk * NB * 2);
      const uint4 sv1 = *reinterpret_cast<const uint4 *>(vsc + (vk + 1) * NB * 2);
      const uint4 sv2 = *reinterpret_cast<const uint4 *>(vsc + (vk + 8) * NB * 2);
      const uint4 sv3 = *reinterpret_cast<const uint4 *>(vsc + (vk + 9) * NB * 2);
      // ---- O^T += V^T P'^T, block J of 32 value columns = m-tiles 2J (columns 32J + 4g, +1) and
      // 2J + 1 (32J + 4g + 2, +3) ----
      const uint8_t *vrow = vx;  // row vk + r, 16-byte chunk ch of the 256-byte row
#pragma unroll
      for (int J = 0; J < NB; ++J) {
        const int ch = 2 * J + (g >> 2);
        const uint32_t off = (uint32_t)(ch >> 3) * L::kBoxBytes + (uint32_t)(g & 3) * 4;
        const uint32_t w0 = *reinterpret_cast<const uint32_t *>(vrow + off + sw128(vk, ch & 7));
        const uint32_t w1 = *reinterpret_cast<const uint32_t *>(vrow + off + sw128(vk + 1, ch & 7));
        const uint32_t w8 = *reinterpret_cast<const uint32_t *>(vrow + off + sw128(vk + 8, ch & 7));
        const uint32_t w9 = *reinterpret_cast<const uint32_t *>(vrow + off + sw128(vk + 9, ch & 7));
        const uint32_t t01 = prmt(w0, w1, 0x5140u), t23 = prmt(w0, w1, 0x7362u);
        const uint32_t t89 = prmt(w8, w9, 0x5140u), tab = prmt(w8, w9, 0x7362u);
        const uint32_t aA[4] = {i8x2_lo_f16(t01), i8x2_hi_f16(t01), i8x2_lo_f16(t89), i8x2_hi_f16(t89)};
        const uint32_t aB[4] = {i8x2_lo_f16(t23), i8x2_hi_f16(t23), i8x2_lo_f16(tab), i8x2_hi_f16(tab)};
        const float s0 = half_at(sv0, J), s1 = half_at(sv1, J), s2 = half_at(sv2, J), s3 = half_at(sv3, J);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const uint32_t b0 = pack_f16(s0 * pv[nt][0], s1 * pv[nt][1]);
          const uint32_t b1 = pack_f16(s2 * pv[nt][2], s3 * pv[nt][3]);
          mma_f16_16816(o[2 * J][nt], aA, b0, b1);
          mma_f16_16816(o[2 * J + 1][nt], aB, b0, b1);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    // per-warp results -> shared reduction buffer (reuses the stage ring)
    __syncwarp();
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        float l = l_run[nt][cc];
        l += __shfl_xor_sync(0xffffffffu, l, 4);
        l += __shfl_xor_sync(0xffffffffu, l, 8);
        l += __shfl_xor_sync(0xffffffffu, l, 16);
        l_run[nt][cc] = l;
      }
    asm volatile("bar.sync 1, %0;\n" ::"n"(kConsumerWarps * 32));
    float *red_o = reinterpret_cast<float *>(ring);
    float *red_m = red_o + kConsumerWarps * 16 * D;
    float *red_l = red_m + kConsumerWarps * 16;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int hd = nt * 8 + c4 * 2;
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        const int dd = (mt >> 1) * 32 + 4 * g + (mt & 1) * 2;  // rows g, g + 8 of m-tile mt
        red_o[(warp * 16 + hd) * D + dd] = o[mt][nt][0] * (1.f / 256.f);
        red_o[(warp * 16 + hd + 1) * D + dd] = o[mt][nt][1] * (1.f / 256.f);
        red_o[(warp * 16 + hd) * D + dd + 1] = o[mt][nt][2] * (1.f / 256.f);
        red_o[(warp * 16 + hd + 1) * D + dd + 1] = o[mt][nt][3] * (1.f / 256.f);
      }
      if (lane < 4) {
        red_m[warp * 16 + hd] = m_run[nt][0];
        red_m[warp * 16 + hd + 1] = m_run[nt][1];
        red_l[warp * 16 + hd] = l_run[nt][0];
        red_l[warp * 16 + hd + 1] = l_run[nt][1];
      }
    }
    asm volatile("bar.sync 1, %0;\n" ::"n"(kConsumerWarps * 32));
    for (int idx = threadIdx.x; idx < p.group * D; idx += kConsumerWarps * 32) {
      const int hd = idx / D, dd = idx % D;
      float mt = -INFINITY;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) mt = fmaxf(mt, red_m[w * 16 + hd]);
      float lt = 0.f, ot = 0.f;
      if (mt != -INFINITY) {
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
          const float f = exp2f(red_m[w * 16 + hd] - mt);
          lt += red_l[w * 16 + hd] * f;
          ot += red_o[(w * 16 + hd) * D + dd] * f;
        }
      }
      const size_t row = ((size_t)b * p.H_q + kvh * p.group + hd) * p.n_splits + split;
      p.part_o[row * D + dd] = ot;
      if (dd == 0) {
        p.part_ml[row * 2 + 0] = mt;
        p.part_ml[row * 2 + 1] = lt;
      }
    }
  }
}

template <int D, int NT>
cudaError_t launch_q8_split(const DecodeQ8Params &p, cudaStream_t s) {
  auto kern = attn_decode_q8_split_kernel<D, NT>;
  const int smem = DecodeQ8Smem<D>::kTotal;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3(p.n_splits, p.H_kv, p.B), kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

// Keys per split: 8192 for large batches; for small ones shorter splits, so that B x H_kv x splits
// still gives the 148 SMs about two CTAs each (one sequence, 4 kv heads and an 84K-token cache: 83
// splits of 1024 keys instead of 11 of 8192).  The split count depends only on (B, T_cache), so the
// workspace query (which has no H_kv) and the launch agree.
int attn_decode_splits(int B, int T_cache) {
  if (T_cache <= 0) return 1;
  int per = 8192;
  if (B < 16) per = B <= 2 ? 1024 : (B <= 4 ? 2048 : 4096);
  const int n = (T_cache + per - 1) / per;
  return n < 1 ? 1 : (n > 128 ? 128 : n);
}

size_t attn_decode_workspace(int B, int H_q, int d, int T_cache) {
  const size_t rows = (size_t)B * H_q * attn_decode_splits(B, T_cache);
  const size_t o_bytes = (rows * d * sizeof(float) + 255) & ~size_t(255);
  return o_bytes + rows * 2 * sizeof(float);
}

cudaError_t launch_attn_decode(const AttnDecodeArgs &a, cudaStream_t s) {
  if (a.B == 0) return cudaSuccess;
  DecodeSplitParams p;
  const int n_splits = attn_decode_splits(a.B, a.T_cache);
  int split_len = (a.T_cache + n_splits - 1) / n_splits;
  split_len = (split_len + kTileKeys - 1) / kTileKeys * kTileKeys;
  const size_t rows = (size_t)a.B * a.H_q * n_splits;
  p.part_o = reinterpret_cast<float *>(a.workspace);
  p.part_ml = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(a.workspace) +
                                        ((rows * a.d * sizeof(float) + 255) & ~size_t(255)));
  p.q = a.q;
  p.cache_len = a.cache_len;
  p.B = a.B;
  p.T_cache = a.T_cache;
  p.H_q = a.H_q;
  p.H_kv = a.H_kv;
  p.group = a.H_q / a.H_kv;
  p.n_splits = n_splits;
  p.split_len = split_len;
  p.scale_log2 = a.scale * kLog2e;
  p.status = device_status_ptr();
  if (a.T_cache > 0) {
    const uint64_t dims[4] = {(uint64_t)a.d, (uint64_t)a.H_kv, (uint64_t)a.T_cache, (uint64_t)a.B};
    const uint64_t strides[3] = {(uint64_t)a.d * 2, (uint64_t)a.H_kv * a.d * 2,
                                 (uint64_t)a.T_cache * a.H_kv * a.d * 2};
    const uint32_t box[4] = {64, 1, (uint32_t)kTileKeys, 1};
    if (encode_tmap(&p.tm_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.k_cache, dims, strides, box,
                    CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS ||
        encode_tmap(&p.tm_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.v_cache, dims, strides, box,
                    CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS) {
      set_error("gqa_attn_decode: cuTensorMapEncodeTiled failed for the KV cache");
      return cudaErrorInvalidValue;
    }
  } else {
    memset(&p.tm_k, 0, sizeof(p.tm_k));
    memset(&p.tm_v, 0, sizeof(p.tm_v));
  }
  cudaError_t e;
  const bool wide = p.group > 8;
  if (a.d == 256) e = wide ? launch_split<256, 2>(p, s) : launch_split<256, 1>(p, s);
  else e = wide ? launch_split<128, 2>(p, s) : launch_split<128, 1>(p, s);
  if (e != cudaSuccess) return e;
  const unsigned rows_out = (unsigned)(a.B * a.H_q);
  if (a.d == 256) attn_decode_combine_kernel<256><<<rows_out, 256, 0, s>>>(p.part_o, p.part_ml, a.gate, a.o, n_splits);
  else attn_decode_combine_kernel<128><<<rows_out, 128, 0, s>>>(p.part_o, p.part_ml, a.gate, a.o, n_splits);
  return cudaGetLastError();
}

// The q8_0 cache: the split kernel above, then the same log-sum-exp combine.
cudaError_t launch_attn_decode_q8(const AttnDecodeQ8Args &a, cudaStream_t s) {
  if (a.B == 0) return cudaSuccess;
  if (a.d != 256) {
    set_error("gqa_attn_decode_q8_0: only d = 256 is built");
    return cudaErrorInvalidValue;
  }
  DecodeQ8Params p;
  const int n_splits = attn_decode_splits(a.B, a.T_cache);
  int split_len = (a.T_cache + n_splits - 1) / n_splits;
  split_len = (split_len + kTileKeys - 1) / kTileKeys * kTileKeys;
  const size_t rows = (size_t)a.B * a.H_q * n_splits;
  p.part_o = reinterpret_cast<float *>(a.workspace);
  p.part_ml = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(a.workspace) +
                                        ((rows * a.d * sizeof(float) + 255) & ~size_t(255)));
  p.q = a.q;
  p.cache_len = a.cache_len;
  p.B = a.B;
  p.T_cache = a.T_cache;
  p.H_q = a.H_q;
  p.H_kv = a.H_kv;
  p.group = a.H_q / a.H_kv;
  p.n_splits = n_splits;
  p.split_len = split_len;
  p.scale_log2 = a.scale * kLog2e;
  p.status = device_status_ptr();
  if (a.T_cache > 0) {
    const uint64_t dx[4] = {(uint64_t)a.d, (uint64_t)a.H_kv, (uint64_t)a.T_cache, (uint64_t)a.B};
    const uint64_t sx[3] = {(uint64_t)a.d, (uint64_t)a.H_kv * a.d, (uint64_t)a.T_cache * a.H_kv * a.d};
    const uint32_t bx[4] = {128, 1, (uint32_t)kTileKeys, 1};
    const uint64_t ds[4] = {(uint64_t)a.d / 32, (uint64_t)a.H_kv, (uint64_t)a.T_cache, (uint64_t)a.B};
    const uint64_t ss[3] = {(uint64_t)a.d / 32 * 2, (uint64_t)a.H_kv * a.d / 32 * 2,
                            (uint64_t)a.T_cache * a.H_kv * a.d / 32 * 2};
    const uint32_t bs[4] = {(uint32_t)a.d / 32, 1, (uint32_t)kTileKeys, 1};
    if (encode_tmap(&p.tm_kx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, a.k_values, dx, sx, bx, CU_TENSOR_MAP_SWIZZLE_128B) ||
        encode_tmap(&p.tm_vx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, a.v_values, dx, sx, bx, CU_TENSOR_MAP_SWIZZLE_128B) ||
        encode_tmap(&p.tm_ks, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, a.k_scales, ds, ss, bs, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        encode_tmap(&p.tm_vs, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, a.v_scales, ds, ss, bs, CU_TENSOR_MAP_SWIZZLE_NONE)) {
      set_error("gqa_attn_decode_q8_0: cuTensorMapEncodeTiled failed for the q8_0 cache");
      return cudaErrorInvalidValue;
    }
  } else {
    memset(&p.tm_kx, 0, sizeof(p.tm_kx));
    memset(&p.tm_vx, 0, sizeof(p.tm_vx));
    memset(&p.tm_ks, 0, sizeof(p.tm_ks));
    memset(&p.tm_vs, 0, sizeof(p.tm_vs));
  }
  cudaError_t e = p.group > 8 ? launch_q8_split<256, 2>(p, s) : launch_q8_split<256, 1>(p, s);
  if (e != cudaSuccess) return e;
  attn_decode_combine_kernel<256><<<(unsigned)(a.B * a.H_q), 256, 0, s>>>(p.part_o, p.part_ml, a.gate, a.o, n_splits);
  return cudaGetLastError();
}

}  // namespace hh
