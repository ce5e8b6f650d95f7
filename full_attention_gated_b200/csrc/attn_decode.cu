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

}  // namespace

int attn_decode_splits(int T_cache) {
  if (T_cache <= 0) return 1;
  const int per = 8192;
  int n = (T_cache + per - 1) / per;
  return n < 1 ? 1 : (n > 64 ? 64 : n);
}

size_t attn_decode_workspace(int B, int H_q, int d, int T_cache) {
  const size_t rows = (size_t)B * H_q * attn_decode_splits(T_cache);
  const size_t o_bytes = (rows * d * sizeof(float) + 255) & ~size_t(255);
  return o_bytes + rows * 2 * sizeof(float);
}

cudaError_t launch_attn_decode(const AttnDecodeArgs &a, cudaStream_t s) {
  if (a.B == 0) return cudaSuccess;
  DecodeSplitParams p;
  const int n_splits = attn_decode_splits(a.T_cache);
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

}  // namespace hh
