// phba.cu -- PHBA ("PHBA: Prefix-State Hybrid Block Attention", abstract and Figure 1): top-K
// block routing with block-aligned prefix states and one softmax over tokens and state slots,
// per sequence and head, at d = 128 with M = 128 memory slots and blocks of C in {64, 128, 256}.
//
// The page names the parts and prints no formula.  What is computed (the C ABI states the same):
//   prefix states  Kt_{t+1}[m] = a_{t,m} Kt_t[m] + (1 - a_{t,m}) kraw_t, Vt likewise with v_t, from
//                  zero; entry j is the memory after the j C tokens before block j;
//   routing        query t keeps the min(K, t / C) earlier blocks j of highest
//                  qrope_t . mean_{s in block j} krope_s (a tie goes to the lower j);
//   attention      one softmax (scale 1 / sqrt(d)) over all tokens of the kept blocks, the own
//                  block's tokens s <= t (logits qrope . krope, values v) and the M slots of the
//                  prefix states of the kept blocks and of the own block, block 0's (empty)
//                  excluded (logits qraw . Kt, values Vt).
//
// Kernels:
//   phba_slots_local    per (block, head, sequence): the block's contribution to the memory from
//                       zero, L_j = W_j^T [K_j | V_j] with W_j[s][m] = (1 - a_s,m) prod_{s<r<C} a_r,m,
//                       on the 5th-generation tensor cores (W as two bf16 terms, fp32 accumulation
//                       in tensor memory), and the block's decay D_j[m] = prod_s a_s,m;
//   phba_slots_combine  entry j + 1 = D_j entry j + L_j, sequential over blocks in fp32, stored bf16;
//   phba_block_means    the mean rotated key of every complete block (fp32);
//   phba_route          per 128 queries: scores against the block means (fp32), the top K of every
//                       query kept in registers by its own thread, and the size of every (head,
//                       block) bucket (shared-memory counters, one global add per block);
//   phba_bucket_scan    offsets of the buckets and of their 128-row tiles;
//   phba_bucket_fill    every query into its own block's bucket (causal rows first) and into the
//                       bucket of each block it kept;
//   phba_attn_tiles     per tile of up to 128 gathered queries of one bucket, tcgen05, two tiles per
//                       SM: the block's keys in segments of min(C, 128) tokens, then its memory slots,
//                       S = Qrope K_s^T (Qraw Kt_j^T for the slots) in tensor memory, an online softmax
//                       across the segments (two warps per row quarter) with P written back as bf16,
//                       O += P_s V_s; each row's partial output (normalised, bf16) and log-sum-exp go to
//                       the workspace;
//   phba_merge          per query: its partials combined by their log-sum-exps.
// Every partial covers disjoint entries of the query's softmax, so the merge is exact up to
// rounding: o = sum_k 2^{lse_k} o_k / sum_k 2^{lse_k}.
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace hh {

namespace {

constexpr int kD = 128;         // head dim
constexpr int kM = 128;         // memory slots
constexpr int kRows = 128;      // queries per attention tile
constexpr int kSubTok = 64;     // tokens per sub-chunk of the slot kernel
constexpr int kMaxCand = 512;   // most complete blocks a query may score
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// ============================================================================
// phba_slots_local: one CTA per (block j < nb - 1, head, sequence), 256 threads.
// Sub-chunks of 64 tokens run from the block's end to its start, so that thread m
// (warps 0-3) carries the suffix product of its slot's gates: W[s][m] = (1 - a_s) P_s with
// P_s = prod_{r > s} a_r.  W^T (slots as M, tokens as K) is written as two bf16 terms
// (W_hi + W_lo) into 128-byte-swizzled K-major tiles; K_j and V_j sub-tiles arrive by TMA
// (tokens as K, d contiguous: MN-major B operands).  Warp 4 issues, with one elected lane,
//   Kt_local += W_hi^T K + W_lo^T K   (tensor memory columns 0..127)
//   Vt_local += W_hi^T V + W_lo^T V   (columns 128..255)
// Two buffers: the gates of sub-chunk i + 1 are formed while the MMAs of sub-chunk i run.
// ============================================================================
struct SlotParams {
  CUtensorMap tm_k, tm_v;  // 4-D (d, H, T, B), box (64, 1, 64, 1)
  const float *alpha;      // [B, T, H, M]
  float *L;                // [B, H, nb, 2, M, d]
  float *D;                // [B, H, nb, M]
  int B, T, H, C, nb;
  unsigned *status;
};

struct SlotSmem {
  // per buffer: W_hi^T, W_lo^T [128][64] bf16 (16 KB each), K, V [64 tok][128 d] as two 64-d boxes
  static constexpr int kBuf = 4 * 16384;
  static constexpr int oWhi = 0, oWlo = 16384, oK = 32768, oV = 49152;
  static constexpr int oBar = 2 * kBuf;  // full[2], mdone[2], fin
  static constexpr int kTotal = oBar + 64 + 16;
};

__global__ void __launch_bounds__(256, 1) phba_slots_local_kernel(const __grid_constant__ SlotParams p) {
  using L = SlotSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  uint64_t *full = reinterpret_cast<uint64_t *>(sm + L::oBar);
  uint64_t *mdone = full + 2;
  uint64_t *fin = full + 4;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(full + 5);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int nsub = p.C / kSubTok;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 5; ++i) mbar_init(&full[i], 1);
    fence_barrier_init();
  }
  if (warp == 4) {
    tc::tmem_alloc(smem_u32(tmem_slot), 256);
    tc::tmem_relinquish();
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tbase = *tmem_slot;

  float P = 1.f;  // thread m < 128: the product of the gates after the current token
  bool ok = true;
  int issued = 0;  // TMA batches issued (thread 128)
  // thread m < 128: the gates of its slot over the current sub-chunk; the next sub-chunk's are loaded
  // into the same registers as soon as these are used, so that their latency overlaps the rest
  float a[kSubTok];
  const size_t ast = (size_t)p.H * kM;  // gate stride between tokens
  auto load_gates = [&](int u) {
    const float *ap = p.alpha + (((size_t)b * p.T + (size_t)j * p.C + u * kSubTok) * p.H + h) * kM + threadIdx.x;
#pragma unroll
    for (int s = 0; s < kSubTok; ++s) a[s] = ap[s * ast];
  };
  if (threadIdx.x < 128) load_gates(nsub - 1);
  for (int i = 0; i < nsub; ++i) {
    const int u = nsub - 1 - i, buf = i & 1;
    const uint32_t sbuf = sb + buf * L::kBuf;
    uint8_t *mbuf = sm + buf * L::kBuf;
    // the buffer was last read by the MMAs of sub-chunk i - 2
    if (i >= 2 && (threadIdx.x < 128 || threadIdx.x == 128)) ok = mbar_wait(&mdone[buf], ((i - 2) >> 1) & 1, p.status) && ok;
    if (threadIdx.x == 128 && ok) {
      const int t0 = j * p.C + u * kSubTok;
      mbar_arrive_expect_tx(&full[buf], 4 * 8192);
      tma_load_4d(sbuf + L::oK, &p.tm_k, &full[buf], 0, h, t0, b);
      tma_load_4d(sbuf + L::oK + 8192, &p.tm_k, &full[buf], 64, h, t0, b);
      tma_load_4d(sbuf + L::oV, &p.tm_v, &full[buf], 0, h, t0, b);
      tma_load_4d(sbuf + L::oV + 8192, &p.tm_v, &full[buf], 64, h, t0, b);
      ++issued;
    }
    if (threadIdx.x < 128) {
      const int m = threadIdx.x;
      uint32_t hi[kSubTok / 2], lo[kSubTok / 2];
#pragma unroll
      for (int s = kSubTok - 1; s >= 0; s -= 2) {  // tokens s - 1, s of the pair (s - 1) / 2
        const float w1 = (1.f - a[s]) * P;
        P *= a[s];
        const float w0 = (1.f - a[s - 1]) * P;
        P *= a[s - 1];
        const uint32_t h2 = pack_bf16(w0, w1);
        hi[s >> 1] = h2;
        lo[s >> 1] = pack_bf16(w0 - bf16_lo(h2), w1 - bf16_hi(h2));
      }
      if (u > 0) load_gates(u - 1);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint32_t off = (uint32_t)m * 128u + ((uint32_t)(c ^ (m & 7)) << 4);
        *reinterpret_cast<uint4 *>(mbuf + L::oWhi + off) = make_uint4(hi[4 * c], hi[4 * c + 1], hi[4 * c + 2], hi[4 * c + 3]);
        *reinterpret_cast<uint4 *>(mbuf + L::oWlo + off) = make_uint4(lo[4 * c], lo[4 * c + 1], lo[4 * c + 2], lo[4 * c + 3]);
      }
    }
    tc::fence_proxy_async_smem();
    ok = __syncthreads_and(ok) != 0;
    if (warp == 4 && ok) {
      ok = __all_sync(0xffffffffu, mbar_wait(&full[buf], (i >> 1) & 1, p.status));
      if (ok) {
        tc::fence_after();
        const uint64_t dWh = tc::desc_kmajor_sw128(sbuf + L::oWhi), dWl = tc::desc_kmajor_sw128(sbuf + L::oWlo);
        const uint64_t dK = tc::desc_mnmajor_sw128(sbuf + L::oK, 8192, 1024);
        const uint64_t dV = tc::desc_mnmajor_sw128(sbuf + L::oV, 8192, 1024);
        constexpr uint32_t id = tc::idesc_bf16_f32(128, 128, 0, 1);
#pragma unroll
        for (int kk = 0; kk < kSubTok / 16; ++kk) {
          const uint32_t acc = (i | kk) ? 1u : 0u;
          tc::mma_ss_w(tbase, dWh + kk * 2, dK + kk * 128, id, acc);
          tc::mma_ss_w(tbase, dWl + kk * 2, dK + kk * 128, id, 1u);
          tc::mma_ss_w(tbase + 128, dWh + kk * 2, dV + kk * 128, id, acc);
          tc::mma_ss_w(tbase + 128, dWl + kk * 2, dV + kk * 128, id, 1u);
        }
        tc::commit_w(&mdone[buf]);
      }
    }
    ok = __syncthreads_and(ok) != 0;
  }
  // every MMA issued above completes before tensor memory is read or released
  if (warp == 4) {
    tc::commit_w(fin);
    ok = __all_sync(0xffffffffu, mbar_wait(fin, 0, p.status)) && ok;
  }
  // every TMA batch issued has landed before the CTA exits (on the normal path the MMAs waited on them)
  if (threadIdx.x == 128)
    for (int i = (issued > 2 ? issued - 2 : 0); i < issued; ++i) mbar_wait(&full[i & 1], (i >> 1) & 1, p.status);
  ok = __syncthreads_and(ok) != 0;
  tc::fence_after();
  const size_t e0 = ((size_t)b * p.H + h) * p.nb + j;
  if (ok) {
    // warp w: lane quarter w % 4 (slots), memory w / 4 (0: Kt, 1: Vt)
    const int q4 = warp & 3, which = warp >> 2, m = q4 * 32 + lane;
    float *dst = p.L + (e0 * 2 + which) * (size_t)kM * kD + (size_t)m * kD;
#pragma unroll 1
    for (int c = 0; c < kD / 32; ++c) {
      uint32_t r[32];
      tc::ld32(tbase + ((uint32_t)(q4 * 32) << 16) + which * 128 + c * 32, r);
      tc::wait_ld();
      tc::regfence(r);
#pragma unroll
      for (int e = 0; e < 32; e += 4)
        *reinterpret_cast<float4 *>(dst + c * 32 + e) =
            make_float4(__uint_as_float(r[e]), __uint_as_float(r[e + 1]), __uint_as_float(r[e + 2]), __uint_as_float(r[e + 3]));
    }
    if (threadIdx.x < 128) p.D[e0 * kM + threadIdx.x] = P;
  }
  tc::fence_before();
  __syncthreads();
  if (warp == 4) {
    tc::fence_after();
    tc::tmem_dealloc(tbase, 256);
  }
}

// entry 0 = 0; entry j + 1 = D_j entry j + L_j (fp32), every entry stored as bf16.
// One thread per (sequence, head, slot, four dims).
__global__ void phba_slots_combine_kernel(const float *__restrict__ L, const float *__restrict__ D,
                                          bf16_t *__restrict__ kst, bf16_t *__restrict__ vst, int B, int H, int nb) {
  const size_t n = (size_t)B * H * kM * (kD / 4);
  for (size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x; idx < n; idx += (size_t)gridDim.x * blockDim.x) {
    const int i4 = (int)(idx % (kD / 4)), m = (int)((idx / (kD / 4)) % kM);
    const size_t bh = idx / ((size_t)(kD / 4) * kM);
    float4 pk = make_float4(0.f, 0.f, 0.f, 0.f), pv = pk;
#pragma unroll 4
    for (int j = 0; j < nb; ++j) {
      const size_t e = bh * nb + j;
      const size_t o = (e * kM + m) * kD + 4 * i4;
      *reinterpret_cast<uint2 *>(kst + o) = make_uint2(pack_bf16(pk.x, pk.y), pack_bf16(pk.z, pk.w));
      *reinterpret_cast<uint2 *>(vst + o) = make_uint2(pack_bf16(pv.x, pv.y), pack_bf16(pv.z, pv.w));
      if (j + 1 < nb) {
        const float dj = D[e * kM + m];
        const float4 lk = *reinterpret_cast<const float4 *>(L + ((e * 2) * kM + m) * kD + 4 * i4);
        const float4 lv = *reinterpret_cast<const float4 *>(L + ((e * 2 + 1) * kM + m) * kD + 4 * i4);
        pk = make_float4(fmaf(dj, pk.x, lk.x), fmaf(dj, pk.y, lk.y), fmaf(dj, pk.z, lk.z), fmaf(dj, pk.w, lk.w));
        pv = make_float4(fmaf(dj, pv.x, lv.x), fmaf(dj, pv.y, lv.y), fmaf(dj, pv.z, lv.z), fmaf(dj, pv.w, lv.w));
      }
    }
  }
}

// ============================================================================
// Routing
// ============================================================================
// mean rotated key of complete block j: one CTA per (block, head, sequence), 256 threads.  Warp w sums
// the tokens s = w (mod 8) (lane: four dims, 8-byte loads, C / 8 of them in flight at once), in token
// order; the eight partial sums are then added in warp order.
__global__ void __launch_bounds__(256) phba_block_means_kernel(const bf16_t *__restrict__ krope,
                                                               float *__restrict__ kbar, int T, int H, int C, int nfull) {
  __shared__ float4 part[8][32];
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bf16_t *src = krope + (((size_t)b * T + (size_t)j * C) * H + h) * kD + 4 * lane;
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
  for (int s0 = warp; s0 < C; s0 += 8 * 8) {
    uint2 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = *reinterpret_cast<const uint2 *>(src + (size_t)(s0 + 8 * u) * H * kD);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      a0 += bf16_lo(v[u].x);
      a1 += bf16_hi(v[u].x);
      a2 += bf16_lo(v[u].y);
      a3 += bf16_hi(v[u].y);
    }
  }
  part[warp][lane] = make_float4(a0, a1, a2, a3);
  __syncthreads();
  if (threadIdx.x < 32) {
    float4 t = part[0][lane];
    for (int w = 1; w < 8; ++w) {
      t.x += part[w][lane].x;
      t.y += part[w][lane].y;
      t.z += part[w][lane].z;
      t.w += part[w][lane].w;
    }
    const float inv = 1.f / (float)C;
    *reinterpret_cast<float4 *>(kbar + (((size_t)b * H + h) * nfull + j) * kD + 4 * lane) =
        make_float4(t.x * inv, t.y * inv, t.z * inv, t.w * inv);
  }
}

struct RouteParams {
  const bf16_t *qrope;
  const float *kbar;   // [B, H, nfull, d]
  int32_t *sel;        // [B, T, H, K]
  int32_t *rank;       // [B, T, H, K]: position of the query in the kept block's bucket
  int32_t *cnt;        // [B, H, nb]: queries that kept the block (zeroed by the host)
  int B, T, H, C, K, nb, nfull;
};

// 128 queries per CTA, 256 threads.  Scores: for every chunk of 32 candidate blocks, thread (r8, c8)
// forms the 4 x 4 (query, block) dot products of queries 4 r8 .. and blocks 4 c8 .. over d in order,
// from a transposed query tile and a transposed tile of the chunk's block means.  Selection: thread
// r < 128 then scans its query's scores of the chunk in ascending block order and keeps the K best so
// far in registers, sorted by score (an equal score never displaces an earlier block, so a tie goes to
// the lower block).
constexpr int kRq = 128;   // queries per routing CTA
constexpr int kRc = 32;    // candidate blocks per score chunk
template <int KMAX>  // the kept list's register capacity: K <= KMAX
__global__ void __launch_bounds__(256) phba_route_kernel(const __grid_constant__ RouteParams p) {
  extern __shared__ float rs[];
  float *qs = rs;                                            // [d][kRq + 4] queries
  float *ks = qs + kD * (kRq + 4);                           // [d][kRc + 4] block means of the chunk
  int *kept_s = reinterpret_cast<int *>(ks + kD * (kRc + 4));  // [kRq][16] kept blocks, ascending
  int *lrank = kept_s + kRq * 16;                            // [kRq][16] rank among this CTA's queries
  int *cnt_s = lrank + kRq * 16;                             // [kMaxCand] queries of this CTA per block
  int *base_s = cnt_s + kMaxCand;                            // [kMaxCand] first rank of this CTA per block
  float *sc = ks;  // [kRq][kRc + 1] scores of the chunk, over the block means once they are used
  const int t0 = blockIdx.x * kRq, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  const int t_last = min(p.T - 1, t0 + kRq - 1);
  const int ncand = min(p.nfull, t_last / p.C);  // candidate blocks of the CTA's last query
  const int ncs = ((ncand + kRc - 1) / kRc) * kRc;
  constexpr int ldc = kRc + 1;
  const bool sel_thread = tid < kRq && t0 + tid < p.T;
  const int nt = sel_thread ? (t0 + tid) / p.C : 0;  // candidates of query tid: blocks 0 .. nt - 1
  const int nkeep = min(p.K, nt);
  // the K best so far, sorted by score; bj = INT_MAX marks an empty entry
  float bv[KMAX];
  int bj[KMAX];
#pragma unroll
  for (int k = 0; k < KMAX; ++k) {
    bv[k] = -INFINITY;
    bj[k] = 0x7fffffff;
  }
  int filled = 0;
  float kth = -INFINITY;  // score of the K-th entry once K are filled
  {  // the query tile: 16-byte loads from rows clamped into range, all issued before any is used
    // lanes take consecutive rows of one 16-byte column chunk, so the transposed stores are conflict-free
    uint4 qv[kRq * kD / 8 / 256];
#pragma unroll
    for (int u = 0; u < kRq * kD / 8 / 256; ++u) {
      const int e = tid + u * 256, r = e & (kRq - 1), c = e / kRq;
      qv[u] = *reinterpret_cast<const uint4 *>(p.qrope + (((size_t)b * p.T + min(t0 + r, p.T - 1)) * p.H + h) * kD + c * 8);
    }
#pragma unroll
    for (int u = 0; u < kRq * kD / 8 / 256; ++u) {
      const int e = tid + u * 256, r = e & (kRq - 1), c = e / kRq;
      const bool in = t0 + r < p.T;
      const uint32_t w4[4] = {qv[u].x, qv[u].y, qv[u].z, qv[u].w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        qs[(c * 8 + 2 * k) * (kRq + 4) + r] = in ? bf16_lo(w4[k]) : 0.f;
        qs[(c * 8 + 2 * k + 1) * (kRq + 4) + r] = in ? bf16_hi(w4[k]) : 0.f;
      }
    }
  }
  for (int e = tid; e < kMaxCand; e += 256) cnt_s[e] = 0;
  const int r8 = tid >> 3, c8 = tid & 7;
  for (int jc = 0; jc < ncs; jc += kRc) {
    __syncthreads();  // qs complete; ks free
    {
      float4 kv4[kRc * kD / 4 / 256];
#pragma unroll
      for (int u = 0; u < kRc * kD / 4 / 256; ++u) {
        const int e = tid + u * 256, jj = e & (kRc - 1), c = e / kRc;
        kv4[u] = *reinterpret_cast<const float4 *>(p.kbar + (((size_t)b * p.H + h) * p.nfull + min(jc + jj, ncand - 1)) * kD + 4 * c);
      }
#pragma unroll
      for (int u = 0; u < kRc * kD / 4 / 256; ++u) {
        const int e = tid + u * 256, jj = e & (kRc - 1), c = e / kRc;
        const bool in = jc + jj < ncand;
        ks[(4 * c) * (kRc + 4) + jj] = in ? kv4[u].x : 0.f;
        ks[(4 * c + 1) * (kRc + 4) + jj] = in ? kv4[u].y : 0.f;
        ks[(4 * c + 2) * (kRc + 4) + jj] = in ? kv4[u].z : 0.f;
        ks[(4 * c + 3) * (kRc + 4) + jj] = in ? kv4[u].w : 0.f;
      }
    }
    __syncthreads();
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;
#pragma unroll 8
    for (int i = 0; i < kD; ++i) {
      const float4 qv = *reinterpret_cast<const float4 *>(qs + i * (kRq + 4) + r8 * 4);
      const float4 kv = *reinterpret_cast<const float4 *>(ks + i * (kRc + 4) + c8 * 4);
      const float qa[4] = {qv.x, qv.y, qv.z, qv.w}, ka[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[a][c] = fmaf(qa[a], ka[c], acc[a][c]);
    }
    __syncthreads();  // every thread has read the block means: the scores go over them
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) sc[(r8 * 4 + a) * ldc + c8 * 4 + c] = acc[a][c];
    __syncthreads();
    const float *row = sc + tid * ldc;
    const int jend = min(nt, jc + kRc);
    for (int jb = jc; jb < jend; ++jb) {
      const float v = row[jb - jc];
      if (filled < nkeep || v > kth) {
        // insert v after every entry of score >= v, then shift the rest down by one (the list stays
        // sorted by score, earlier blocks first among equal scores; the last entry falls off)
        float cv = v;
        int cj = jb;
        bool ins = false;
#pragma unroll
        for (int k = 0; k < KMAX; ++k) {
          if (k < nkeep && (ins || bj[k] == 0x7fffffff || cv > bv[k])) {
            const float tv = bv[k];
            const int tj = bj[k];
            bv[k] = cv;
            bj[k] = cj;
            cv = tv;
            cj = tj;
            ins = true;
          }
        }
        filled = min(filled + 1, nkeep);
#pragma unroll
        for (int k = 0; k < KMAX; ++k)
          if (k == nkeep - 1) kth = bv[k];
      }
    }
  }
  __syncthreads();
  if (sel_thread) {
    const int r = tid;
    // ascending block order (empty entries, INT_MAX, go last)
#pragma unroll
    for (int a = 0; a < KMAX - 1; ++a)
#pragma unroll
      for (int c = 0; c < KMAX - 1 - a; ++c)
        if (bj[c] > bj[c + 1]) {
          const int tj = bj[c];
          bj[c] = bj[c + 1];
          bj[c + 1] = tj;
        }
#pragma unroll
    for (int k = 0; k < 16; ++k) kept_s[r * 16 + k] = -1;
#pragma unroll
    for (int k = 0; k < KMAX; ++k)
      if (k < nkeep) kept_s[r * 16 + k] = bj[k];
  }
  __syncthreads();
  // ranks: first among this CTA's queries (shared-memory counters), then one global add per block
  for (int e = tid; e < kRq * 16; e += 256) {
    const int r = e >> 4, k = e & 15;
    if (k < p.K && t0 + r < p.T) {
      const int jb = kept_s[r * 16 + k];
      if (jb >= 0) lrank[e] = atomicAdd(&cnt_s[jb], 1);
    }
  }
  __syncthreads();
  for (int jb = tid; jb < ncand; jb += 256)
    if (cnt_s[jb] > 0) base_s[jb] = atomicAdd(&p.cnt[((size_t)b * p.H + h) * p.nb + jb], cnt_s[jb]);
  __syncthreads();
  for (int e = tid; e < kRq * 16; e += 256) {
    const int r = e >> 4, k = e & 15;
    if (k < p.K && t0 + r < p.T) {
      const int jb = kept_s[r * 16 + k];
      const size_t o = (((size_t)b * p.T + t0 + r) * p.H + h) * p.K + k;
      p.sel[o] = jb;
      p.rank[o] = jb >= 0 ? base_s[jb] + lrank[e] : 0;
    }
  }
}

// Bucket (b, h, j): own-block queries jC .. jC + own_j - 1 first, then the queries that kept j.
// off[bk] / toff[bk]: exclusive prefix sums of bucket sizes and of their 128-row tiles (one CTA).
__global__ void __launch_bounds__(1024) phba_bucket_scan_kernel(const int32_t *__restrict__ cnt, int32_t *__restrict__ off,
                                                                int32_t *__restrict__ toff, int4 *__restrict__ tiles,
                                                                int NB, int nb, int T, int C) {
  __shared__ int ws[2][32];
  const int tid = threadIdx.x, per = (NB + 1023) / 1024;
  const int lo = min(NB, tid * per), hi = min(NB, lo + per);
  auto size_of = [&](int bk) {
    const int j = bk % nb;
    return min(C, T - j * C) + cnt[bk];
  };
  int sn = 0, st = 0;
  for (int bk = lo; bk < hi; ++bk) {
    const int n = size_of(bk);
    sn += n;
    st += (n + kRows - 1) / kRows;
  }
  // block-wide exclusive scan of (sn, st)
  int in = sn, it = st;
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, in, o), c = __shfl_up_sync(0xffffffffu, it, o);
    if ((tid & 31) >= o) {
      in += a;
      it += c;
    }
  }
  if ((tid & 31) == 31) {
    ws[0][tid >> 5] = in;
    ws[1][tid >> 5] = it;
  }
  __syncthreads();
  if (tid < 32) {
    int a = ws[0][tid], c = ws[1][tid];
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, a, o), y = __shfl_up_sync(0xffffffffu, c, o);
      if (tid >= o) {
        a += x;
        c += y;
      }
    }
    ws[0][tid] = a;
    ws[1][tid] = c;
  }
  __syncthreads();
  int bn = in - sn + ((tid >> 5) ? ws[0][(tid >> 5) - 1] : 0);
  int bt = it - st + ((tid >> 5) ? ws[1][(tid >> 5) - 1] : 0);
  for (int bk = lo; bk < hi; ++bk) {
    off[bk] = bn;
    toff[bk] = bt;
    const int n = size_of(bk);
    for (int r0 = 0; r0 < n; r0 += kRows) tiles[bt + r0 / kRows] = make_int4(bk, bn + r0, min(kRows, n - r0), 0);
    bn += n;
    bt += (n + kRows - 1) / kRows;
  }
  if (tid == 1023) {
    off[NB] = bn;
    toff[NB] = bt;
  }
}

// list entries are t * 32 + slot: slot K for the own block (causal), k for the k-th kept block
__global__ void phba_bucket_fill_kernel(const int32_t *__restrict__ sel, const int32_t *__restrict__ rank,
                                        const int32_t *__restrict__ off, int32_t *__restrict__ list, int B, int T, int H,
                                        int C, int K, int nb) {
  const size_t n = (size_t)B * T * H;
  for (size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x; idx < n; idx += (size_t)gridDim.x * blockDim.x) {
    const int h = (int)(idx % H), t = (int)((idx / H) % T), b = (int)(idx / ((size_t)H * T));
    const size_t bh = (size_t)b * H + h;
    const int nt = t / C;
    list[off[bh * nb + nt] + (t - nt * C)] = t * 32 + K;
    for (int k = 0; k < K; ++k) {
      const int j = sel[idx * K + k];
      if (j < 0) continue;
      list[off[bh * nb + j] + min(C, T - j * C) + rank[idx * K + k]] = t * 32 + k;
    }
  }
}

// ============================================================================
// phba_attn_tiles: one CTA per tile of up to 128 rows of one (sequence, head, block) bucket, two
// CTAs per SM (256 tensor-memory columns and about 100 KB of shared memory each), so that one
// tile's loads and handoffs overlap the other's softmax.  The keys of the tile's block are taken
// in segments of W = min(C, 128) tokens, then the block's 128 memory slots (j >= 1), with one
// online softmax across the segments:
//   S_s  = Q K_s^T   (M = 128, N = W, K = 128) into columns 0..127, Q the rotated queries for the
//                    token segments and the raw queries for the slots
//   softmax warps: running row maximum m (the two warps of a row quarter exchange their halves'
//                  maxima), O and the partial row sums rescaled by 2^{m_old - m_new} when m moves,
//                  P = 2^{s - m} written as bf16 pairs over S
//   O   += P_s V_s   (M = 128, N = 128, K = W) into columns 128..255
// Warp 0 issues the MMAs (one elected lane) and the TMA loads of the K and V tiles through two
// slots (slot A: the K tiles, slot B: the V tiles, each refilled once the MMA that read it is
// done); warps 1-3 gather the queries (cp.async, 128-byte swizzle), the raw ones once the last
// token segment's S has read the rotated ones; warps 4-11 run the softmax and the epilogue: each
// row's output O / l (bf16) and log-sum-exp (log2 domain) go to the workspace as its partial.
// ============================================================================
struct AttnParams {
  CUtensorMap tm_kt, tm_vt;  // 4-D (d, H, T, B), box (64, 1, W, 1)
  CUtensorMap tm_ks, tm_vs;  // 2-D (d, B H nb M), box (64, 128)
  const bf16_t *qrope, *qraw;
  const int32_t *list, *toff;
  const int4 *tiles;  // per tile: bucket, first list entry, rows
  bf16_t *po;    // [B, T, H, K + 1, d]
  float *plse;   // [B, T, H, K + 1]
  int B, T, H, C, K, nb, NB;
  float cs;      // scale * log2(e)
  unsigned *status;
};

struct AttnSmem {
  static constexpr int oQ = 0;          // [128 rows] x 2 boxes of 64 d: the rotated queries, later the raw ones
  static constexpr int oA = 32768;      // slot A: a K tile (W or 128 rows x 2 boxes)
  static constexpr int oB = 65536;      // slot B: a V tile (same shape)
  static constexpr int oMeta = 98304;   // row t [128], row slot [128]
  static constexpr int oX = oMeta + 1024;  // row maxima and sums of the two column halves [2][128] each
  static constexpr int oBar = oX + 2048;   // kfull, kfree, vfull, sdone, pfull, odone, qfree, qraw, fin; TMEM slot
  static constexpr int kTotal = oBar + 9 * 8 + 8;
  static constexpr uint32_t kSCol = 0, kOCol = 128, kTmemCols = 256;
};
static_assert(2 * (AttnSmem::kTotal + 1024 + 1024) <= 233472, "two CTAs per SM");

constexpr int kAttnThreads = 384;  // warp 0: loads and MMAs; warps 1-3: query gather; warps 4-11: softmax

// the two softmax warps of a row quarter (64 threads) meet on named barrier 1 + q4 and AND their
// predicates (the barrier number is a constant, so the kernel reserves five barriers, not sixteen,
// and two CTAs fit on an SM)
template <int ID>
__device__ __forceinline__ bool pair_and_id(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, %2, 64, p;\n"
      " selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)pred), "n"(ID)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ bool pair_and(int q4, bool pred) {
  switch (q4) {
    case 0: return pair_and_id<1>(pred);
    case 1: return pair_and_id<2>(pred);
    case 2: return pair_and_id<3>(pred);
    default: return pair_and_id<4>(pred);
  }
}

__global__ void __launch_bounds__(kAttnThreads, 2) phba_attn_tiles_kernel(const __grid_constant__ AttnParams p) {
  using L = AttnSmem;
  const int tile = blockIdx.x;
  // both loads at once: the descriptor array is allocated for the launch's tile bound, so entry
  // `tile` is in bounds even where it is not a tile of this call
  const int n_tiles = p.toff[p.NB];
  const int4 td = p.tiles[tile];
  if (tile >= n_tiles) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  int32_t *row_t = reinterpret_cast<int32_t *>(sm + L::oMeta);
  int32_t *row_slot = row_t + kRows;
  uint64_t *kfull = reinterpret_cast<uint64_t *>(sm + L::oBar);
  uint64_t *kfree = kfull + 1, *vfull = kfull + 2, *sdone = kfull + 3, *pfull = kfull + 4, *odone = kfull + 5,
           *qfree = kfull + 6, *qraw = kfull + 7, *fin = kfull + 8;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(kfull + 9);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int bk = td.x, first = td.y, n_rows = td.z;
  const int j = bk % p.nb, bh = bk / p.nb, h = bh % p.H, b = bh / p.H;
  const bool slots = j >= 1;
  const int C = p.C, W = min(C, 128), n_tok = C / W, n_seg = n_tok + (slots ? 1 : 0);
  const uint32_t tok_bytes = (uint32_t)W * 256u;  // one token segment's K (or V) tile
  const size_t srow = (((size_t)b * p.H + h) * p.nb + j) * kM;  // first memory row of (b, h, j)
  // the K (V) tile of segment s into slot A (B), completing on kfull (vfull)
  auto load_k = [&](int s) {
    if (s < n_tok) {
      mbar_arrive_expect_tx(kfull, tok_bytes);
      tma_load_4d(sb + L::oA, &p.tm_kt, kfull, 0, h, j * C + s * W, b);
      tma_load_4d(sb + L::oA + W * 128, &p.tm_kt, kfull, 64, h, j * C + s * W, b);
    } else {
      mbar_arrive_expect_tx(kfull, 32768u);
      tma_load_2d(sb + L::oA, &p.tm_ks, kfull, 0, (int)srow);
      tma_load_2d(sb + L::oA + 16384, &p.tm_ks, kfull, 64, (int)srow);
    }
  };
  auto load_v = [&](int s) {
    if (s < n_tok) {
      mbar_arrive_expect_tx(vfull, tok_bytes);
      tma_load_4d(sb + L::oB, &p.tm_vt, vfull, 0, h, j * C + s * W, b);
      tma_load_4d(sb + L::oB + W * 128, &p.tm_vt, vfull, 64, h, j * C + s * W, b);
    } else {
      mbar_arrive_expect_tx(vfull, 32768u);
      tma_load_2d(sb + L::oB, &p.tm_vs, vfull, 0, (int)srow);
      tma_load_2d(sb + L::oB + 16384, &p.tm_vs, vfull, 64, (int)srow);
    }
  };
  if (threadIdx.x == 0) {
    for (int i = 0; i < 9; ++i) mbar_init(&kfull[i], i == 4 ? 8 : i == 7 ? 3 : 1);
    fence_barrier_init();
    load_k(0);
    load_v(0);
  }
  if (warp == 0) {
    tc::tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tc::tmem_relinquish();
  }
  // gather the rows' rotated queries: each half-warp one row, lane = 16-byte chunk; rows
  // 2 (w + 12 i) + (lane >> 4)
  {
    constexpr int kW = kAttnThreads / 32;
    const int c16 = lane & 15;
    for (int i = 0; 2 * (warp + kW * i) < kRows; ++i) {
      const int r = 2 * (warp + kW * i) + (lane >> 4);
      const int ent = r < n_rows ? p.list[first + r] : -1;
      const int t = ent >= 0 ? (ent >> 5) : -1;
      const bf16_t *src = t >= 0 ? p.qrope + (((size_t)b * p.T + t) * p.H + h) * kD + c16 * 8 : p.qrope;
      const uint32_t dst = sb + L::oQ + (c16 >> 3) * 16384 + r * 128 + (((c16 & 7) ^ (r & 7)) << 4);
      cp_async16_zfill(dst, src, t >= 0);
      if (c16 == 0) {
        row_t[r] = t;
        row_slot[r] = ent >= 0 ? (ent & 31) : 0;
      }
    }
  }
  cp_async_commit();
  cp_async_wait<0>();
  tc::fence_proxy_async_smem();
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 0) {
    auto wait_all = [&](uint64_t *bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, p.status));
    };
    const uint64_t dQ = tc::desc_kmajor_sw128(sb + L::oQ), dK = tc::desc_kmajor_sw128(sb + L::oA);
    constexpr uint32_t idO = tc::idesc_bf16_f32(128, kD, 0, 1);
    const uint32_t tS = tbase + L::kSCol, tO = tbase + L::kOCol;
    int k_loaded = 1, v_loaded = 1;  // tiles issued into slot A / B so far (phases armed)
    bool ok = true;
    for (int s = 0; s < n_seg && ok; ++s) {
      const int w = s < n_tok ? W : kM;  // keys of this segment
      const uint32_t par = (uint32_t)s & 1u;
      if (s == n_tok && !wait_all(qraw, 0)) { ok = false; break; }  // the raw queries are gathered
      if (!wait_all(kfull, par)) { ok = false; break; }
      if (s > 0 && !wait_all(odone, par ^ 1u)) { ok = false; break; }  // P of segment s - 1 (over S) is read
      tc::fence_after();
      // ---- S_s = Q K_s^T ----
      {
        const uint32_t idS = tc::idesc_bf16_f32(128, (uint32_t)w, 0, 0);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t qo = (uint32_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
          const uint32_t ko = (uint32_t)(((kk >> 2) * w * 128 + (kk & 3) * 32) >> 4);
          tc::mma_ss_w(tS, dQ + qo, dK + ko, idS, kk ? 1u : 0u);
        }
        tc::commit_w(sdone);
        tc::commit_w(kfree);
        if (slots && s == n_tok - 1) tc::commit_w(qfree);  // the rotated queries are read
      }
      if (s + 1 < n_seg) {  // slot A: the next K tile, once S_s has read this one
        if (!wait_all(kfree, par)) { ok = false; break; }
        if (lane == 0) load_k(s + 1);
        ++k_loaded;
      }
      // ---- O += P_s V_s ----
      if (!wait_all(pfull, par) || !wait_all(vfull, par)) { ok = false; break; }
      tc::fence_after();
      {
        const uint64_t dV = tc::desc_mnmajor_sw128(sb + L::oB, (uint32_t)w * 128u, 1024);
        // P of keys 16 kk ..: the first half's at column 8 kk, the second half's at w/2 + 8 (kk - w/32)
        for (int kk = 0; kk < w / 16; ++kk) {
          const uint32_t pc = kk < w / 32 ? (uint32_t)(8 * kk) : (uint32_t)(w / 2 + 8 * (kk - w / 32));
          tc::mma_ts_w(tO, tS + pc, dV + (uint32_t)kk * 128u, idO, (s | kk) ? 1u : 0u);
        }
        tc::commit_w(odone);
      }
      if (s + 1 < n_seg) {  // slot B: the next V tile, once this segment's product has read this one
        if (!wait_all(odone, par)) { ok = false; break; }
        if (lane == 0) load_v(s + 1);
        ++v_loaded;
      }
    }
    // every MMA completes before tensor memory is released; every load lands before exit
    tc::commit_w(fin);
    mbar_wait(fin, 0, p.status);
    if (lane == 0) {
      mbar_wait(kfull, (uint32_t)(k_loaded - 1) & 1u, p.status);
      mbar_wait(vfull, (uint32_t)(v_loaded - 1) & 1u, p.status);
    }
    __syncwarp();
  } else if (warp < 4) {
    // ---- the raw queries, once the last token segment's S has read the rotated ones ----
    if (slots) {
      const bool w = __all_sync(0xffffffffu, mbar_wait(qfree, 0, p.status));
      if (w) {
        const int c16 = lane & 15;
        for (int i = 0; 2 * ((warp - 1) + 3 * i) < kRows; ++i) {
          const int r = 2 * ((warp - 1) + 3 * i) + (lane >> 4);
          const int t = row_t[r];
          const bf16_t *src = t >= 0 ? p.qraw + (((size_t)b * p.T + t) * p.H + h) * kD + c16 * 8 : p.qraw;
          const uint32_t dst = sb + L::oQ + (c16 >> 3) * 16384 + r * 128 + (((c16 & 7) ^ (r & 7)) << 4);
          cp_async16_zfill(dst, src, t >= 0);
        }
        cp_async_commit();
        cp_async_wait<0>();
        tc::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(qraw);
      }
    }
  } else {
    // ---- softmax: two warps per row quarter, each one thread per row over half of a segment's
    // columns.  Each warp writes its P as bf16 pairs at the start of its own S columns, so that no
    // warp overwrites columns the other still reads. ----
    const int q4 = warp & 3, half = (warp - 4) >> 2, r = q4 * 32 + lane;
    const uint32_t tl = tbase + ((uint32_t)(q4 * 32) << 16);
    float *xmax = reinterpret_cast<float *>(sm + L::oX);  // [2][128]
    float *xsum = xmax + 256;                              // [2][128]
    const int t = row_t[r], slot = row_slot[r];
    const int lim = (t >= 0 && slot == p.K) ? t - j * C : C - 1;  // last valid token column
    float m_run = -INFINITY, l = 0.f;
    bool ok = true;
    for (int s = 0; s < n_seg; ++s) {
      const int w = s < n_tok ? W : kM;
      const int c0 = half * (w / 2);                      // first S column of this warp
      const int key0 = s < n_tok ? s * W + c0 : -1;       // its first token column (-1: slots)
      const uint32_t tS = tl + L::kSCol + c0;
      bool wt = mbar_wait(sdone, (uint32_t)s & 1u, p.status);
      wt = __all_sync(0xffffffffu, wt);
      float mx = -INFINITY;
      if (wt) {
        tc::fence_after();
        for (int c = 0; c < w / 64; ++c) {
          uint32_t v[32];
          tc::ld32(tS + c * 32, v);
          tc::wait_ld();
          tc::regfence(v);
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (key0 < 0 || key0 + c * 32 + e <= lim) mx = fmaxf(mx, __uint_as_float(v[e]));
        }
      }
      xmax[half * 128 + r] = mx;
      wt = pair_and(q4, wt);
      if (!wt) {
        ok = false;
        break;
      }
      const float m_new = fmaxf(m_run, fmaxf(mx, xmax[(half ^ 1) * 128 + r]));
      // the running values move with the maximum: l and (s > 0) this warp's 64 columns of O
      const float alpha = m_run == -INFINITY ? 0.f : ex2f((m_run - m_new) * p.cs);
      l *= alpha;
      if (s > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          uint32_t v[32];
          tc::ld32(tl + L::kOCol + half * 64 + c * 32, v);
          tc::wait_ld();
          tc::regfence(v);
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
          tc::st32u(tl + L::kOCol + half * 64 + c * 32, v);
        }
      }
      m_run = m_new;
      const float nm = m_new == -INFINITY ? 0.f : -m_new * p.cs;
      for (int c = 0; c < w / 64; ++c) {
        uint32_t v[32], pk[16];
        tc::ld32(tS + c * 32, v);
        tc::wait_ld();
        tc::regfence(v);
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const bool ok0 = key0 < 0 || key0 + c * 32 + e <= lim, ok1 = key0 < 0 || key0 + c * 32 + e + 1 <= lim;
          const float e0 = ok0 ? ex2f(fmaf(__uint_as_float(v[e]), p.cs, nm)) : 0.f;
          const float e1 = ok1 ? ex2f(fmaf(__uint_as_float(v[e + 1]), p.cs, nm)) : 0.f;
          l += e0 + e1;
          pk[e >> 1] = pack_bf16(e0, e1);
        }
        tc::st16u(tS + c * 16, pk);
      }
      tc::wait_st();
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(pfull);
    }
    // ---- epilogue: this warp's 64 columns of O / l, and (half 0) the row's log-sum-exp ----
    bool we = ok && mbar_wait(odone, (uint32_t)(n_seg - 1) & 1u, p.status);
    we = __all_sync(0xffffffffu, we);
    xsum[half * 128 + r] = l;
    we = pair_and(q4, we);
    if (we) {
      tc::fence_after();
      l += xsum[(half ^ 1) * 128 + r];
      const float inv = 1.f / l;
      const size_t orow = (((size_t)b * p.T + (t >= 0 ? t : 0)) * p.H + h) * (p.K + 1) + slot;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t v[32];
        tc::ld32(tl + L::kOCol + half * 64 + c * 32, v);
        tc::wait_ld();
        tc::regfence(v);
        if (t >= 0) {
#pragma unroll
          for (int e = 0; e < 32; e += 8)
            *reinterpret_cast<uint4 *>(p.po + orow * kD + half * 64 + c * 32 + e) =
                make_uint4(pack_bf16(__uint_as_float(v[e]) * inv, __uint_as_float(v[e + 1]) * inv),
                           pack_bf16(__uint_as_float(v[e + 2]) * inv, __uint_as_float(v[e + 3]) * inv),
                           pack_bf16(__uint_as_float(v[e + 4]) * inv, __uint_as_float(v[e + 5]) * inv),
                           pack_bf16(__uint_as_float(v[e + 6]) * inv, __uint_as_float(v[e + 7]) * inv));
        }
      }
      if (t >= 0 && half == 0) p.plse[orow] = m_run * p.cs + __log2f(l);
    }
  }
  tc::fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after();
    tc::tmem_dealloc(tbase, L::kTmemCols);
  }
}

// per (sequence, token, head), one warp: o = sum_k 2^{lse_k} o_k / sum_k 2^{lse_k} over the own
// block's partial and those of the kept blocks
__global__ void phba_merge_kernel(const bf16_t *__restrict__ po, const float *__restrict__ plse,
                                  const int32_t *__restrict__ sel, bf16_t *__restrict__ o, int B, int T, int H, int K) {
  const size_t n = (size_t)B * T * H;
  const int lane = threadIdx.x & 31;
  for (size_t idx = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; idx < n;
       idx += ((size_t)gridDim.x * blockDim.x) >> 5) {
    // lane k <= K reads partial k's log-sum-exp (-inf where block k was not kept); every lane reads its
    // four columns of every partial at once (entries of blocks not kept are in bounds and never used)
    const bool kept = lane <= K && (lane == K || sel[idx * K + lane] >= 0);
    const float lraw = lane <= K ? plse[idx * (K + 1) + lane] : 0.f;
    uint2 v[17];
#pragma unroll
    for (int k = 0; k < 17; ++k)
      if (k <= K) v[k] = *reinterpret_cast<const uint2 *>(po + (idx * (K + 1) + k) * kD + 4 * lane);
    const float lk = kept ? lraw : -INFINITY;
    float mx = lk;
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
    const float wl = kept ? ex2f(lk - mx) : 0.f;
    float acc[4] = {0.f, 0.f, 0.f, 0.f}, den = 0.f;
#pragma unroll
    for (int k = 0; k < 17; ++k) {
      if (k > K) break;
      const float w = __shfl_sync(0xffffffffu, wl, k);
      if (w == 0.f) continue;
      den += w;
      acc[0] = fmaf(w, bf16_lo(v[k].x), acc[0]);
      acc[1] = fmaf(w, bf16_hi(v[k].x), acc[1]);
      acc[2] = fmaf(w, bf16_lo(v[k].y), acc[2]);
      acc[3] = fmaf(w, bf16_hi(v[k].y), acc[3]);
    }
    const float inv = 1.f / den;
    *reinterpret_cast<uint2 *>(o + idx * kD + 4 * lane) =
        make_uint2(pack_bf16(acc[0] * inv, acc[1] * inv), pack_bf16(acc[2] * inv, acc[3] * inv));
  }
}

size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

int sm_count() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

}  // namespace

size_t phba_states_workspace_bytes(int B, int T, int H, int C) {
  const size_t nb = ((size_t)T + C - 1) / C;
  return al256((size_t)B * H * nb * 2 * kM * kD * 4) + al256((size_t)B * H * nb * kM * 4);
}

cudaError_t launch_phba_states(const PhbaStatesArgs &a, cudaStream_t s) {
  const int nb = (a.T + a.C - 1) / a.C;
  uint8_t *w = reinterpret_cast<uint8_t *>(a.workspace);
  float *Lw = reinterpret_cast<float *>(w);
  float *Dw = reinterpret_cast<float *>(w + al256((size_t)a.B * a.H * nb * 2 * kM * kD * 4));
  cudaError_t e;
  if (nb > 1) {
    SlotParams p;
    memset(&p, 0, sizeof(p));
    const uint32_t box[4] = {64, 1, kSubTok, 1};
    const uint64_t dims[4] = {(uint64_t)kD, (uint64_t)a.H, (uint64_t)a.T, (uint64_t)a.B};
    const uint64_t str[3] = {(uint64_t)kD * 2, (uint64_t)a.H * kD * 2, (uint64_t)a.T * a.H * kD * 2};
    if (encode_tmap(&p.tm_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.k_raw, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
        encode_tmap(&p.tm_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.v, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) {
      set_error("phba_prefix_states: cuTensorMapEncodeTiled failed");
      return cudaErrorInvalidValue;
    }
    p.alpha = a.alpha;
    p.L = Lw;
    p.D = Dw;
    p.B = a.B;
    p.T = a.T;
    p.H = a.H;
    p.C = a.C;
    p.nb = nb;
    p.status = device_status_ptr();
    const int smem = SlotSmem::kTotal + 1024;
    if ((e = cudaFuncSetAttribute(phba_slots_local_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess)
      return e;
    phba_slots_local_kernel<<<dim3(nb - 1, a.H, a.B), 256, smem, s>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const size_t threads = (size_t)a.B * a.H * kM * (kD / 4);
  const unsigned grid = (unsigned)((threads + 255) / 256);
  phba_slots_combine_kernel<<<grid, 256, 0, s>>>(Lw, Dw, a.kstate, a.vstate, a.B, a.H, nb);
  return cudaGetLastError();
}

namespace {
struct FwdLayout {
  size_t kbar, sel, rank, cnt, off, toff, tiles, list, po, plse, total;
};
FwdLayout fwd_layout(int B, int T, int H, int C, int K) {
  const size_t nb = ((size_t)T + C - 1) / C, nfull = (size_t)T / C, NB = (size_t)B * H * nb;
  const size_t q = (size_t)B * T * H;
  FwdLayout l;
  size_t o = 0;
  l.kbar = o;
  o += al256((nfull ? nfull : 1) * B * H * kD * 4);
  l.sel = o;
  o += al256(q * (K ? K : 1) * 4);
  l.rank = o;
  o += al256(q * (K ? K : 1) * 4);
  l.cnt = o;
  o += al256(NB * 4);
  l.off = o;
  o += al256((NB + 1) * 4);
  l.toff = o;
  o += al256((NB + 1) * 4);
  l.tiles = o;
  o += al256((NB + (q * (K + 1) + kRows - 1) / kRows) * 16);
  l.list = o;
  o += al256(q * (K + 1) * 4);
  l.po = o;
  o += al256(q * (K + 1) * kD * 2);
  l.plse = o;
  o += al256(q * (K + 1) * 4);
  l.total = o;
  return l;
}
}  // namespace

size_t phba_fwd_workspace_bytes(int B, int T, int H, int C, int K) { return fwd_layout(B, T, H, C, K).total; }

cudaError_t launch_phba_fwd(const PhbaFwdArgs &a, cudaStream_t s) {
  const int nb = (a.T + a.C - 1) / a.C, nfull = a.T / a.C, NB = a.B * a.H * nb;
  const FwdLayout l = fwd_layout(a.B, a.T, a.H, a.C, a.K);
  uint8_t *w = reinterpret_cast<uint8_t *>(a.workspace);
  float *kbar = reinterpret_cast<float *>(w + l.kbar);
  int32_t *sel = a.sel ? a.sel : reinterpret_cast<int32_t *>(w + l.sel);
  int32_t *rank = reinterpret_cast<int32_t *>(w + l.rank);
  int32_t *cnt = reinterpret_cast<int32_t *>(w + l.cnt);
  int32_t *off = reinterpret_cast<int32_t *>(w + l.off);
  int32_t *toff = reinterpret_cast<int32_t *>(w + l.toff);
  int32_t *list = reinterpret_cast<int32_t *>(w + l.list);
  int4 *tiles = reinterpret_cast<int4 *>(w + l.tiles);
  bf16_t *po = reinterpret_cast<bf16_t *>(w + l.po);
  float *plse = reinterpret_cast<float *>(w + l.plse);
  cudaError_t e;
  // routing
  if ((e = cudaMemsetAsync(cnt, 0, (size_t)NB * 4, s)) != cudaSuccess) return e;
  if (nfull > 0) {
    phba_block_means_kernel<<<dim3(nfull, a.H, a.B), 256, 0, s>>>(a.k_rope, kbar, a.T, a.H, a.C, nfull);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (a.K > 0) {
    RouteParams rp;
    rp.qrope = a.q_rope;
    rp.kbar = kbar;
    rp.sel = sel;
    rp.rank = rank;
    rp.cnt = cnt;
    rp.B = a.B;
    rp.T = a.T;
    rp.H = a.H;
    rp.C = a.C;
    rp.K = a.K;
    rp.nb = nb;
    rp.nfull = nfull;
    static_assert(kRq * (kRc + 1) <= kD * (kRc + 4), "the chunk's scores fit over its block means");
    const int smem = (kD * (kRq + 4) + kD * (kRc + 4) + 2 * kRq * 16 + 2 * kMaxCand) * 4;
    auto route = a.K <= 4 ? phba_route_kernel<4> : a.K <= 8 ? phba_route_kernel<8> : phba_route_kernel<16>;
    if ((e = cudaFuncSetAttribute(route, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess) return e;
    route<<<dim3((a.T + kRq - 1) / kRq, a.H, a.B), 256, smem, s>>>(rp);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  phba_bucket_scan_kernel<<<1, 1024, 0, s>>>(cnt, off, toff, tiles, NB, nb, a.T, a.C);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  {
    const size_t n = (size_t)a.B * a.T * a.H;
    const unsigned grid = (unsigned)min((n + 255) / 256, (size_t)sm_count() * 16);
    phba_bucket_fill_kernel<<<grid, 256, 0, s>>>(sel, rank, off, list, a.B, a.T, a.H, a.C, a.K, nb);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // attention tiles
  {
    AttnParams p;
    memset(&p, 0, sizeof(p));
    const uint32_t box_t[4] = {64, 1, (uint32_t)min(a.C, 128), 1};  // one key segment
    const uint64_t dims[4] = {(uint64_t)kD, (uint64_t)a.H, (uint64_t)a.T, (uint64_t)a.B};
    const uint64_t str[3] = {(uint64_t)kD * 2, (uint64_t)a.H * kD * 2, (uint64_t)a.T * a.H * kD * 2};
    const uint32_t box_s[2] = {64, (uint32_t)kM};
    const uint64_t sdims[2] = {(uint64_t)kD, (uint64_t)a.B * a.H * nb * kM};
    const uint64_t sstr[1] = {(uint64_t)kD * 2};
    if (encode_tmap(&p.tm_kt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.k_rope, dims, str, box_t, CU_TENSOR_MAP_SWIZZLE_128B) ||
        encode_tmap(&p.tm_vt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.v, dims, str, box_t, CU_TENSOR_MAP_SWIZZLE_128B) ||
        encode_tmap(&p.tm_ks, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.kstate, sdims, sstr, box_s, CU_TENSOR_MAP_SWIZZLE_128B) ||
        encode_tmap(&p.tm_vs, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.vstate, sdims, sstr, box_s, CU_TENSOR_MAP_SWIZZLE_128B)) {
      set_error("phba_fwd: cuTensorMapEncodeTiled failed");
      return cudaErrorInvalidValue;
    }
    p.qrope = a.q_rope;
    p.qraw = a.q_raw;
    p.list = list;
    p.toff = toff;
    p.tiles = tiles;
    p.po = po;
    p.plse = plse;
    p.B = a.B;
    p.T = a.T;
    p.H = a.H;
    p.C = a.C;
    p.K = a.K;
    p.nb = nb;
    p.NB = NB;
    p.cs = a.scale * kLog2e;
    p.status = device_status_ptr();
    const int smem = AttnSmem::kTotal + 1024;
    if ((e = cudaFuncSetAttribute(phba_attn_tiles_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess)
      return e;
    const size_t bound = (size_t)NB + ((size_t)a.B * a.H * a.T * (a.K + 1) + kRows - 1) / kRows;
    phba_attn_tiles_kernel<<<(unsigned)bound, kAttnThreads, smem, s>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {
    const size_t warps = (size_t)a.B * a.T * a.H;
    const unsigned grid = (unsigned)min((warps + 7) / 8, (size_t)sm_count() * 32);
    phba_merge_kernel<<<grid, 256, 0, s>>>(po, plse, sel, a.o, a.B, a.T, a.H, a.K);
  }
  return cudaGetLastError();
}

}  // namespace hh
