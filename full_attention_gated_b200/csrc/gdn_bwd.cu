// gdn_bwd.cu -- gradients of the gated delta rule over a sequence: the backward pass of
// gdn_chunk_fwd.
//
// The layers are trained ("HydraHead: From Head-Level Functional Heterogeneity to
// Specialized Attention Hybridization", abstract: the hybrid heads come out of a transfer
// and distillation pipeline; "PHBA: Prefix-State Hybrid Block Attention", Figure 3: training
// throughput), which needs the gradients of
//     L = sum_t o_t . dO_t + S_T . dS_T
// through S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T, o_t = scale S_t q_t,
// with respect to q, k, v, g, beta and S_0.  In the chunked form (C = 64) the chunk map is
// affine, S_{c+1} = S_c A_c + B_c, and the chunk's output is O_c = scale (Qt_c S_c^T + P_c U'_c),
// so the backward splits into
//   1. the forward pass with the start state S_c of every chunk kept (gdn_scan's chunk_states);
//   2. a reverse scan over chunks carrying the state's cotangent,
//          dS_c = dS_{c+1} A_c^T + scale dO_c^T Qt_c,      dS_n = dS_T,  dS_0 -> dS0,
//      whose per-chunk terms A_c^T and E_c = scale dO_c^T Qt_c are formed for all chunks at once
//      first, so that the sequential chain is one product per chunk;
//   3. per chunk, independently, the cotangents of the chunk's maps,
//          dA = S_c^T dS_{c+1},  dB = dS_{c+1},  dQt = scale dO S_c,  dP = scale dO U'^T,
//          dU' = scale P^T dO,
//      pulled back through B = U'^T diag(e) K, A = gamma_C I - W^T diag(e) K, Qt = diag(gamma) Q - P W,
//      P = tril(D o Q K^T), W = T diag(beta gamma) K, U' = T diag(beta) V, T = (I + A_in)^-1 with
//      A_in = strict_tril(beta_i D_ij k_i.k_j), D_ij = exp(G_i - G_j), G = cumsum(g), to q, k, v, g
//      and beta.
// Steps 2 and 3 keep fp32 values; their products run on the 5th-generation tensor cores with every
// fp32 operand split into two bf16 terms (fp32-accurate, tc_mm below), and the chunk's forward
// quantities are recomputed from the inputs.  Step 1 is the forward pass itself.  Kernels:
//   gdn_bwd_maps   per (head, chunk): A_c^T and E_c (256 threads, one CTA per SM);
//   gdn_bwd_scan   per (head, sequence, half of the state's rows): the chain dS_c, one product per
//                  chunk (the halves are independent: the chain acts on the rows of dS);
//   gdn_bwd_chunk  per (head, chunk): step 3 (128 threads, two CTAs per SM, 64-row A tiles).
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace hh {

namespace {

constexpr int kC = 64;
constexpr int kD = 128;
constexpr int kBT = 256;  // threads per CTA of the maps and scan kernels


// ---- C = alpha op(A) op(B) + beta C on the 5th-generation tensor cores, fp32 accurate ----
// op(A) is M x K: A row-major with leading dimension lda, or its transpose (ta); op(B) is K x N likewise
// (tb).  M, N, K in {64, 128}; beta = 0 does not read C.  Every fp32 operand x is split into two bf16
// terms, x = hi + lo with hi = bf16(x) and lo = bf16(x - hi), and the product is hi.hi + hi.lo + lo.hi
// (the lo.lo term is below fp32 rounding), accumulated in fp32 in tensor memory: about 2^-16 relative
// error per product, against 2^-8 for plain bf16 operands.  bf16 sources give lo = 0 exactly.
// Each operand is staged in the majorness it already has in memory, so no transpose is needed: A is
// K-major when K is contiguous (!ta) and MN-major otherwise, B likewise.  Tiles hold 128 rows of
// 128-byte-swizzled 64-column boxes; the MMAs always run with M = 128, and rows of D past M (from rows
// of A past M) are not read back.
constexpr int kBTerm = 32768;  // one bf16 term of B: 2 boxes x 128 rows x 128 bytes
struct TcMm {
  uint8_t *tiles;   // 1024-byte-aligned: A hi | A lo | B hi | B lo
  uint32_t stiles;  // its shared-memory address
  int a_cap;        // rows of a K-major A tile (64 or 128): A products have M <= a_cap
  uint32_t tmem;    // the accumulator: 128 lanes x 128 fp32 columns
  uint64_t *bar;    // MMA completion
  uint32_t phase;
  unsigned *status;
  bool ok;          // false once a wait gave up: later products are skipped
  __device__ int a_term() const { return a_cap * 256; }  // bytes of one A term
};
// shared memory of the tiles for a given A capacity
constexpr int tc_mm_smem(int a_cap) { return 2 * a_cap * 256 + 2 * kBTerm + 1024; }

__device__ __forceinline__ void load8(const float *p, float (&v)[8]) {
  const float4 a = *reinterpret_cast<const float4 *>(p), b = *reinterpret_cast<const float4 *>(p + 4);
  v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
}
__device__ __forceinline__ void load8(const bf16_t *p, float (&v)[8]) {
  const uint4 a = *reinterpret_cast<const uint4 *>(p);
  v[0] = bf16_lo(a.x), v[1] = bf16_hi(a.x), v[2] = bf16_lo(a.y), v[3] = bf16_hi(a.y);
  v[4] = bf16_lo(a.z), v[5] = bf16_hi(a.z), v[6] = bf16_lo(a.w), v[7] = bf16_hi(a.w);
}
// one 16-byte chunk (8 values) as hi and lo terms at byte `off` of the two term tiles
__device__ __forceinline__ void store_terms(const float (&v)[8], uint8_t *hi, int lo_off, uint32_t off) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    h[k] = pack_bf16(v[2 * k], v[2 * k + 1]);
    l[k] = pack_bf16(v[2 * k] - bf16_lo(h[k]), v[2 * k + 1] - bf16_hi(h[k]));
  }
  *reinterpret_cast<uint4 *>(hi + off) = make_uint4(h[0], h[1], h[2], h[3]);
  *reinterpret_cast<uint4 *>(hi + lo_off + off) = make_uint4(l[0], l[1], l[2], l[3]);
}
// Operand staging: src is rows x cols, row-major with leading dimension ld (cols contiguous), into
// 128-byte rows of 64-column boxes `box` bytes apart, 16-byte chunks swizzled by the row.
struct Stage {
  int rows, sh, box, lo_off;  // sh: log2 of the 16-byte chunks per row (3: 64 cols, 4: 128 cols)
  uint8_t *dst;
  __device__ int total() const { return rows << sh; }
  __device__ uint32_t off(int e) const {
    const int r = e >> sh, c = e & ((1 << sh) - 1);
    return (uint32_t)(c >> 3) * (uint32_t)box + (uint32_t)r * 128u + ((uint32_t)((c & 7) ^ (r & 7)) << 4);
  }
};
// Both operands, NT threads, in rounds of R chunks per thread per operand with all of a round's loads
// issued before any store.
template <int NT, typename TA, typename TB>
__device__ __forceinline__ void stage_pair(const TA *a, int lda, const Stage &sa, const TB *b, int ldb,
                                           const Stage &sb) {
  constexpr int R = NT >= 256 ? 8 : 4;
  const int n = max(sa.total(), sb.total());
  for (int base = 0; base < n; base += R * NT) {
    float va[R][8], vb[R][8];
#pragma unroll
    for (int it = 0; it < R; ++it) {
      const int e = base + threadIdx.x + it * NT;
      if (e < sa.total()) load8(a + (size_t)(e >> sa.sh) * lda + 8 * (e & ((1 << sa.sh) - 1)), va[it]);
      if (e < sb.total()) load8(b + (size_t)(e >> sb.sh) * ldb + 8 * (e & ((1 << sb.sh) - 1)), vb[it]);
    }
#pragma unroll
    for (int it = 0; it < R; ++it) {
      const int e = base + threadIdx.x + it * NT;
      if (e < sa.total()) store_terms(va[it], sa.dst, sa.lo_off, sa.off(e));
      if (e < sb.total()) store_terms(vb[it], sb.dst, sb.lo_off, sb.off(e));
    }
  }
}

template <int NT, typename TA, typename TB>
__device__ __noinline__ void tc_mm(float *C, int ldc, const TA *A, int lda, bool ta, const TB *B, int ldb, bool tb,
                                   int M, int N, int K, float alpha, float beta, TcMm &mm) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int at = mm.a_term();
  // A: K-major (rows M, boxes a_cap rows apart) or MN-major (rows K, boxes 128 rows apart)
  const int a_box = ta ? 16384 : mm.a_cap * 128;
  {
    const Stage sa{ta ? K : M, (ta ? M : K) == 128 ? 4 : 3, a_box, at, mm.tiles};
    const Stage sb{tb ? N : K, (tb ? K : N) == 128 ? 4 : 3, 16384, kBTerm, mm.tiles + 2 * at};
    stage_pair<NT>(A, lda, sa, B, ldb, sb);
  }
  tc::fence_proxy_async_smem();
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  if (warp == 0 && mm.ok) {
    const uint32_t sA = mm.stiles, sB = mm.stiles + 2 * at;
    const uint32_t id = tc::idesc_bf16_f32(128, N, ta ? 1 : 0, tb ? 0 : 1);
    uint64_t dA[2], dB[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      dA[t] = ta ? tc::desc_mnmajor_sw128(sA + t * at, 16384, 1024) : tc::desc_kmajor_sw128(sA + t * at);
      dB[t] = tb ? tc::desc_kmajor_sw128(sB + t * kBTerm) : tc::desc_mnmajor_sw128(sB + t * kBTerm, 16384, 1024);
    }
    for (int kk = 0; kk < K / 16; ++kk) {
      const uint32_t mnmaj = (uint32_t)kk * 128u;
      const uint32_t oa = ta ? mnmaj : (uint32_t)(((kk >> 2) * a_box + (kk & 3) * 32) >> 4);
      const uint32_t ob = tb ? (uint32_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4) : mnmaj;
      tc::mma_ss_w(mm.tmem, dA[0] + oa, dB[0] + ob, id, kk ? 1u : 0u);
      tc::mma_ss_w(mm.tmem, dA[0] + oa, dB[1] + ob, id, 1u);
      tc::mma_ss_w(mm.tmem, dA[1] + oa, dB[0] + ob, id, 1u);
    }
    tc::commit_w(mm.bar);
  }
  // read back: warp w takes the rows of lane quarter w % 4 and a 1 / (NT / 128) share of the columns.
  // With beta != 0 the old values of C are loaded while the MMAs run, all at once.
  constexpr int kParts = NT / 128;  // column parts per row quarter
  const int q4 = warp & 3, part = warp >> 2, row = q4 * 32 + lane;
  const int ncol = N / kParts;  // 32, 64 or 128 columns per warp
  const bool mine = q4 * 32 < M;
  float *crow = C + (size_t)row * ldc + part * ncol;
  float4 old[32];
  if (beta != 0.f && mine) {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i < ncol / 4) old[i] = *reinterpret_cast<const float4 *>(crow + 4 * i);
  }
  bool w = mm.ok ? mbar_wait(mm.bar, mm.phase, mm.status) : false;
  mm.phase ^= mm.ok ? 1u : 0u;
  mm.ok = __syncthreads_and(w) != 0;
  tc::fence_after();
  if (mm.ok && mine) {
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      if (h * 32 >= ncol) break;
      uint32_t v[32];
      tc::ld32(mm.tmem + ((uint32_t)(q4 * 32) << 16) + part * ncol + h * 32, v);
      tc::wait_ld();
      tc::regfence(v);
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        float4 o = make_float4(alpha * __uint_as_float(v[i]), alpha * __uint_as_float(v[i + 1]),
                               alpha * __uint_as_float(v[i + 2]), alpha * __uint_as_float(v[i + 3]));
        if (beta != 0.f) {
          const float4 x = old[h * 8 + i / 4];
          o.x = fmaf(beta, x.x, o.x);
          o.y = fmaf(beta, x.y, o.y);
          o.z = fmaf(beta, x.z, o.z);
          o.w = fmaf(beta, x.w, o.w);
        }
        *reinterpret_cast<float4 *>(crow + h * 32 + i) = o;
      }
    }
  }
  tc::fence_before();
  __syncthreads();
}

// tensor memory and the completion barrier of tc_mm: set up at kernel start, released at the end
__device__ TcMm tc_mm_begin(uint8_t *dyn_smem, int a_cap, uint64_t *bar, uint32_t *tmem_slot, unsigned *status) {
  TcMm mm;
  mm.a_cap = a_cap;
  mm.tiles = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
  mm.stiles = smem_u32(mm.tiles);
  mm.bar = bar;
  mm.phase = 0;
  mm.status = status;
  mm.ok = true;
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  if ((threadIdx.x >> 5) == 0) {
    tc::tmem_alloc(smem_u32(tmem_slot), 128);
    tc::tmem_relinquish();
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  mm.tmem = *tmem_slot;
  return mm;
}
__device__ void tc_mm_end(const TcMm &mm) {
  tc::fence_before();
  __syncthreads();
  if ((threadIdx.x >> 5) == 0) {
    tc::fence_after();
    tc::tmem_dealloc(mm.tmem, 128);
  }
}
constexpr int kBwdDynSmem = tc_mm_smem(128);     // the maps and scan kernels: 128-row A products
constexpr int kBTC = 128;                        // threads of the pullback: two CTAs per SM
constexpr int kBwdChunkSmem = tc_mm_smem(64);    // the pullback: 64-row A products

// rows [t0, t0 + 64) of head h of a [B, T, H, 128] bf16 tensor -> fp32 [64][128], zero past T
// (16-byte loads, four per thread, all issued before any is used)
template <int NT = kBT>
__device__ void load_rows(float *dst, const bf16_t *src, int b, int T, int H, int h, int t0) {
  uint4 v[kC * kD / 8 / NT];
#pragma unroll
  for (int it = 0; it < kC * kD / 8 / NT; ++it) {
    const int e = threadIdx.x + it * NT, t = e >> 4, c = e & 15;
    v[it] = t0 + t < T ? *reinterpret_cast<const uint4 *>(src + (((size_t)b * T + t0 + t) * H + h) * kD + 8 * c)
                       : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int it = 0; it < kC * kD / 8 / NT; ++it) {
    const int e = threadIdx.x + it * NT;
    const uint32_t w[4] = {v[it].x, v[it].y, v[it].z, v[it].w};
    float4 *d = reinterpret_cast<float4 *>(dst + 8 * e);
    d[0] = make_float4(bf16_lo(w[0]), bf16_hi(w[0]), bf16_lo(w[1]), bf16_hi(w[1]));
    d[1] = make_float4(bf16_lo(w[2]), bf16_hi(w[2]), bf16_lo(w[3]), bf16_hi(w[3]));
  }
}

// out[r] = sum_j X[r][j] Y[r][j] (Y null: sum_j X[r][j]) for the 64 rows of [64][n] fp32 arrays,
// n = 64 or 128.  Warp w takes rows w, w + 8, ...; each lane a slice of the row (all loads at once),
// then a shuffle sum.  Ends with a barrier.
template <int NT>
__device__ void row_dots(const float *X, const float *Y, int n, float *out) {
  constexpr int kW = NT / 32, kR = kC / kW;  // warps, rows per warp
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float acc[kR];
#pragma unroll
  for (int i = 0; i < kR; ++i) {
    const int r = warp + kW * i;
    if (n == 128) {
      const float4 x = *reinterpret_cast<const float4 *>(X + r * 128 + 4 * lane);
      const float4 y = Y ? *reinterpret_cast<const float4 *>(Y + r * 128 + 4 * lane) : make_float4(1.f, 1.f, 1.f, 1.f);
      acc[i] = fmaf(x.x, y.x, fmaf(x.y, y.y, fmaf(x.z, y.z, x.w * y.w)));
    } else {
      const float2 x = *reinterpret_cast<const float2 *>(X + r * 64 + 2 * lane);
      const float2 y = Y ? *reinterpret_cast<const float2 *>(Y + r * 64 + 2 * lane) : make_float2(1.f, 1.f);
      acc[i] = fmaf(x.x, y.x, x.y * y.y);
    }
  }
#pragma unroll
  for (int i = 0; i < kR; ++i) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
    if (lane == 0) out[warp + kW * i] = acc[i];
  }
  __syncthreads();
}

struct BwdParams {
  const bf16_t *q, *k, *v, *dO;
  const float *g, *beta, *dS_T;  // dS_T nullable
  const float *chunk_states;     // [B, H_v, n_chunks, 128 (k), 128 (v)]: S^T at each chunk's start
  const bf16_t *rec_w, *rec_q;   // forward records: -W_e^T, Qt^T [B, H_v, n_chunks][128][64] bf16
  const float *rec_f;            // [B, H_v, n_chunks][2][64]: gamma, exp(G_C - G)
  float *dS;                     // [B, H_v, n_chunks][128 (v)][128 (k)]: dS_{c+1} of every chunk
  float *dq, *dk, *dv, *dg, *dbeta, *dS0;  // dS0 nullable
  float *At;                     // [B, H_v, n_chunks][128][128]: A_c^T of every chunk
  float *chunk_scratch;          // per pullback CTA: kChunkScratch floats
  int B, T, H_qk, H_v, group, n_chunks, n_items;
  float scale;
  unsigned *status;
};

// per-CTA scratch of the pullback (floats)
constexpr int kMat = kC * kD;  // 64 x 128
constexpr int kSq = kC * kC;   // 64 x 64
constexpr int kChunkScratchMaps = 2 * kC * kD;  // K and dO of a chunk, in the maps kernel
enum : int {
  oQf = 0, oKf = oQf + kMat, oVf = oKf + kMat, oDO = oVf + kMat, oW = oDO + kMat, oUp = oW + kMat, oRW = oUp + kMat,
  oRU = oRW + kMat, odQt = oRU + kMat, odUp = odQt + kMat, odW = odUp + kMat, odQ = odW + kMat, odK = odQ + kMat,
  odV = odK + kMat, oT1 = odV + kMat, oT2 = oT1 + kMat, odA = oT2 + kMat, oKK = odA + kD * kD, oQK = oKK + kSq,
  oDm = oQK + kSq, oTm = oDm + kSq, oP = oTm + kSq, odP = oP + kSq, odD = odP + kSq, odTm = odD + kSq, oS1 = odTm + kSq,
  oS2 = oS1 + kSq, kChunkScratch = oS2 + kSq
};

// ---- the reverse scan's per-chunk terms, all chunks at once (persistent grid over (chunk, head)):
//   At_c = A_c^T = gamma_C I - K^T W_e   (128 x 128, so that dS_c = dS_{c+1} At_c + E_c),
//   E_c  = scale dO_c^T Qt_c             (128 x 128), written where dS_c will be formed (dS0 for c = 0). ----
__global__ void __launch_bounds__(kBT, 1) gdn_bwd_maps_kernel(const __grid_constant__ BwdParams p) {
  extern __shared__ uint8_t dyn_smem[];
  __shared__ uint64_t mm_bar;
  __shared__ uint32_t tmem_slot;
  TcMm mm = tc_mm_begin(dyn_smem, 128, &mm_bar, &tmem_slot, p.status);
  float *Kc = p.chunk_scratch + (size_t)blockIdx.x * kChunkScratchMaps, *dOc = Kc + kC * kD;
  for (int item = blockIdx.x; item < p.n_items && mm.ok; item += gridDim.x) {
    const int h = item % p.H_v, rest = item / p.H_v, c = rest % p.n_chunks, b = rest / p.n_chunks;
    const size_t rec = ((size_t)b * p.H_v + h) * p.n_chunks + c;
    load_rows(Kc, p.k, b, p.T, p.H_qk, h / p.group, c * kC);
    load_rows(dOc, p.dO, b, p.T, p.H_v, h, c * kC);
    __syncthreads();
    const bf16_t *rw = p.rec_w + rec * kD * kC, *rq = p.rec_q + rec * kD * kC;  // -W_e^T, Qt^T [128][64]
    float *At = p.At + rec * kD * kD;
    tc_mm<kBT>(At, kD, Kc, kD, true, rw, kC, true, kD, kD, kC, 1.f, 0.f, mm);  // K^T (-W_e)
    if (threadIdx.x < kD) At[threadIdx.x * (kD + 1)] += p.rec_f[rec * 128 + kC - 1];  // + gamma_C I
    float *E = c > 0 ? p.dS + (rec - 1) * kD * kD : (p.dS0 ? p.dS0 + ((size_t)b * p.H_v + h) * kD * kD : nullptr);
    if (E) tc_mm<kBT>(E, kD, dOc, kD, true, rq, kC, true, kD, kD, kC, p.scale, 0.f, mm);  // scale dO^T Qt
    __syncthreads();
  }
  tc_mm_end(mm);
}

// ---- reverse scan, chunks from last to first: dS_c = dS_{c+1} At_c + E_c, one product per chunk.
// Row v of dS_c depends only on row v of dS_{c+1} (At acts on the right), so each CTA carries 64 rows
// of one (head, sequence): grid (heads, B, 2). ----
__global__ void __launch_bounds__(kBT, 1) gdn_bwd_scan_kernel(const __grid_constant__ BwdParams p) {
  extern __shared__ uint8_t dyn_smem[];
  __shared__ uint64_t mm_bar;
  __shared__ uint32_t tmem_slot;
  TcMm mm = tc_mm_begin(dyn_smem, 128, &mm_bar, &tmem_slot, p.status);
  const int h = blockIdx.x, b = blockIdx.y, rb = blockIdx.z;  // rows 64 rb .. 64 rb + 63 of dS
  const size_t rec0 = ((size_t)b * p.H_v + h) * p.n_chunks;
  const int n = p.n_chunks;
  const size_t roff = (size_t)rb * 64 * kD;  // first element of this CTA's rows
  {  // dS_n = dS_T (or zero)
    float *last = p.dS + (rec0 + n - 1) * kD * kD + roff;
    const float *src = p.dS_T ? p.dS_T + ((size_t)b * p.H_v + h) * kD * kD + roff : nullptr;
    for (int i = threadIdx.x; i < 64 * kD; i += kBT) last[i] = src ? src[i] : 0.f;
  }
  __syncthreads();
  for (int c = n - 1; c >= 0; --c) {
    const float *cur = p.dS + (rec0 + c) * kD * kD + roff;  // dS_{c+1}, this CTA's rows
    float *nxt = c > 0 ? p.dS + (rec0 + c - 1) * kD * kD + roff
                       : (p.dS0 ? p.dS0 + ((size_t)b * p.H_v + h) * kD * kD + roff : nullptr);
    if (!nxt || !mm.ok) break;
    tc_mm<kBT>(nxt, kD, cur, kD, false, p.At + (rec0 + c) * kD * kD, kD, false, 64, kD, kD, 1.f, 1.f, mm);
  }
  tc_mm_end(mm);
}

// ---- per-chunk pullback: a persistent grid over (chunk, head, sequence) ----
__global__ void __launch_bounds__(kBTC, 2) gdn_bwd_chunk_kernel(const __grid_constant__ BwdParams p) {
  extern __shared__ uint8_t dyn_smem[];
  __shared__ uint64_t mm_bar;
  __shared__ uint32_t tmem_slot;
  TcMm mm = tc_mm_begin(dyn_smem, 64, &mm_bar, &tmem_slot, p.status);
  // A_in and T live in the product tiles while T = (I + A_in)^-1 is formed (no product runs then)
  float(*Ash)[kC + 1] = reinterpret_cast<float(*)[kC + 1]>(mm.tiles);
  float(*Tsh)[kC + 1] = reinterpret_cast<float(*)[kC + 1]>(mm.tiles + 2 * 64 * 256);
  static_assert(kC * (kC + 1) * 4 <= 2 * 64 * 256 && kC * (kC + 1) * 4 <= 2 * kBTerm, "A_in and T fit in the tiles");
  __shared__ float G[kC], gam[kC], ee[kC], bb[kC], dgam[kC], de[kC], dbeta[kC], dG[kC], tmp[kC], tmp2[kC];
  __shared__ float red[2];
  float *sc = p.chunk_scratch + (size_t)blockIdx.x * kChunkScratch;
  float *Qf = sc + oQf, *Kf = sc + oKf, *Vf = sc + oVf, *dOf = sc + oDO, *W = sc + oW, *Up = sc + oUp, *RW = sc + oRW,
        *RU = sc + oRU, *dQt = sc + odQt, *dUp = sc + odUp, *dW = sc + odW, *dQ = sc + odQ, *dK = sc + odK,
        *dV = sc + odV, *T1 = sc + oT1, *T2 = sc + oT2, *dA = sc + odA, *KK = sc + oKK, *QK = sc + oQK, *Dm = sc + oDm,
        *Tm = sc + oTm, *P = sc + oP, *dP = sc + odP, *dD = sc + odD, *dTm = sc + odTm, *S1 = sc + oS1, *S2 = sc + oS2;
  const int tid = threadIdx.x;
  for (int item = blockIdx.x; item < p.n_items && mm.ok; item += gridDim.x) {
    const int h = item % p.H_v, rest = item / p.H_v, c = rest % p.n_chunks, b = rest / p.n_chunks;
    const int qh = h / p.group, t0 = c * kC, nv = min(kC, p.T - t0);
    const size_t rec = ((size_t)b * p.H_v + h) * p.n_chunks + c;
    const float *ST = p.chunk_states + rec * kD * kD;  // S_c^T [k][v]
    const float *dS = p.dS + rec * kD * kD;            // dS_{c+1} [v][k]
    // ---- inputs of the chunk (zero past T) and its gates ----
    load_rows<kBTC>(Qf, p.q, b, p.T, p.H_qk, qh, t0);
    load_rows<kBTC>(Kf, p.k, b, p.T, p.H_qk, qh, t0);
    load_rows<kBTC>(Vf, p.v, b, p.T, p.H_v, h, t0);
    load_rows<kBTC>(dOf, p.dO, b, p.T, p.H_v, h, t0);
    if (tid < 32) {
      float gv[2], bv[2];
#pragma unroll
      for (int e2 = 0; e2 < 2; ++e2) {
        const int t = 2 * tid + e2;
        const size_t idx = ((size_t)b * p.T + t0 + t) * p.H_v + h;
        gv[e2] = t < nv ? p.g[idx] : 0.f;
        bv[e2] = t < nv ? p.beta[idx] : 0.f;
      }
      float run = gv[0] + gv[1];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float o = __shfl_up_sync(0xffffffffu, run, off);
        if (tid >= off) run += o;
      }
      const float GC = __shfl_sync(0xffffffffu, run, 31);
      G[2 * tid] = run - gv[1];
      G[2 * tid + 1] = run;
      gam[2 * tid] = expf(run - gv[1]);
      gam[2 * tid + 1] = expf(run);
      ee[2 * tid] = expf(GC - (run - gv[1]));
      ee[2 * tid + 1] = expf(GC - run);
      bb[2 * tid] = bv[0];
      bb[2 * tid + 1] = bv[1];
    }
    __syncthreads();
    // ---- forward quantities of the chunk, fp32 ----
    tc_mm<kBTC>(KK, kC, Kf, kD, false, Kf, kD, true, kC, kC, kD, 1.f, 0.f, mm);
    tc_mm<kBTC>(QK, kC, Qf, kD, false, Kf, kD, true, kC, kC, kD, 1.f, 0.f, mm);
#pragma unroll 4
    for (int i = tid; i < kSq; i += kBTC) {  // D (lower with the diagonal; zero above), A_in, P
      const int r = i >> 6, cc = i & 63;
      const float d = cc <= r ? expf(G[r] - G[cc]) : 0.f;
      Dm[i] = d;
      Ash[r][cc] = cc < r ? bb[r] * d * KK[i] : 0.f;
      P[i] = d * QK[i];
    }
    __syncthreads();
    {  // (I + A_in)^-1 by forward substitution, column j by the two lanes 2 j, 2 j + 1 (one warp)
      const int j = tid >> 1, part = tid & 1;
      for (int t = part; t < kC; t += 2) Tsh[t][j] = t == j ? 1.f : 0.f;
      __syncwarp();
      for (int t = 1; t < kC; ++t) {
        float s = 0.f;
        if (t > j)
          for (int i = j + part; i < t; i += 2) s = fmaf(Ash[t][i], Tsh[i][j], s);
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        if (t > j && part == 0) Tsh[t][j] = -s;
        __syncwarp();
      }
    }
    __syncthreads();
#pragma unroll 4
    for (int i = tid; i < kSq; i += kBTC) Tm[i] = Tsh[i >> 6][i & 63];
#pragma unroll 8
    for (int i = tid; i < kMat; i += kBTC) {
      const int t = i >> 7;
      RW[i] = bb[t] * gam[t] * Kf[i];
      RU[i] = bb[t] * Vf[i];
    }
    __syncthreads();
    tc_mm<kBTC>(W, kD, Tm, kC, false, RW, kD, false, kC, kD, kC, 1.f, 0.f, mm);
    tc_mm<kBTC>(Up, kD, Tm, kC, false, RU, kD, false, kC, kD, kC, 1.f, 0.f, mm);
    // ---- cotangents of the chunk's maps ----
    tc_mm<kBTC>(dA, kD, ST, kD, false, dS, kD, false, kC, kD, kD, 1.f, 0.f, mm);  // S_c^T dS_{c+1}, rows 0..63
    tc_mm<kBTC>(dA + kC * kD, kD, ST + kC * kD, kD, false, dS, kD, false, kC, kD, kD, 1.f, 0.f, mm);  // 64..127
    tc_mm<kBTC>(dQt, kD, dOf, kD, false, ST, kD, true, kC, kD, kD, p.scale, 0.f, mm);     // scale dO S_c
    tc_mm<kBTC>(dP, kC, dOf, kD, false, Up, kD, true, kC, kC, kD, p.scale, 0.f, mm);      // scale dO U'^T
    tc_mm<kBTC>(dUp, kD, P, kC, true, dOf, kD, false, kC, kD, kC, p.scale, 0.f, mm);      // scale P^T dO
    // ---- B = U'^T diag(e) K ----
    tc_mm<kBTC>(T1, kD, Up, kD, false, dS, kD, false, kC, kD, kD, 1.f, 0.f, mm);          // U' dB
    tc_mm<kBTC>(T2, kD, Kf, kD, false, dS, kD, true, kC, kD, kD, 1.f, 0.f, mm);           // K dB^T
#pragma unroll 8
    for (int i = tid; i < kMat; i += kBTC) {
      const int t = i >> 7;
      dK[i] = ee[t] * T1[i];
      dUp[i] += ee[t] * T2[i];
    }
    __syncthreads();
    row_dots<kBTC>(T1, Kf, kD, de);
    // ---- A = gamma_C I - W^T diag(e) K ----
    tc_mm<kBTC>(T1, kD, W, kD, false, dA, kD, false, kC, kD, kD, 1.f, 0.f, mm);           // W dA
    tc_mm<kBTC>(T2, kD, Kf, kD, false, dA, kD, true, kC, kD, kD, 1.f, 0.f, mm);           // K dA^T
#pragma unroll 8
    for (int i = tid; i < kMat; i += kBTC) {
      const int t = i >> 7;
      dK[i] -= ee[t] * T1[i];
      dW[i] = -ee[t] * T2[i];
      dQ[i] = gam[t] * dQt[i];  // Qt = diag(gamma) Q - P W: the gamma Q part
    }
    if (tid < 32) {  // d gamma_C: the trace of dA
      float tr = dA[(4 * tid) * (kD + 1)] + dA[(4 * tid + 1) * (kD + 1)] + dA[(4 * tid + 2) * (kD + 1)] +
                 dA[(4 * tid + 3) * (kD + 1)];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) tr += __shfl_xor_sync(0xffffffffu, tr, o);
      if (tid == 0) red[0] = tr;
    }
    __syncthreads();
    row_dots<kBTC>(T1, Kf, kD, tmp);
    row_dots<kBTC>(dQt, Qf, kD, dgam);
    if (tid < kC) de[tid] -= tmp[tid];
    __syncthreads();
    // ---- Qt = diag(gamma) Q - P W ----
    tc_mm<kBTC>(dP, kC, dQt, kD, false, W, kD, true, kC, kC, kD, -1.f, 1.f, mm);          // dP -= dQt W^T
    tc_mm<kBTC>(dW, kD, P, kC, true, dQt, kD, false, kC, kD, kC, -1.f, 1.f, mm);          // dW -= P^T dQt
    // ---- P = tril(D o Q K^T) ----
#pragma unroll 4
    for (int i = tid; i < kSq; i += kBTC) {
      const int r = i >> 6, cc = i & 63;
      const float dpm = cc <= r ? dP[i] : 0.f;
      dD[i] = dpm * QK[i];
      S1[i] = dpm * Dm[i];  // dQK
    }
    __syncthreads();
    tc_mm<kBTC>(dQ, kD, S1, kC, false, Kf, kD, false, kC, kD, kC, 1.f, 1.f, mm);          // dQ += dQK K
    tc_mm<kBTC>(dK, kD, S1, kC, true, Qf, kD, false, kC, kD, kC, 1.f, 1.f, mm);           // dK += dQK^T Q
    // ---- W = T diag(beta gamma) K, U' = T diag(beta) V ----
    tc_mm<kBTC>(dTm, kC, dW, kD, false, RW, kD, true, kC, kC, kD, 1.f, 0.f, mm);          // dW RW^T
    tc_mm<kBTC>(dTm, kC, dUp, kD, false, RU, kD, true, kC, kC, kD, 1.f, 1.f, mm);         // + dUp RU^T
    tc_mm<kBTC>(T1, kD, Tm, kC, true, dW, kD, false, kC, kD, kC, 1.f, 0.f, mm);           // dRW = T^T dW
    tc_mm<kBTC>(T2, kD, Tm, kC, true, dUp, kD, false, kC, kD, kC, 1.f, 0.f, mm);          // dRU = T^T dU'
#pragma unroll 8
    for (int i = tid; i < kMat; i += kBTC) {
      const int t = i >> 7;
      dK[i] += bb[t] * gam[t] * T1[i];
      dV[i] = bb[t] * T2[i];
    }
    __syncthreads();
    row_dots<kBTC>(T1, Kf, kD, tmp);
    row_dots<kBTC>(T2, Vf, kD, tmp2);
    if (tid < kC) {
      dbeta[tid] = gam[tid] * tmp[tid] + tmp2[tid];
      dgam[tid] += bb[tid] * tmp[tid];
    }
    __syncthreads();
    // ---- T = (I + A_in)^-1: dA_in = strict_tril(-T^T dT T^T) ----
    tc_mm<kBTC>(S1, kC, Tm, kC, true, dTm, kC, false, kC, kC, kC, 1.f, 0.f, mm);          // T^T dT
    tc_mm<kBTC>(S2, kC, S1, kC, false, Tm, kC, true, kC, kC, kC, -1.f, 0.f, mm);          // -(T^T dT) T^T
    // ---- A_in = strict_tril(beta_i D_ij K K^T_ij) ----
#pragma unroll 4
    for (int i = tid; i < kSq; i += kBTC) {
      const int r = i >> 6, cc = i & 63;
      const float dain = cc < r ? S2[i] : 0.f;
      S1[i] = bb[r] * dain * Dm[i];  // dKK
      dD[i] += bb[r] * dain * KK[i];
      S2[i] = dain * Dm[i] * KK[i];  // for d beta
    }
    __syncthreads();
    row_dots<kBTC>(S2, nullptr, kC, tmp);
    if (tid < kC) dbeta[tid] += tmp[tid];
    tc_mm<kBTC>(dK, kD, S1, kC, false, Kf, kD, false, kC, kD, kC, 1.f, 1.f, mm);          // dK += dKK K
    tc_mm<kBTC>(dK, kD, S1, kC, true, Kf, kD, false, kC, kD, kC, 1.f, 1.f, mm);           // dK += dKK^T K
    // ---- D_ij = exp(G_i - G_j), gamma = exp(G), e = exp(G_C - G), gamma_C = exp(G_C), G = cumsum(g) ----
    row_dots<kBTC>(dD, Dm, kC, tmp);  // row sums of dD o D
    if (tid < kC) {
      float cs = 0.f;  // column sums
#pragma unroll 16
      for (int j = 0; j < kC; ++j) cs += dD[j * kC + tid] * Dm[j * kC + tid];
      dG[tid] = tmp[tid] - cs + dgam[tid] * gam[tid] - de[tid] * ee[tid];
    }
    __syncthreads();
    if (tid == 0) {
      float s = 0.f;
      for (int j = 0; j < kC; ++j) s += de[j] * ee[j];
      dG[kC - 1] += s + red[0] * expf(G[kC - 1]);
      float run = 0.f;  // dg_t = sum_{u >= t} dG_u
      for (int t = kC - 1; t >= 0; --t) {
        run += dG[t];
        dG[t] = run;
      }
    }
    __syncthreads();
    // ---- outputs (the q/k gradients of the value heads sharing a q/k head accumulate) ----
#pragma unroll 4
    for (int i4 = tid; i4 < nv * kD / 4; i4 += kBTC) {
      const int t = i4 >> 5, j = (i4 & 31) * 4;
      const size_t rq = (((size_t)b * p.T + t0 + t) * p.H_qk + qh) * kD + j;
      atomicAdd(reinterpret_cast<float4 *>(p.dq + rq), reinterpret_cast<const float4 *>(dQ)[i4]);
      atomicAdd(reinterpret_cast<float4 *>(p.dk + rq), reinterpret_cast<const float4 *>(dK)[i4]);
      *reinterpret_cast<float4 *>(p.dv + (((size_t)b * p.T + t0 + t) * p.H_v + h) * kD + j) =
          reinterpret_cast<const float4 *>(dV)[i4];
    }
    if (tid < nv) {
      const size_t idx = ((size_t)b * p.T + t0 + tid) * p.H_v + h;
      p.dg[idx] = dG[tid];
      p.dbeta[idx] = dbeta[tid];
    }
    __syncthreads();
  }
  tc_mm_end(mm);
}

}  // namespace

size_t gdn_bwd_chunk_ctas(int B, int T, int H_v) {
  const size_t n_chunks = ((size_t)T + kC - 1) / kC;
  const size_t items = (size_t)B * H_v * n_chunks;
  return items < 296 ? items : 296;
}

size_t gdn_bwd_workspace_bytes(int B, int T, int H_v) {
  const size_t n_chunks = ((size_t)T + kC - 1) / kC;
  const size_t heads = (size_t)B * H_v;
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  return al(gdn_workspace_bytes(B, T, H_v)) + al((size_t)B * T * H_v * kD * 2) +       // records, forward o
         3 * al(heads * n_chunks * kD * kD * 4) +                                        // chunk states, dS, At
         al(gdn_bwd_chunk_ctas(B, T, H_v) * kChunkScratch * 4);
}

cudaError_t launch_gdn_bwd(const GdnBwdArgs &a, cudaStream_t s) {
  const int n_chunks = (a.T + kC - 1) / kC;
  const size_t heads = (size_t)a.B * a.H_v;
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  uint8_t *w = reinterpret_cast<uint8_t *>(a.workspace);
  uint8_t *rec = w;
  w += al(gdn_workspace_bytes(a.B, a.T, a.H_v));
  bf16_t *o_fwd = reinterpret_cast<bf16_t *>(w);
  w += al((size_t)a.B * a.T * a.H_v * kD * 2);
  float *states = reinterpret_cast<float *>(w);
  w += al(heads * n_chunks * kD * kD * 4);
  float *dS = reinterpret_cast<float *>(w);
  w += al(heads * n_chunks * kD * kD * 4);
  float *At = reinterpret_cast<float *>(w);
  w += al(heads * n_chunks * kD * kD * 4);
  float *chunk_scratch = reinterpret_cast<float *>(w);

  // 1. the forward pass, keeping every chunk's start state
  GdnChunkArgs f;
  memset(&f, 0, sizeof(f));
  f.q = a.q;
  f.k = a.k;
  f.v = a.v;
  f.g = a.g;
  f.beta = a.beta;
  f.state_in = a.state_in;
  f.o = o_fwd;
  f.B = a.B;
  f.T = a.T;
  f.n_heads = a.H_v;
  f.group = a.H_v / a.H_qk;
  f.qk_heads = a.H_qk;
  f.v_heads = a.H_v;
  f.scale = a.scale;
  f.workspace = rec;
  f.chunk_states = states;
  cudaError_t e = launch_gdn_chunk(f, s);
  if (e != cudaSuccess) return e;
  // the record layout of gdn_chunk.cu: -W_e^T | U'^T | P | Qt^T | factors
  const size_t nrec = heads * n_chunks;
  BwdParams p;
  memset(&p, 0, sizeof(p));
  p.q = a.q;
  p.k = a.k;
  p.v = a.v;
  p.dO = a.dO;
  p.g = a.g;
  p.beta = a.beta;
  p.dS_T = a.dS_T;
  p.chunk_states = states;
  p.rec_w = reinterpret_cast<const bf16_t *>(rec);
  p.rec_q = reinterpret_cast<const bf16_t *>(rec + nrec * (2 * kD * kC * 2 + kC * kC * 2));
  p.rec_f = reinterpret_cast<const float *>(rec + nrec * (3 * kD * kC * 2 + kC * kC * 2));
  p.dS = dS;
  p.dq = a.dq;
  p.dk = a.dk;
  p.dv = a.dv;
  p.dg = a.dg;
  p.dbeta = a.dbeta;
  p.dS0 = a.dS0;
  p.At = At;
  p.chunk_scratch = chunk_scratch;
  p.B = a.B;
  p.T = a.T;
  p.H_qk = a.H_qk;
  p.H_v = a.H_v;
  p.group = a.H_v / a.H_qk;
  p.n_chunks = n_chunks;
  p.n_items = (int)nrec;
  p.scale = a.scale;
  // 2. the reverse scan of the state's cotangent
  p.status = device_status_ptr();
  if ((e = cudaFuncSetAttribute(gdn_bwd_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kBwdDynSmem)) !=
          cudaSuccess ||
      (e = cudaFuncSetAttribute(gdn_bwd_maps_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kBwdDynSmem)) !=
          cudaSuccess ||
      (e = cudaFuncSetAttribute(gdn_bwd_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kBwdChunkSmem)) !=
          cudaSuccess)
    return e;
  int dev = 0, n_sm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  const size_t ctas = gdn_bwd_chunk_ctas(a.B, a.T, a.H_v);  // the per-CTA scratch is sized for this many
  const unsigned grid = (unsigned)(ctas < (size_t)n_sm ? ctas : (size_t)n_sm);
  gdn_bwd_maps_kernel<<<grid, kBT, kBwdDynSmem, s>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  gdn_bwd_scan_kernel<<<dim3(a.H_v, a.B, 2), kBT, kBwdDynSmem, s>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // 3. the per-chunk pullback; q and k gradients accumulate over the value heads of a q/k head
  if ((e = cudaMemsetAsync(a.dq, 0, (size_t)a.B * a.T * a.H_qk * kD * 4, s)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(a.dk, 0, (size_t)a.B * a.T * a.H_qk * kD * 4, s)) != cudaSuccess) return e;
  gdn_bwd_chunk_kernel<<<(unsigned)(ctas < 2 * (size_t)n_sm ? ctas : 2 * (size_t)n_sm), kBTC, kBwdChunkSmem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace hh
