// gdn_decode.cu -- one decode token of the gated delta rule per sequence.
//
// The linear-attention layers carry a state whose size does not depend on the
// sequence length ("The Hybrid Attention in Qwen3.8-27B", section "Why 27B
// parameters can carry 262K tokens"; "The economics of hybrid attention",
// TL;DR: about 150 MiB per sequence).  A decode step therefore streams every state
// once: per value head, S (d_v x d_k fp32, 64 KiB) is read and written once.
//
// Per row j of S (rows evolve independently) with a = exp(g):
//   r_j = S_j . k,  p_j = S_j . q
//   u_j = beta (v_j - a r_j)
//   S_j <- a S_j + u_j k^T                  (== a S (I - beta k k^T) + beta v k^T, row j)
//   o_j = scale (a p_j + u_j (k . q))       (== scale * S_new q, row j)
//
// Layout: one warp owns 4 rows; lane l holds columns 4l..4l+3 of each row
// (one 16-byte streaming load / store per row per lane, fully coalesced).
// A CTA of 8 warps covers 32 rows; 4 CTAs cover one 128 x 128 state.
// HBM roofline: 2 x 64 KiB of state per (sequence, value head) plus small
// vectors; nothing is re-read.
#include "common.cuh"
#include "internal.h"

namespace hh {

namespace {

constexpr int kD = 128;
constexpr int kRowsPerWarp = 4;
constexpr int kWarps = 8;
constexpr int kRowsPerCta = kRowsPerWarp * kWarps;  // 32
constexpr int kCtasPerState = kD / kRowsPerCta;      // 4

__global__ void __launch_bounds__(kWarps * 32) gdn_decode_kernel(GdnDecodeArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x / kCtasPerState;  // b * H_v + h
  const int row0 = (blockIdx.x % kCtasPerState) * kRowsPerCta + warp * kRowsPerWarp;
  const int b = bh / a.H_v, h = bh - b * a.H_v;
  const int hq = h / (a.H_v / a.H_qk);

  float *S = a.state + (size_t)bh * kD * kD;
  // issue the state loads first: they are the HBM traffic
  float4 s[kRowsPerWarp];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r)
    s[r] = __ldcs(reinterpret_cast<const float4 *>(S + (size_t)(row0 + r) * kD) + lane);

  const size_t qk_off = ((size_t)b * a.H_qk + hq) * kD + lane * 4;
  const uint2 kk = *reinterpret_cast<const uint2 *>(a.k + qk_off);
  const uint2 qq = *reinterpret_cast<const uint2 *>(a.q + qk_off);
  const float kf[4] = {bf16_lo(kk.x), bf16_hi(kk.x), bf16_lo(kk.y), bf16_hi(kk.y)};
  const float qf[4] = {bf16_lo(qq.x), bf16_hi(qq.x), bf16_lo(qq.y), bf16_hi(qq.y)};
  const float decay = expf(a.g[bh]);
  const float beta = a.beta[bh];
  const float kdotq = warp_sum(kf[0] * qf[0] + kf[1] * qf[1] + kf[2] * qf[2] + kf[3] * qf[3]);

  float vrow[kRowsPerWarp];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) vrow[r] = bf16_to_f(a.v[(size_t)bh * kD + row0 + r]);

#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const float rk = warp_sum(s[r].x * kf[0] + s[r].y * kf[1] + s[r].z * kf[2] + s[r].w * kf[3]);
    const float rq = warp_sum(s[r].x * qf[0] + s[r].y * qf[1] + s[r].z * qf[2] + s[r].w * qf[3]);
    const float u = beta * (vrow[r] - decay * rk);
    float4 n;
    n.x = fmaf(decay, s[r].x, u * kf[0]);
    n.y = fmaf(decay, s[r].y, u * kf[1]);
    n.z = fmaf(decay, s[r].z, u * kf[2]);
    n.w = fmaf(decay, s[r].w, u * kf[3]);
    __stcs(reinterpret_cast<float4 *>(S + (size_t)(row0 + r) * kD) + lane, n);
    if (lane == r) a.o[(size_t)bh * kD + row0 + r] = f_to_bf16(a.scale * fmaf(decay, rq, u * kdotq));
  }
}

}  // namespace

cudaError_t launch_gdn_decode(const GdnDecodeArgs &a, cudaStream_t s) {
  const long long blocks = (long long)a.B * a.H_v * kCtasPerState;
  if (blocks == 0) return cudaSuccess;
  gdn_decode_kernel<<<(unsigned)blocks, kWarps * 32, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace hh
