// attn_fwd.cu -- causal grouped-query softmax attention over a sequence
// (prefill), with the optional sigmoid output gate and the optional per-head
// RMS fusion used by the head-level hybrid layer: the dispatch to the kernels.
//
// The attention layers of the hybrid stack are ordinary softmax attention with
// 24 query heads over 4 key/value heads at head dim 256 ("The Hybrid Attention
// in Qwen3.8-27B", "Grouped-query attention multiplies on top of that"); in the
// HydraHead layer the FA heads are softmax heads of head dim 128 with their own
// K/V ("HydraHead ...", abstract).  The pages print no kernel; both kernels are
// flash attention (online softmax, no T x T matrix in memory):
//   o_t = sum_{j<=t} exp(s_tj - m_t) v_j / sum_{j<=t} exp(s_tj - m_t),
//   s_tj = scale q_t . k_j,  then o_t *= sigmoid(G_t) when a gate is given.
#include "internal.h"

namespace hh {

cudaError_t launch_attn_fwd(const AttnFwdArgs &a, cudaStream_t s) {
  if (a.B == 0 || a.T == 0 || a.n_heads == 0) return cudaSuccess;
  // d = 256: CTA pairs, M = 256 across two SMs, each CTA streaming half of every K/V tile
  // (attn_fwd_tc2.cu).  d = 128: one CTA per 128 query rows with two softmax groups taking
  // the key tiles in turn (attn_fwd_tc.cu); there a tile is half the MMA work, and the
  // pair's cross-CTA handshakes did not pay for themselves.
  return a.d == 256 ? launch_attn_fwd_pair(a, s) : launch_attn_fwd_tc(a, s);
}

}  // namespace hh
