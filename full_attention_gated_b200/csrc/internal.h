// internal.h -- launchers behind the C ABI (host side).  Not part of the
// public interface; abi.cpp validates arguments before calling these.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace hh {

typedef uint16_t bf16_t;

constexpr int kMaxMappedHeads = 64;

// Gated delta rule over a sequence.  Head i of the launch (0 <= i < n_heads)
// reads value/decay/state/output head vh(i) and q/k head qh(i):
//   use_map ? (map[i], map[i]) : (i, i / group).
// Tensors are indexed with their own head counts (qk_heads, v_heads).
struct GdnChunkArgs {
  const bf16_t *q, *k, *v;
  const float *g, *beta;
  const float *state_in;  // nullable
  float *state_out;       // nullable
  bf16_t *o;
  int B, T, n_heads, group, qk_heads, v_heads;
  int use_map;
  int map[kMaxMappedHeads];
  float scale;
  int rms;  // 1: o rows are RMS-normalised (head fusion), 0: plain outputs
  float eps;
  void *workspace;  // gdn_workspace_bytes(B, T, n_heads) bytes, 256-byte aligned
  float *chunk_states;  // nullable: S^T at the start of every chunk, [B, n_heads, n_chunks, d_k, d_v] fp32
};
size_t gdn_workspace_bytes(int B, int T, int n_heads);
cudaError_t launch_gdn_chunk(const GdnChunkArgs &a, cudaStream_t s);

// Gradients of the gated delta rule (the backward pass of gdn_chunk_fwd), fp32 outputs.
struct GdnBwdArgs {
  const bf16_t *q, *k, *v, *dO;
  const float *g, *beta;
  const float *state_in;  // nullable (zeros)
  const float *dS_T;      // nullable (zero cotangent of the final state)
  float *dq, *dk, *dv, *dg, *dbeta;
  float *dS0;             // nullable
  int B, T, H_qk, H_v;
  float scale;
  void *workspace;        // gdn_bwd_workspace_bytes(B, T, H_v) bytes, 256-byte aligned
};
size_t gdn_bwd_workspace_bytes(int B, int T, int H_v);
cudaError_t launch_gdn_bwd(const GdnBwdArgs &a, cudaStream_t s);

struct GdnDecodeArgs {
  const bf16_t *q, *k, *v;
  const float *g, *beta;
  float *state;
  bf16_t *o;
  int B, H_qk, H_v;
  float scale;
};
cudaError_t launch_gdn_decode(const GdnDecodeArgs &a, cudaStream_t s);

// Softmax attention prefill.  Head i of the launch reads q/gate/o head qh(i)
// and k/v head kh(i):  use_map ? (map[i], map[i]) : (i, i / group).
struct AttnFwdArgs {
  const bf16_t *q, *k, *v, *gate;  // gate nullable
  bf16_t *o;
  int B, T, n_heads, group, q_heads, kv_heads, d;
  int use_map;
  int map[kMaxMappedHeads];
  float scale;
  int causal;
  int rms;
  float eps;
};
cudaError_t launch_attn_fwd(const AttnFwdArgs &a, cudaStream_t s);
// tcgen05 / TMEM implementation (attn_fwd_tc.cu)
cudaError_t launch_attn_fwd_tc(const AttnFwdArgs &a, cudaStream_t s);
// CTA-pair (cta_group::2, M = 256) implementation (attn_fwd_tc2.cu)
cudaError_t launch_attn_fwd_pair(const AttnFwdArgs &a, cudaStream_t s);

struct AttnDecodeArgs {
  const bf16_t *q, *k_cache, *v_cache, *gate;
  const int32_t *cache_len;
  bf16_t *o;
  void *workspace;
  int B, T_cache, H_q, H_kv, d;
  float scale;
};
// GQA decode over a q8_0 cache: int8 values [B, T_cache, H_kv, d] and fp16 scales
// [B, T_cache, H_kv, d/32] (one per 32 consecutive elements), for K and for V.
struct AttnDecodeQ8Args {
  const bf16_t *q, *gate;
  const int8_t *k_values, *v_values;
  const uint16_t *k_scales, *v_scales;
  const int32_t *cache_len;
  bf16_t *o;
  void *workspace;
  int B, T_cache, H_q, H_kv, d;
  float scale;
};
cudaError_t launch_attn_decode_q8(const AttnDecodeQ8Args &a, cudaStream_t s);
int attn_decode_splits(int B, int T_cache);
size_t attn_decode_workspace(int B, int H_q, int d, int T_cache);
cudaError_t launch_attn_decode(const AttnDecodeArgs &a, cudaStream_t s);

// PHBA prefix states: the gated slot memory (M = 128 slots, d = 128) before every block of C tokens.
struct PhbaStatesArgs {
  const bf16_t *k_raw, *v;   // [B, T, H, 128]
  const float *alpha;        // [B, T, H, 128]
  bf16_t *kstate, *vstate;   // [B, H, nb, 128, 128]
  int B, T, H, C;
  void *workspace;           // phba_states_workspace_bytes(B, T, H, C) bytes, 256-byte aligned
};
size_t phba_states_workspace_bytes(int B, int T, int H, int C);
cudaError_t launch_phba_states(const PhbaStatesArgs &a, cudaStream_t s);
// PHBA routing and attention over tokens and prefix-state slots.
struct PhbaFwdArgs {
  const bf16_t *q_rope, *k_rope, *q_raw, *v;  // [B, T, H, 128]
  const bf16_t *kstate, *vstate;              // [B, H, nb, 128, 128]
  bf16_t *o;                                  // [B, T, H, 128]
  int32_t *sel;                               // nullable: [B, T, H, K] kept blocks, ascending, -1 after
  int B, T, H, C, K;
  float scale;
  void *workspace;                            // phba_fwd_workspace_bytes(B, T, H, C, K), 256-byte aligned
};
size_t phba_fwd_workspace_bytes(int B, int T, int H, int C, int K);
cudaError_t launch_phba_fwd(const PhbaFwdArgs &a, cudaStream_t s);
// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
// dims/strides: dims[0] innermost; strides[i] is the byte stride of dim i+1.
CUresult encode_tmap(CUtensorMap *map, CUtensorMapDataType dtype, int rank, const void *base,
                     const uint64_t *dims, const uint64_t *strides_bytes, const uint32_t *box,
                     CUtensorMapSwizzle swizzle);

// Shared argument checks of the C entry points (abi.cpp).  Each returns HH_OK, or a
// negative status with the error message set; check_decode_args returns kNothingToDo
// for a valid call with B = 0.
constexpr int kNothingToDo = 1;
int check_device(const char *fn);
int check_decode_args(const char *fn, const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                      const int32_t *cache_len, const uint16_t *gate, const uint16_t *o, int B, int T_cache, int H_q,
                      int H_kv, int d, float scale);

void set_error(const char *fmt, ...);
const char *last_error();
void clear_error();
// address of this device's status word (nullptr if it cannot be resolved)
unsigned *device_status_ptr();

}  // namespace hh
