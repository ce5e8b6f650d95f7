// abi.cpp -- the extern "C" entry points of libhh.so (declared in include/hh.h):
// argument validation, head routing for the hybrid layer, launch and error
// mapping.  Every check runs before anything is enqueued.
#include "../../include/hh.h"

#include <cuda_runtime.h>
#include <math.h>
#include <string.h>

#include <mutex>

#include "internal.h"

using namespace hh;

namespace {

// the delta-rule kernels index chunks with a grid dimension (at most 65535 chunks of 64 tokens)
constexpr long long kMaxGdnTokens = 64LL * 65535;

#define HH_FAIL(code, ...)    \
  do {                        \
    hh::set_error(__VA_ARGS__); \
    return (code);            \
  } while (0)

bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool al4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

int launch_result(cudaError_t e, const char *fn) {
  if (e != cudaSuccess) {
    if (!hh::last_error()[0]) hh::set_error("%s: CUDA error: %s", fn, cudaGetErrorString(e));
    return HH_ERR_CUDA;
  }
  return HH_OK;
}

// Library-owned side stream and events per device for the hybrid layer's
// fork/join (the softmax heads run on it beside the delta-rule heads).
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
int side_stream(SideStream **out) {
  static std::mutex mu;
  static SideStream per_dev[128];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) HH_FAIL(HH_ERR_CUDA, "no CUDA device");
  std::lock_guard<std::mutex> lock(mu);
  SideStream &ss = per_dev[dev];
  if (!ss.s) {
    if (cudaStreamCreateWithFlags(&ss.s, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming) != cudaSuccess)
      HH_FAIL(HH_ERR_CUDA, "hybrid_head_layer_fwd: could not create the side stream");
  }
  *out = &ss;
  return HH_OK;
}

}  // namespace

namespace hh {

// The kernels are built for sm_100a only; refuse other devices up front.
int check_device(const char *fn) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) HH_FAIL(HH_ERR_CUDA, "%s: no CUDA device (%s)", fn, cudaGetErrorString(e));
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0)
    HH_FAIL(HH_ERR_UNSUPPORTED, "%s: device %d is sm_%d%d; this library is built for sm_100a (B200)", fn, dev, major,
            minor);
  return HH_OK;
}

// Every check of a GQA decode call except its scratch (shared by gqa_attn_decode and
// gqa_attn_decode_noalloc, so that the two entry points accept exactly the same calls).
int check_decode_args(const char *fn, const hh_bf16 *q, const hh_bf16 *k_cache, const hh_bf16 *v_cache,
                      const int32_t *cache_len, const hh_bf16 *gate, const hh_bf16 *o, int B, int T_cache, int H_q,
                      int H_kv, int d, float scale) {
  if (B < 0 || T_cache < 0 || H_q <= 0 || H_kv <= 0 || d <= 0)
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: sizes must be positive (B, T_cache may be 0)", fn);
  if (H_q % H_kv != 0) HH_FAIL(HH_ERR_INVALID_ARG, "%s: H_q (%d) must be a multiple of H_kv (%d)", fn, H_q, H_kv);
  if (H_q / H_kv > 16) HH_FAIL(HH_ERR_UNSUPPORTED, "%s: at most 16 query heads per kv head", fn);
  if (d != 128 && d != 256) HH_FAIL(HH_ERR_UNSUPPORTED, "%s: only d = 128 or 256 is built", fn);
  if (!isfinite(scale)) HH_FAIL(HH_ERR_INVALID_ARG, "%s: scale must be finite", fn);
  if (B > 65535 || H_kv > 65535 || (long long)T_cache > (1LL << 30))
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: sizes too large", fn);
  if (B == 0) return kNothingToDo;
  if (!q || !o || (T_cache > 0 && (!k_cache || !v_cache)))
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: null tensor pointer", fn);
  if (!al16(q) || !al16(o) || (gate && !al16(gate)) || (k_cache && !al16(k_cache)) || (v_cache && !al16(v_cache)) ||
      (cache_len && !al4(cache_len)))
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: tensors must be 16-byte aligned", fn);
  return HH_OK;
}

}  // namespace hh

extern "C" {

const char *hh_last_error(void) { return hh::last_error(); }

const char *hh_version(void) { return "libhh 0.1 (sm_100a)"; }

int hh_device_status(hh_stream stream) {
  hh::clear_error();
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) HH_FAIL(HH_ERR_CUDA, "hh_device_status: %s", cudaGetErrorString(e));
  unsigned *p = hh::device_status_ptr();
  if (!p) HH_FAIL(HH_ERR_CUDA, "hh_device_status: status word not resolvable");
  unsigned w = 0;
  if (cudaMemcpy(&w, p, sizeof(w), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemset(p, 0, sizeof(w)) != cudaSuccess)
    HH_FAIL(HH_ERR_CUDA, "hh_device_status: could not read the status word");
  if (w & 1u) HH_FAIL(HH_ERR_TIMEOUT, "a kernel's bounded wait expired; its outputs are incomplete");
  return HH_OK;
}

size_t gdn_chunk_fwd_workspace_size(int B, int T, int H_v, int d_v, int chunk) {
  if (B <= 0 || T <= 0 || H_v <= 0 || d_v != 128 || chunk != 64) return 0;
  return hh::gdn_workspace_bytes(B, T, H_v);
}

int gdn_chunk_fwd(const hh_bf16 *q, const hh_bf16 *k, const hh_bf16 *v, const float *g, const float *beta,
                  const float *state_in, float *state_out, hh_bf16 *o, void *workspace, size_t ws_bytes, int B, int T,
                  int H_qk, int H_v, int d_k, int d_v, float scale, int chunk, hh_stream stream) {
  static const char *fn = "gdn_chunk_fwd";
  hh::clear_error();
  if (B < 0 || T < 0 || H_qk <= 0 || H_v <= 0 || d_k <= 0 || d_v <= 0 || chunk <= 0)
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: sizes must be positive (B, T may be 0)", fn);
  if (H_v % H_qk != 0) HH_FAIL(HH_ERR_INVALID_ARG, "%s: H_v (%d) must be a multiple of H_qk (%d)", fn, H_v, H_qk);
  if (d_k != 128 || d_v != 128) HH_FAIL(HH_ERR_UNSUPPORTED, "%s: only d_k = d_v = 128 is built", fn);
  if (chunk != 64) HH_FAIL(HH_ERR_UNSUPPORTED, "%s: only chunk = 64 is built", fn);
  if (!isfinite(scale)) HH_FAIL(HH_ERR_INVALID_ARG, "%s: scale must be finite", fn);
  if ((long long)T * H_v > (1LL << 31) || (long long)B * H_v > 65535 || B > 65535 ||
      (long long)B * H_v * ((T + 63) / 64) * 128 >= (1LL << 31))
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: sizes too large", fn);
  if ((long long)T > kMaxGdnTokens) HH_FAIL(HH_ERR_UNSUPPORTED, "%s: T above %lld tokens", fn, kMaxGdnTokens);
  if (B > 0 && T > 0) {
    if (!q || !k || !v || !g || !beta || !o) HH_FAIL(HH_ERR_INVALID_ARG, "%s: null tensor pointer", fn);
    if (!al16(q) || !al16(k) || !al16(v) || !al16(o) || !al4(g) || !al4(beta))
      HH_FAIL(HH_ERR_INVALID_ARG, "%s: bf16 tensors must be 16-byte aligned, g/beta 4-byte aligned", fn);
    const size_t need = hh::gdn_workspace_bytes(B, T, H_v);
    if (!workspace || ws_bytes < need)
      HH_FAIL(HH_ERR_INVALID_ARG, "%s: workspace of %zu bytes needed (got %zu)", fn, need, ws_bytes);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
      HH_FAIL(HH_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", fn);
  }
  if ((state_in && !al16(state_in)) || (state_out && !al16(state_out)))
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: states must be 16-byte aligned", fn);
  if (B == 0) return HH_OK;
  if (int r = hh::check_device(fn)) return r;
  GdnChunkArgs a;
  memset(&a, 0, sizeof(a));
  a.q = q;
  a.k = k;
  a.v = v;
  a.g = g;
  a.beta = beta;
  a.state_in = state_in;
  a.state_out = state_out;
  a.o = o;
  a.B = B;
  a.T = T;
  a.n_heads = H_v;
  a.group = H_v / H_qk;
  a.qk_heads = H_qk;
  a.v_heads = H_v;
  a.scale = scale;
  a.workspace = workspace;
  return launch_result(launch_gdn_chunk(a, reinterpret_cast<cudaStream_t>(stream)), fn);
}

size_t gdn_chunk_bwd_workspace_size(int B, int T, int H_v, int d_v, int chunk) {
  if (B <= 0 || T <= 0 || H_v <= 0 || d_v != 128 || chunk != 64) return 0;
  return hh::gdn_bwd_workspace_bytes(B, T, H_v);
}

int gdn_chunk_bwd(const hh_bf16 *q, const hh_bf16 *k, const hh_bf16 *v, const float *g, const float *beta,
                  const float *state_in, const hh_bf16 *dO, const float *dstate_out, float *dq, float *dk, float *dv,
                  float *dg, float *dbeta, float *dstate_in, void *workspace, size_t ws_bytes, int B, int T, int H_qk,
                  int H_v, int d_k, int d_v, float scale, int chunk, hh_stream stream) {
  static const char *fn = "gdn_chunk_bwd";
  hh::clear_error();
  if (B < 0 || T < 0 || H_qk <= 0 || H_v <= 0 || d_k <= 0 || d_v <= 0 || chunk <= 0)
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: sizes must be positive (B, T may be 0)", fn);
  if (H_v % H_qk != 0) HH_FAIL(HH_ERR_INVALID_ARG, "%s: H_v (%d) must be a multiple of H_qk (%d)", fn, H_v, H_qk);
  if (d_k != 128 || d_v != 128) HH_FAIL(HH_ERR_UNSUPPORTED, "%s: only d_k = d_v = 128 is built", fn);
  if (chunk != 64) HH_FAIL(HH_ERR_UNSUPPORTED, "%s: only chunk = 64 is built", fn);
  if (!isfinite(scale)) HH_FAIL(HH_ERR_INVALID_ARG, "%s: scale must be finite", fn);
  if ((long long)T * H_v > (1LL << 31) || (long long)B * H_v > 65535 || B > 65535 ||
      (long long)B * H_v * ((T + 63) / 64) * 128 >= (1LL << 31))
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: sizes too large", fn);
  if ((long long)T > kMaxGdnTokens) HH_FAIL(HH_ERR_UNSUPPORTED, "%s: T above %lld tokens", fn, kMaxGdnTokens);
  if (B == 0) return HH_OK;
  if (T == 0) HH_FAIL(HH_ERR_UNSUPPORTED, "%s: T = 0 (the gradient is dS0 = dS_T; nothing to run)", fn);
  if (!q || !k || !v || !g || !beta || !dO || !dq || !dk || !dv || !dg || !dbeta)
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: null tensor pointer", fn);
  if (!al16(q) || !al16(k) || !al16(v) || !al16(dO) || !al16(dq) || !al16(dk) || !al16(dv) || !al4(g) || !al4(beta) ||
      !al4(dg) || !al4(dbeta))
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: tensors must be 16-byte aligned (g, beta and their gradients 4-byte)", fn);
  if ((state_in && !al16(state_in)) || (dstate_out && !al16(dstate_out)) || (dstate_in && !al16(dstate_in)))
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: states must be 16-byte aligned", fn);
  const size_t need = hh::gdn_bwd_workspace_bytes(B, T, H_v);
  if (!workspace || ws_bytes < need)
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: workspace of %zu bytes needed (got %zu)", fn, need, ws_bytes);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", fn);
  if (int r = hh::check_device(fn)) return r;
  GdnBwdArgs a;
  memset(&a, 0, sizeof(a));
  a.q = q;
  a.k = k;
  a.v = v;
  a.dO = dO;
  a.g = g;
  a.beta = beta;
  a.state_in = state_in;
  a.dS_T = dstate_out;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.dg = dg;
  a.dbeta = dbeta;
  a.dS0 = dstate_in;
  a.B = B;
  a.T = T;
  a.H_qk = H_qk;
  a.H_v = H_v;
  a.scale = scale;
  a.workspace = workspace;
  return launch_result(launch_gdn_bwd(a, reinterpret_cast<cudaStream_t>(stream)), fn);
}

int gdn_decode_step(const hh_bf16 *q, const hh_bf16 *k, const hh_bf16 *v, const float *g, const float *beta,
                    float *state, hh_bf16 *o, int B, int H_qk, int H_v, int d_k, int d_v, float scale,
                    hh_stream stream) {
  static const char *fn = "gdn_decode_step";
  hh::clear_error();
  if (B < 0 || H_qk <= 0 || H_v <= 0 || d_k <= 0 || d_v <= 0)
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: sizes must be positive (B may be 0)", fn);
  if (H_v % H_qk != 0) HH_FAIL(HH_ERR_INVALID_ARG, "%s: H_v (%d) must be a multiple of H_qk (%d)", fn, H_v, H_qk);
  if (d_k != 128 || d_v != 128) HH_FAIL(HH_ERR_UNSUPPORTED, "%s: only d_k = d_v = 128 is built", fn);
  if (!isfinite(scale)) HH_FAIL(HH_ERR_INVALID_ARG, "%s: scale must be finite", fn);
  if ((long long)B * H_v * 4 > (1LL << 31)) HH_FAIL(HH_ERR_INVALID_ARG, "%s: sizes too large", fn);
  if (B == 0) return HH_OK;
  if (!q || !k || !v || !g || !beta || !state || !o) HH_FAIL(HH_ERR_INVALID_ARG, "%s: null tensor pointer", fn);
  if (!al16(q) || !al16(k) || !al16(v) || !al16(o) || !al16(state) || !al4(g) || !al4(beta))
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: tensors must be 16-byte aligned (g/beta 4-byte)", fn);
  if (int r = hh::check_device(fn)) return r;
  GdnDecodeArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.g = g;
  a.beta = beta;
  a.state = state;
  a.o = o;
  a.B = B;
  a.H_qk = H_qk;
  a.H_v = H_v;
  a.scale = scale;
  return launch_result(launch_gdn_decode(a, reinterpret_cast<cudaStream_t>(stream)), fn);
}

int gqa_attn_fwd(const hh_bf16 *q, const hh_bf16 *k, const hh_bf16 *v, const hh_bf16 *gate, hh_bf16 *o, int B,
                 int T, int H_q, int H_kv, int d, float scale, int causal, hh_stream stream) {
  static const char *fn = "gqa_attn_fwd";
  hh::clear_error();
  if (B < 0 || T < 0 || H_q <= 0 || H_kv <= 0 || d <= 0)
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: sizes must be positive (B, T may be 0)", fn);
  if (H_q % H_kv != 0) HH_FAIL(HH_ERR_INVALID_ARG, "%s: H_q (%d) must be a multiple of H_kv (%d)", fn, H_q, H_kv);
  if (d != 128 && d != 256) HH_FAIL(HH_ERR_UNSUPPORTED, "%s: only d = 128 or 256 is built", fn);
  if (causal != 0 && causal != 1) HH_FAIL(HH_ERR_INVALID_ARG, "%s: causal must be 0 or 1", fn);
  if (!isfinite(scale)) HH_FAIL(HH_ERR_INVALID_ARG, "%s: scale must be finite", fn);
  if (H_q > 65535 || B > 65535 || (long long)T > (1LL << 30))
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: sizes too large", fn);
  if (B == 0 || T == 0) return HH_OK;
  if (!q || !k || !v || !o) HH_FAIL(HH_ERR_INVALID_ARG, "%s: null tensor pointer", fn);
  if (!al16(q) || !al16(k) || !al16(v) || !al16(o) || (gate && !al16(gate)))
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: tensors must be 16-byte aligned", fn);
  if (int r = hh::check_device(fn)) return r;
  AttnFwdArgs a;
  memset(&a, 0, sizeof(a));
  a.q = q;
  a.k = k;
  a.v = v;
  a.gate = gate;
  a.o = o;
  a.B = B;
  a.T = T;
  a.n_heads = H_q;
  a.group = H_q / H_kv;
  a.q_heads = H_q;
  a.kv_heads = H_kv;
  a.d = d;
  a.scale = scale;
  a.causal = causal;
  return launch_result(launch_attn_fwd(a, reinterpret_cast<cudaStream_t>(stream)), fn);
}

size_t gqa_attn_decode_workspace_size(int B, int H_q, int d, int T_cache) {
  if (B <= 0 || H_q <= 0 || d <= 0 || T_cache < 0) return 0;
  return hh::attn_decode_workspace(B, H_q, d, T_cache);
}

int gqa_attn_decode(const hh_bf16 *q, const hh_bf16 *k_cache, const hh_bf16 *v_cache, const int32_t *cache_len,
                    const hh_bf16 *gate, hh_bf16 *o, void *workspace, size_t ws_bytes, int B, int T_cache, int H_q,
                    int H_kv, int d, float scale, hh_stream stream) {
  static const char *fn = "gqa_attn_decode";
  hh::clear_error();
  const int v = hh::check_decode_args(fn, q, k_cache, v_cache, cache_len, gate, o, B, T_cache, H_q, H_kv, d, scale);
  if (v < 0) return v;
  if (v == hh::kNothingToDo) return HH_OK;
  const size_t need = hh::attn_decode_workspace(B, H_q, d, T_cache);
  if (!workspace || ws_bytes < need)
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: workspace of %zu bytes needed (got %zu)", fn, need, ws_bytes);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", fn);
  if (int r = hh::check_device(fn)) return r;
  AttnDecodeArgs a;
  a.q = q;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.gate = gate;
  a.cache_len = cache_len;
  a.o = o;
  a.workspace = workspace;
  a.B = B;
  a.T_cache = T_cache;
  a.H_q = H_q;
  a.H_kv = H_kv;
  a.d = d;
  a.scale = scale;
  return launch_result(launch_attn_decode(a, reinterpret_cast<cudaStream_t>(stream)), fn);
}

int gqa_attn_decode_q8_0(const hh_bf16 *q, const int8_t *k_values, const uint16_t *k_scales, const int8_t *v_values,
                         const uint16_t *v_scales, const int32_t *cache_len, const hh_bf16 *gate, hh_bf16 *o,
                         void *workspace, size_t ws_bytes, int B, int T_cache, int H_q, int H_kv, int d, float scale,
                         hh_stream stream) {
  static const char *fn = "gqa_attn_decode_q8_0";
  hh::clear_error();
  const int v = hh::check_decode_args(fn, q, reinterpret_cast<const hh_bf16 *>(k_values),
                                      reinterpret_cast<const hh_bf16 *>(v_values), cache_len, gate, o, B, T_cache, H_q,
                                      H_kv, d, scale);
  if (v < 0) return v;
  if (d != 256) HH_FAIL(HH_ERR_UNSUPPORTED, "%s: only d = 256 is built for the q8_0 cache", fn);
  if (v == hh::kNothingToDo) return HH_OK;
  if (T_cache > 0 && (!k_scales || !v_scales)) HH_FAIL(HH_ERR_INVALID_ARG, "%s: null scale pointer", fn);
  if ((k_scales && !al16(k_scales)) || (v_scales && !al16(v_scales)))
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: scale arrays must be 16-byte aligned", fn);
  const size_t need = hh::attn_decode_workspace(B, H_q, d, T_cache);
  if (!workspace || ws_bytes < need)
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: workspace of %zu bytes needed (got %zu)", fn, need, ws_bytes);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", fn);
  if (int r = hh::check_device(fn)) return r;
  AttnDecodeQ8Args a;
  a.q = q;
  a.gate = gate;
  a.k_values = k_values;
  a.v_values = v_values;
  a.k_scales = k_scales;
  a.v_scales = v_scales;
  a.cache_len = cache_len;
  a.o = o;
  a.workspace = workspace;
  a.B = B;
  a.T_cache = T_cache;
  a.H_q = H_q;
  a.H_kv = H_kv;
  a.d = d;
  a.scale = scale;
  return launch_result(launch_attn_decode_q8(a, reinterpret_cast<cudaStream_t>(stream)), fn);
}

size_t hybrid_head_layer_workspace_size(int B, int T, int H, int d) {
  if (B <= 0 || T <= 0 || H <= 0 || d != 128) return 0;
  return hh::gdn_workspace_bytes(B, T, H);  // the delta-rule heads' scratch (upper bound: every head)
}

int hybrid_head_layer_fwd(const hh_bf16 *q, const hh_bf16 *k, const hh_bf16 *v, const float *g, const float *beta,
                          const uint8_t *head_is_fa, const float *state_in, float *state_out, hh_bf16 *out,
                          void *workspace, size_t ws_bytes, int B, int T, int H, int d, float scale_la, float scale_fa,
                          float eps, int chunk, hh_stream stream) {
  static const char *fn = "hybrid_head_layer_fwd";
  hh::clear_error();
  if (B < 0 || T < 0 || H <= 0 || d <= 0 || chunk <= 0)
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: sizes must be positive (B, T may be 0)", fn);
  if (H > kMaxMappedHeads) HH_FAIL(HH_ERR_UNSUPPORTED, "%s: at most %d heads", fn, kMaxMappedHeads);
  if (d != 128) HH_FAIL(HH_ERR_UNSUPPORTED, "%s: only d = 128 is built", fn);
  if (chunk != 64) HH_FAIL(HH_ERR_UNSUPPORTED, "%s: only chunk = 64 is built", fn);
  if (!head_is_fa) HH_FAIL(HH_ERR_INVALID_ARG, "%s: head_is_fa (host array) is null", fn);
  if (!isfinite(scale_la) || !isfinite(scale_fa) || !isfinite(eps) || eps < 0.f)
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: scales and eps must be finite, eps >= 0", fn);
  if ((long long)T > (1LL << 30) || B > 65535 || (long long)B * H * ((T + 63) / 64) * 128 >= (1LL << 31))
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: sizes too large", fn);
  if ((long long)T > kMaxGdnTokens) HH_FAIL(HH_ERR_UNSUPPORTED, "%s: T above %lld tokens", fn, kMaxGdnTokens);
  int la[kMaxMappedHeads], fa[kMaxMappedHeads], n_la = 0, n_fa = 0;
  for (int h = 0; h < H; ++h) {
    if (head_is_fa[h]) fa[n_fa++] = h;
    else la[n_la++] = h;
  }
  if (B > 0 && T > 0) {
    if (!q || !k || !v || !out) HH_FAIL(HH_ERR_INVALID_ARG, "%s: null tensor pointer", fn);
    if (n_la > 0 && (!g || !beta)) HH_FAIL(HH_ERR_INVALID_ARG, "%s: g/beta needed for LA heads", fn);
    if (!al16(q) || !al16(k) || !al16(v) || !al16(out) || (g && !al4(g)) || (beta && !al4(beta)))
      HH_FAIL(HH_ERR_INVALID_ARG, "%s: tensors must be 16-byte aligned (g/beta 4-byte)", fn);
    const size_t need = n_la ? hh::gdn_workspace_bytes(B, T, n_la) : 0;
    if (need && (!workspace || ws_bytes < need))
      HH_FAIL(HH_ERR_INVALID_ARG, "%s: workspace of %zu bytes needed (got %zu)", fn, need, ws_bytes);
    if (need && (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
      HH_FAIL(HH_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", fn);
  }
  if ((state_in && !al16(state_in)) || (state_out && !al16(state_out)))
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: states must be 16-byte aligned", fn);
  if (B == 0) return HH_OK;
  if (int r = hh::check_device(fn)) return r;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  GdnChunkArgs ga;
  memset(&ga, 0, sizeof(ga));
  ga.q = q;
  ga.k = k;
  ga.v = v;
  ga.g = g;
  ga.beta = beta;
  ga.state_in = state_in;
  ga.state_out = state_out;
  ga.o = out;  // [B, T, H*d] == [B, T, H, d]
  ga.B = B;
  ga.T = T;
  ga.n_heads = n_la;
  ga.group = 1;
  ga.qk_heads = H;
  ga.v_heads = H;
  ga.use_map = 1;
  memcpy(ga.map, la, sizeof(int) * n_la);
  ga.scale = scale_la;
  ga.rms = 1;
  ga.eps = eps;
  ga.workspace = workspace;

  AttnFwdArgs fa_args;
  memset(&fa_args, 0, sizeof(fa_args));
  fa_args.q = q;
  fa_args.k = k;
  fa_args.v = v;
  fa_args.o = out;
  fa_args.B = B;
  fa_args.T = T;
  fa_args.n_heads = n_fa;
  fa_args.group = 1;
  fa_args.q_heads = H;
  fa_args.kv_heads = H;
  fa_args.d = d;
  fa_args.use_map = 1;
  memcpy(fa_args.map, fa, sizeof(int) * n_fa);
  fa_args.scale = scale_fa;
  fa_args.causal = 1;
  fa_args.rms = 1;
  fa_args.eps = eps;

  if (n_la == 0 || n_fa == 0 || T == 0) {
    if (n_la) {
      if (int r = launch_result(launch_gdn_chunk(ga, s), fn)) return r;
    }
    if (n_fa && T > 0) return launch_result(launch_attn_fwd(fa_args, s), fn);
    return HH_OK;
  }
  // Fork: the delta-rule heads (few long sequential chains) are launched first, on the
  // caller's stream, so their CTAs are resident before the softmax heads, on the side
  // stream, fill the GPU.
  SideStream *ss = nullptr;
  if (int r = side_stream(&ss)) return r;
  if (cudaEventRecord(ss->fork, s) != cudaSuccess || cudaStreamWaitEvent(ss->s, ss->fork, 0) != cudaSuccess)
    HH_FAIL(HH_ERR_CUDA, "%s: fork failed", fn);
  if (int r = launch_result(launch_gdn_chunk(ga, s), fn)) return r;
  int r = launch_result(launch_attn_fwd(fa_args, ss->s), fn);
  if (cudaEventRecord(ss->join, ss->s) != cudaSuccess || cudaStreamWaitEvent(s, ss->join, 0) != cudaSuccess)
    HH_FAIL(HH_ERR_CUDA, "%s: join failed", fn);
  return r;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// PHBA
// ---------------------------------------------------------------------------
namespace {
bool phba_sizes_ok(int B, int T, int H, int C) {
  const long long nb = ((long long)T + C - 1) / C;
  return (long long)B * H * nb * 128 < (1LL << 31) && (long long)B * T * H * 17 < (1LL << 31) && B <= 65535 &&
         H <= 65535;
}
}  // namespace

size_t phba_prefix_states_workspace_size(int B, int T, int H, int d, int M, int C) {
  if (B <= 0 || T <= 0 || H <= 0 || d != 128 || M != 128 || (C != 64 && C != 128 && C != 256)) return 0;
  if (!phba_sizes_ok(B, T, H, C)) return 0;
  return hh::phba_states_workspace_bytes(B, T, H, C);
}

int phba_prefix_states(const hh_bf16 *k_raw, const hh_bf16 *v, const float *alpha, hh_bf16 *kstate,
                       hh_bf16 *vstate, void *workspace, size_t ws_bytes, int B, int T, int H, int d, int M, int C,
                       hh_stream stream) {
  static const char *fn = "phba_prefix_states";
  hh::clear_error();
  if (B < 0 || T <= 0 || H <= 0 || d <= 0 || M <= 0 || C <= 0)
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: sizes must be positive (B may be 0)", fn);
  if (d != 128 || M != 128) HH_FAIL(HH_ERR_UNSUPPORTED, "%s: only d = M = 128 is built", fn);
  if (C != 64 && C != 128 && C != 256) HH_FAIL(HH_ERR_UNSUPPORTED, "%s: block length C must be 64, 128 or 256", fn);
  if (!phba_sizes_ok(B, T, H, C)) HH_FAIL(HH_ERR_INVALID_ARG, "%s: sizes too large", fn);
  if (B == 0) return HH_OK;
  if (!k_raw || !v || !alpha || !kstate || !vstate) HH_FAIL(HH_ERR_INVALID_ARG, "%s: null tensor pointer", fn);
  if (!al16(k_raw) || !al16(v) || !al16(alpha) || !al16(kstate) || !al16(vstate))
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: tensors must be 16-byte aligned", fn);
  const size_t need = hh::phba_states_workspace_bytes(B, T, H, C);
  if (!workspace || ws_bytes < need)
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: workspace of %zu bytes needed (got %zu)", fn, need, ws_bytes);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", fn);
  if (int r = hh::check_device(fn)) return r;
  hh::PhbaStatesArgs a;
  a.k_raw = k_raw;
  a.v = v;
  a.alpha = alpha;
  a.kstate = kstate;
  a.vstate = vstate;
  a.B = B;
  a.T = T;
  a.H = H;
  a.C = C;
  a.workspace = workspace;
  return launch_result(hh::launch_phba_states(a, reinterpret_cast<cudaStream_t>(stream)), fn);
}

size_t phba_fwd_workspace_size(int B, int T, int H, int d, int M, int C, int K) {
  if (B <= 0 || T <= 0 || H <= 0 || d != 128 || M != 128 || (C != 64 && C != 128 && C != 256) || K < 0 || K > 16)
    return 0;
  if (!phba_sizes_ok(B, T, H, C) || T / C > 512) return 0;
  return hh::phba_fwd_workspace_bytes(B, T, H, C, K);
}

int phba_fwd(const hh_bf16 *q_rope, const hh_bf16 *k_rope, const hh_bf16 *q_raw, const hh_bf16 *v,
             const hh_bf16 *kstate, const hh_bf16 *vstate, hh_bf16 *o, int32_t *sel, void *workspace, size_t ws_bytes,
             int B, int T, int H, int d, int M, int C, int K, float scale, hh_stream stream) {
  static const char *fn = "phba_fwd";
  hh::clear_error();
  if (B < 0 || T <= 0 || H <= 0 || d <= 0 || M <= 0 || C <= 0 || K < 0)
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: sizes must be positive (B may be 0, K >= 0)", fn);
  if (d != 128 || M != 128) HH_FAIL(HH_ERR_UNSUPPORTED, "%s: only d = M = 128 is built", fn);
  if (C != 64 && C != 128 && C != 256) HH_FAIL(HH_ERR_UNSUPPORTED, "%s: block length C must be 64, 128 or 256", fn);
  if (K > 16) HH_FAIL(HH_ERR_UNSUPPORTED, "%s: at most K = 16 kept blocks", fn);
  if (T / C > 512) HH_FAIL(HH_ERR_UNSUPPORTED, "%s: at most 512 complete blocks (T / C = %d)", fn, T / C);
  if (!isfinite(scale)) HH_FAIL(HH_ERR_INVALID_ARG, "%s: scale must be finite", fn);
  if (!phba_sizes_ok(B, T, H, C)) HH_FAIL(HH_ERR_INVALID_ARG, "%s: sizes too large", fn);
  if (B == 0) return HH_OK;
  if (!q_rope || !k_rope || !q_raw || !v || !kstate || !vstate || !o)
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: null tensor pointer", fn);
  if (!al16(q_rope) || !al16(k_rope) || !al16(q_raw) || !al16(v) || !al16(kstate) || !al16(vstate) || !al16(o) ||
      (sel && !al4(sel)))
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: tensors must be 16-byte aligned (sel 4-byte)", fn);
  const size_t need = hh::phba_fwd_workspace_bytes(B, T, H, C, K);
  if (!workspace || ws_bytes < need)
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: workspace of %zu bytes needed (got %zu)", fn, need, ws_bytes);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    HH_FAIL(HH_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", fn);
  if (int r = hh::check_device(fn)) return r;
  hh::PhbaFwdArgs a;
  a.q_rope = q_rope;
  a.k_rope = k_rope;
  a.q_raw = q_raw;
  a.v = v;
  a.kstate = kstate;
  a.vstate = vstate;
  a.o = o;
  a.sel = sel;
  a.B = B;
  a.T = T;
  a.H = H;
  a.C = C;
  a.K = K;
  a.scale = scale;
  a.workspace = workspace;
  return launch_result(hh::launch_phba_fwd(a, reinterpret_cast<cudaStream_t>(stream)), fn);
}
