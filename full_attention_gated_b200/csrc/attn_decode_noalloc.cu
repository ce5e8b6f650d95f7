// attn_decode_noalloc.cu -- gqa_attn_decode_noalloc: the split-K GQA decode
// with its scratch in a fixed device array inside this library, so that the
// caller passes only inputs and outputs and nothing is allocated anywhere.
//
// Who needs it: callers that cannot allocate device memory themselves, such as
// a plugin running inside a host framework that hands it only its input and
// output buffers and no allocator, or a serving loop whose memory budget is
// fixed up front.  Such callers also must not fall back to cudaMalloc /
// cudaFree per call, because those calls can synchronise the device and stall
// unrelated work.
//
// The scratch (partial softmax statistics and partial outputs of every split)
// is the file-scope array below.  Every GPU that loads this library holds it
// until the process exits.  Its device address is looked up once per device
// (cudaGetSymbolAddress, with that device current) on the first call made on
// that device, so that first call should come before any stream capture.  All
// calls on a device share the array and it keeps the last call's contents;
// nothing in it needs to start at zero (every partial is written before it is
// read), but calls whose work overlaps on the GPU (different streams, or
// different host threads) race on it and must be serialised by the caller.
#include <cuda_runtime.h>
#include <math.h>
#include <string.h>

#include <mutex>

#include "../../include/hh.h"
#include "internal.h"

namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[HH_NOALLOC_SCRATCH_BYTES];

// Device address of g_decode_scratch on the current device (set up once per device).
int scratch_address(void **out) {
  static std::mutex mu;
  static void *addr[128] = {nullptr};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 128) {
    hh::set_error("gqa_attn_decode_noalloc: no current CUDA device (%s)", cudaGetErrorString(e));
    return HH_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || !p) {
      hh::set_error("gqa_attn_decode_noalloc: cudaGetSymbolAddress of the scratch array failed (%s)",
                    cudaGetErrorString(e));
      return HH_ERR_CUDA;
    }
    addr[dev] = p;
  }
  *out = addr[dev];
  return HH_OK;
}

}  // namespace

extern "C" int gqa_attn_decode_noalloc(const hh_bf16 *q, const hh_bf16 *k_cache, const hh_bf16 *v_cache,
                                       const int32_t *cache_len, const hh_bf16 *gate, hh_bf16 *o, int B,
                                       int T_cache, int H_q, int H_kv, int d, float scale, hh_stream stream) {
  static const char *fn = "gqa_attn_decode_noalloc";
  hh::clear_error();
  // the same checks as gqa_attn_decode (shared code), then the fixed scratch's size limit
  const int v = hh::check_decode_args(fn, q, k_cache, v_cache, cache_len, gate, o, B, T_cache, H_q, H_kv, d, scale);
  if (v < 0) return v;
  if (v == hh::kNothingToDo) return HH_OK;
  const size_t need = hh::attn_decode_workspace(B, H_q, d, T_cache);
  if (need > (size_t)HH_NOALLOC_SCRATCH_BYTES) {
    hh::set_error("%s: this shape needs %zu bytes of scratch, more than the library's fixed %zu bytes; "
                  "use gqa_attn_decode with a caller-provided workspace",
                  fn, need, (size_t)HH_NOALLOC_SCRATCH_BYTES);
    return HH_ERR_UNSUPPORTED;
  }
  if (int r = hh::check_device(fn)) return r;
  void *scratch = nullptr;
  if (int r = scratch_address(&scratch)) return r;
  hh::AttnDecodeArgs a;
  a.q = q;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.gate = gate;
  a.cache_len = cache_len;
  a.o = o;
  a.workspace = scratch;
  a.B = B;
  a.T_cache = T_cache;
  a.H_q = H_q;
  a.H_kv = H_kv;
  a.d = d;
  a.scale = scale;
  cudaError_t e = hh::launch_attn_decode(a, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    if (!hh::last_error()[0]) hh::set_error("%s: CUDA error: %s", fn, cudaGetErrorString(e));
    return HH_ERR_CUDA;
  }
  return HH_OK;
}
