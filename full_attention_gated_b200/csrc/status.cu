// status.cu -- per-device status word, tensor-map encoding and the
// thread-local error string shared by the launchers.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdio.h>

#include <mutex>

#include "../../include/hh.h"

#include "common.cuh"
#include "internal.h"

namespace hh {

// One status word per device that loads the library.  Kernels get its
// address; hh_device_status reads and clears it.
static __device__ unsigned g_status_word;

static thread_local char t_err[512];

void set_error(const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_err, sizeof(t_err), fmt, ap);
  va_end(ap);
}
const char *last_error() { return t_err; }
void clear_error() { t_err[0] = 0; }

unsigned *device_status_ptr() {
  static std::mutex mu;
  static unsigned *ptrs[128] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<unsigned *>(p);
  }
  return ptrs[dev];
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

CUresult encode_tmap(CUtensorMap *map, CUtensorMapDataType dtype, int rank, const void *base, const uint64_t *dims,
                     const uint64_t *strides_bytes, const uint32_t *box, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = get_encode();
  if (!fn) return CUDA_ERROR_NOT_FOUND;
  cuuint64_t d[5], st[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) st[i] = strides_bytes[i];
  }
  return fn(map, dtype, (cuuint32_t)rank, const_cast<void *>(base), d, st, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

// Waits on an mbarrier that nothing ever arrives on, with a bounded wait of
// `limit_ns`; the expiry sets the device status word like any other kernel's.
__global__ void selftest_wait_kernel(unsigned *status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(&bar, 0)) {
    if (global_ns() - t0 > limit_ns) {
      atomicOr(status, kStatusTimeout);
      return;
    }
  }
}

}  // namespace hh

extern "C" HH_API int hh_selftest_wait_timeout(unsigned limit_us, hh_stream stream) {
  hh::clear_error();
  if (limit_us == 0 || limit_us > 2000000u) {
    hh::set_error("hh_selftest_wait_timeout: limit_us must be in 1 .. 2,000,000");
    return HH_ERR_INVALID_ARG;
  }
  unsigned *st = hh::device_status_ptr();
  if (!st) {
    hh::set_error("hh_selftest_wait_timeout: no CUDA device");
    return HH_ERR_CUDA;
  }
  hh::selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(st, (uint64_t)limit_us * 1000ull);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    hh::set_error("hh_selftest_wait_timeout: %s", cudaGetErrorString(e));
    return HH_ERR_CUDA;
  }
  return HH_OK;
}
