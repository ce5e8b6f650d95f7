// gen_inputs.cu -- libhh_gen.so: device-side seeded input generation for
// tensors too large to stage through host memory (the 34 GB decode KV cache).
// It holds none of the layer's arithmetic.
//
// Element i of a tensor (seed, stream) is the bf16 rounding of
//   (sum of the eight 16-bit halves of Philox4x32-10(ctr, key) - 262140) / sigma
// with ctr = (i mod 2^32, i / 2^32, stream, 0x48480000), key = (seed mod 2^32,
// seed / 2^32) and sigma = sqrt(8 (65536^2 - 1) / 12): an Irwin-Hall(8)
// approximation of N(0, 1).  Philox4x32-10 is the counter-based generator of
// Salmon, Moraes, Dror and Shaw, "Parallel random numbers: as easy as 1, 2, 3"
// (SC'11).  The host-side twin used by the tests is in inputs.py; both are
// written from that definition and checked against each other bit for bit.
// hh_gen_q8_0 draws a q8_0 cache (int8 values, fp16 scales) from the same normals.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

namespace {

__device__ __forceinline__ void philox_round(uint32_t &c0, uint32_t &c1, uint32_t &c2, uint32_t &c3, uint32_t k0,
                                             uint32_t k1) {
  const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
  const uint32_t hi0 = __umulhi(M0, c0), lo0 = M0 * c0;
  const uint32_t hi1 = __umulhi(M1, c2), lo1 = M1 * c2;
  const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
  c0 = n0;
  c1 = lo1;
  c2 = n2;
  c3 = lo0;
}

__global__ void fill_normal_bf16_kernel(uint16_t *__restrict__ dst, uint64_t n, uint64_t seed, uint32_t stream,
                                        float inv_sigma) {
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    uint32_t c0 = (uint32_t)i, c1 = (uint32_t)(i >> 32), c2 = stream, c3 = 0x48480000u;
    uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);
#pragma unroll
    for (int r = 0; r < 10; ++r) {
      philox_round(c0, c1, c2, c3, k0, k1);
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const int s = (int)(c0 & 0xFFFFu) + (int)(c0 >> 16) + (int)(c1 & 0xFFFFu) + (int)(c1 >> 16) +
                  (int)(c2 & 0xFFFFu) + (int)(c2 >> 16) + (int)(c3 & 0xFFFFu) + (int)(c3 >> 16);
    const float val = __fmul_rn((float)(s - 262140), inv_sigma);
    dst[i] = __bfloat16_as_ushort(__float2bfloat16_rn(val));
  }
}

// bf16 bits of element i of tensor (seed, stream): the Irwin-Hall(8) normal above
__device__ __forceinline__ uint16_t counter_normal_bits(uint64_t i, uint64_t seed, uint32_t stream, float inv_sigma) {
  uint32_t c0 = (uint32_t)i, c1 = (uint32_t)(i >> 32), c2 = stream, c3 = 0x48480000u;
  uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    philox_round(c0, c1, c2, c3, k0, k1);
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  const int s = (int)(c0 & 0xFFFFu) + (int)(c0 >> 16) + (int)(c1 & 0xFFFFu) + (int)(c1 >> 16) +
                (int)(c2 & 0xFFFFu) + (int)(c2 >> 16) + (int)(c3 & 0xFFFFu) + (int)(c3 >> 16);
  return __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn((float)(s - 262140), inv_sigma)));
}

// q8_0 cache drawn in its format: value i = clip(rint(32 z_i), -127, 127) with z_i the bf16 normal of
// (seed, stream_x, i); scale j = (64 + (bits of the bf16 normal of (seed, stream_s, j) & 63)) / 4096, exact in fp16.
__global__ void fill_q8_0_kernel(int8_t *__restrict__ vals, uint16_t *__restrict__ scales, uint64_t n_vals,
                                 uint64_t seed, uint32_t stream_x, uint32_t stream_s, float inv_sigma) {
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_vals; i += stride) {
    const float z = __uint_as_float((uint32_t)counter_normal_bits(i, seed, stream_x, inv_sigma) << 16);
    const float x = fminf(fmaxf(rintf(32.f * z), -127.f), 127.f);
    vals[i] = (int8_t)(int)x;
    if ((i & 31u) == 0) {
      const uint64_t j = i >> 5;
      const uint32_t h = counter_normal_bits(j, seed, stream_s, inv_sigma) & 63u;
      scales[j] = __half_as_ushort(__float2half_rn((float)(64u + h) * (1.f / 4096.f)));
    }
  }
}

}  // namespace

extern "C" __attribute__((visibility("default"))) int hh_gen_q8_0(int8_t *vals, uint16_t *scales, uint64_t n_vals,
                                                                  uint64_t seed, uint32_t stream_x, uint32_t stream_s,
                                                                  cudaStream_t s) {
  if (n_vals == 0) return 0;
  if (!vals || !scales || (n_vals & 31u)) return -1;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const float inv_sigma = (float)(1.0 / sqrt(8.0 * (65536.0 * 65536.0 - 1.0) / 12.0));
  fill_q8_0_kernel<<<sms * 8, 256, 0, s>>>(vals, scales, n_vals, seed, stream_x, stream_s, inv_sigma);
  return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

extern "C" __attribute__((visibility("default"))) int hh_gen_normal_bf16(uint16_t *dst, uint64_t n, uint64_t seed,
                                                                         uint32_t stream, cudaStream_t s) {
  if (n == 0) return 0;
  if (!dst) return -1;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // 1 / sigma of the Irwin-Hall(8) sum: computed in double on the host, rounded to float
  const float inv_sigma = (float)(1.0 / sqrt(8.0 * (65536.0 * 65536.0 - 1.0) / 12.0));
  fill_normal_bf16_kernel<<<sms * 8, 256, 0, s>>>(dst, n, seed, stream, inv_sigma);
  return cudaGetLastError() == cudaSuccess ? 0 : -3;
}
