// Device implementation of the seeded synthetic-input generator (see
// include/dcu_gen.h for the definition).  Integer hashing and one binary64
// multiply per element: bit-identical to the host implementation.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/dcu_gen.h"

namespace {

constexpr uint64_t kGolden = 0x9E3779B97F4A7C15ull;

__host__ __device__ inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ inline uint16_t f64_to_bf16_bits(double v) {
  unsigned long long b = (unsigned long long)__double_as_longlong(v);
  b = b + ((1ull << 44) - 1) + ((b >> 45) & 1ull);
  b &= ~((1ull << 45) - 1);
  float f = __double2float_rn(__longlong_as_double((long long)b));  // exact: 8 significant bits
  return (uint16_t)(__float_as_uint(f) >> 16);
}

__global__ void k_normal(void *out, int64_t n, uint64_t base, uint64_t start, double scale, int dtype) {
  for (int64_t k = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; k < n; k += (int64_t)gridDim.x * blockDim.x) {
    const uint64_t h = mix64(base + (start + (uint64_t)k + 1ull) * kGolden);
    const int64_t S = (int64_t)(h & 0xFFFF) + (int64_t)((h >> 16) & 0xFFFF) + (int64_t)((h >> 32) & 0xFFFF) +
                      (int64_t)((h >> 48) & 0xFFFF);
    const double v = __dmul_rn((double)(S - 131070), scale);
    if (dtype == 0)
      reinterpret_cast<uint16_t *>(out)[k] = f64_to_bf16_bits(v);
    else
      reinterpret_cast<float *>(out)[k] = __double2float_rn(v);
  }
}

__global__ void k_fill(void *out, int64_t n, float value, int dtype) {
  for (int64_t k = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; k < n; k += (int64_t)gridDim.x * blockDim.x) {
    if (dtype == 0)
      reinterpret_cast<__nv_bfloat16 *>(out)[k] = __float2bfloat16_rn(value);
    else
      reinterpret_cast<float *>(out)[k] = value;
  }
}

}  // namespace

extern "C" int dcugen_normal(void *out, int64_t n, uint64_t seed, uint32_t tid, uint64_t start, double std,
                             int32_t dtype, void *stream) {
  if (n <= 0) return 0;
  const uint64_t base = mix64(((seed & 0xFFFFFFFFull) << 32) ^ (uint64_t)tid);
  const double scale = (std * 1.7320508075688772) / 65536.0;
  k_normal<<<148 * 32, 256, 0, (cudaStream_t)stream>>>(out, n, base, start, scale, dtype);
  return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

extern "C" int dcugen_fill(void *out, int64_t n, float value, int32_t dtype, void *stream) {
  if (n <= 0) return 0;
  k_fill<<<148 * 8, 256, 0, (cudaStream_t)stream>>>(out, n, value, dtype);
  return cudaGetLastError() == cudaSuccess ? 0 : -3;
}
