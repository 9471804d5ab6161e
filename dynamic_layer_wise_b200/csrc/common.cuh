// Shared device helpers of libdcu (sm_100a).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>
#include <utility>
#include <vector>

#include "../../include/dcu.h"

namespace dcu {

typedef __nv_bfloat16 bf16;

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(bf16 x) { return __bfloat162float(x); }

template <class T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float x) { return __float2bfloat16_rn(x); }

template <class T> __device__ __forceinline__ uint32_t bits_of(T x);
template <> __device__ __forceinline__ uint32_t bits_of<float>(float x) { return __float_as_uint(x); }
template <> __device__ __forceinline__ uint32_t bits_of<bf16>(bf16 x) { return (uint32_t)__bfloat16_as_ushort(x); }

// 16-byte vector of T: 4 floats or 8 bf16.
template <class T> struct Vec;
template <> struct Vec<float> { static constexpr int n = 4; };
template <> struct Vec<bf16> { static constexpr int n = 8; };

template <class T>
__device__ __forceinline__ void load_vec(const T *p, float (&v)[Vec<T>::n], uint32_t (&b)[Vec<T>::n]) {
  uint4 u = *reinterpret_cast<const uint4 *>(p);
  const T *e = reinterpret_cast<const T *>(&u);
#pragma unroll
  for (int i = 0; i < Vec<T>::n; ++i) { v[i] = to_f(e[i]); b[i] = bits_of<T>(e[i]); }
}

template <class T>
__device__ __forceinline__ void load_vec(const T *p, float (&v)[Vec<T>::n]) {
  uint4 u = *reinterpret_cast<const uint4 *>(p);
  const T *e = reinterpret_cast<const T *>(&u);
#pragma unroll
  for (int i = 0; i < Vec<T>::n; ++i) v[i] = to_f(e[i]);
}

template <class T>
__device__ __forceinline__ void store_vec(T *p, const float (&v)[Vec<T>::n]) {
  uint4 u;
  T *e = reinterpret_cast<T *>(&u);
#pragma unroll
  for (int i = 0; i < Vec<T>::n; ++i) e[i] = from_f<T>(v[i]);
  *reinterpret_cast<uint4 *>(p) = u;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ int warp_sum(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block-wide sum with a fixed reduction tree (deterministic).  `red` must
// hold blockDim.x / 32 elements; every thread gets the result.
template <class T>
__device__ __forceinline__ T block_sum(T v, T *red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  T t = (threadIdx.x < nw) ? red[threadIdx.x] : T(0);
  if (w == 0) t = warp_sum(t);
  if (threadIdx.x == 0) red[0] = t;
  __syncthreads();
  T r = red[0];
  __syncthreads();
  return r;
}

// Exclusive prefix sum over the block of one int per thread (thread order);
// returns the exclusive prefix, total in *total.  `red` holds 32 ints.
__device__ __forceinline__ int block_exclusive_scan(int v, int *red, int *total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) red[w] = x;
  __syncthreads();
  if (w == 0) {
    int t = (lane < nw) ? red[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    red[lane] = t;  // inclusive scan of warp totals
  }
  __syncthreads();
  int base = (w > 0) ? red[w - 1] : 0;
  *total = red[nw - 1];
  __syncthreads();
  return base + x - v;
}

// Cosine distance of [DLLM] "关键设计 1" from fp64 partial sums, with the
// equal-rows / zero-norm rules; clamped to [0, 2].
__device__ __forceinline__ float finish_cosine_distance(double dot, double nx, double ny, bool same) {
  if (same) return 0.0f;
  if (nx == 0.0 && ny == 0.0) return 0.0f;
  if (nx == 0.0 || ny == 0.0) return 1.0f;
  double d = 1.0 - dot / (sqrt(nx) * sqrt(ny));
  d = d < 0.0 ? 0.0 : (d > 2.0 ? 2.0 : d);
  return (float)d;
}

// Lets the next kernel of the stream, when launched with programmatic stream
// serialization, start its independent prologue now.
__device__ __forceinline__ void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Programmatic dependent launch: waits until the previous kernel of the stream
// has completed and its writes are visible (a no-op without a programmatic edge).
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// First statement of every kernel launched by launch_pdl: wait for the
// predecessor, then let the successor be scheduled (so at most one kernel of
// the stream waits ahead of the running one).
__device__ __forceinline__ void pdl_enter() {
  griddep_wait();
  allow_dependents();
}

// Asks for the largest shared-memory carveout for `kern` on the current device
// (once per kernel and device).  Under programmatic dependent launch the next
// kernel's CTAs are scheduled while this one runs; a GEMM CTA needs 220 KB of
// shared memory, which an SM configured for a small carveout cannot give until
// it drains.
inline void prefer_max_smem(const void *kern) {
  static std::mutex mu;
  static std::vector<std::pair<const void *, int>> done;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return;
  std::lock_guard<std::mutex> lock(mu);
  for (const auto &d : done)
    if (d.first == kern && d.second == dev) return;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared) ==
      cudaSuccess)
    done.emplace_back(kern, dev);
  else
    cudaGetLastError();
}

// Launch with programmatic stream serialization: the kernel's CTAs may be
// scheduled while its predecessor finishes, hiding the launch latency; the
// kernel must call pdl_enter() (or griddep_wait()) before touching anything
// the predecessor reads or writes.
template <class... Exp, class... Act>
inline cudaError_t launch_pdl(void (*kern)(Exp...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Act &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  prefer_max_smem(reinterpret_cast<const void *>(kern));
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Act &&>(args)...);
}

// Raises the dynamic shared memory limit of kernel `kern` to `bytes` on the
// current device, once per device: the attribute belongs to the device's copy
// of the kernel, so a flag per process would leave a second GPU without it.
// `done` holds one bit per device (devices 64 and up set it on every call);
// setting the attribute twice is harmless, so concurrent first calls are safe.
template <class... Exp>
inline cudaError_t ensure_smem_limit(void (*kern)(Exp...), int bytes, std::atomic<uint64_t> &done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// Row r of the packed recompute set -> global row b*N + i (written by the
// select / plan kernels).
struct RowPlan {
  const int32_t *rowmap;   // [cap] global row index b*N + i
  const int32_t *m_total;  // device scalar
};

}  // namespace dcu
