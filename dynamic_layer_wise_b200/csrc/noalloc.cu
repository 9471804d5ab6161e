// Allocation-free LM-head confidence for callers that cannot call cudaMalloc.
//
// Some callers of this library run where device allocation is not theirs to
// do: inside a host framework that owns every device allocation through its
// own pool, or in a process whose allocator is frozen once serving starts.
// They can pass inputs and outputs they already own, but cannot let the
// library allocate scratch.  dcu_lm_confidence_noalloc serves them: it keeps
// its scratch in one file-scope device array, sized at compile time and held
// by every GPU that loads the library until the process exits.
//
// The work is the same as the LM-head stage of commit_select (final RMSNorm,
// logits, max-probability confidence and argmax), reusing that stage's
// gather+RMSNorm and GEMM kernels; the vocabulary is processed in chunks of
// kNaVChunk entries whose softmax statistics are merged online, so the logits
// scratch stays small whatever the vocabulary size.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace {

constexpr int kNaMaxRows = 256;    // rows per call
constexpr int kNaMaxD = 8192;      // d_model
constexpr int kNaVChunk = 4096;    // vocabulary entries per logits chunk

struct NaState {
  double sum;  // sum of exp(z - mx) over the chunks seen so far
  float mx;    // running maximum logit
  int arg;     // lowest id reaching the running maximum
};

constexpr size_t kRowsBytes = (size_t)kNaMaxRows * kNaMaxD * 4;      // normalised rows (<= 4 bytes/elem)
constexpr size_t kLogitBytes = (size_t)kNaMaxRows * kNaVChunk * 4;   // one logits chunk, fp32
constexpr size_t kStateBytes = (size_t)kNaMaxRows * sizeof(NaState);
constexpr size_t kMapBytes = (size_t)kNaMaxRows * 4 + 256;           // identity row map + row count
constexpr size_t kScratchBytes = kRowsBytes + kLogitBytes + kStateBytes + kMapBytes;  // ~12 MB

static __device__ __align__(256) unsigned char g_na_scratch[kScratchBytes];

// Host-side device addresses of g_na_scratch, one per device, taken on the
// first call on that device (with that device current).
std::mutex g_na_mutex;
void *g_na_ptr[128] = {};

__global__ void k_na_plan(int m, int32_t *rowmap, int32_t *m_total) {
  for (int r = threadIdx.x; r < m; r += blockDim.x) rowmap[r] = r;
  if (threadIdx.x == 0) *m_total = m;
}

// Softmax statistics of one logits chunk [m][ncols] (ids base..base+ncols),
// merged into the running state of each row.
__global__ void k_na_merge(const float *__restrict__ z, int ldz, int ncols, int base, int m, int first,
                           NaState *__restrict__ st) {
  __shared__ float smax[32];
  __shared__ int sidx[32];
  __shared__ double sred[32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int r = blockIdx.x; r < m; r += gridDim.x) {
    const float *zr = z + (size_t)r * ldz;
    float best = -INFINITY;
    int bi = 0x7fffffff;
    for (int v = threadIdx.x; v < ncols; v += blockDim.x) {
      const float x = zr[v];
      if (x > best) { best = x; bi = v; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ob > best || (ob == best && oi < bi)) { best = ob; bi = oi; }
    }
    __syncthreads();
    if (lane == 0) { smax[w] = best; sidx[w] = bi; }
    __syncthreads();
    if (w == 0) {
      best = lane < nw ? smax[lane] : -INFINITY;
      bi = lane < nw ? sidx[lane] : 0x7fffffff;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ob > best || (ob == best && oi < bi)) { best = ob; bi = oi; }
      }
      if (lane == 0) { smax[0] = best; sidx[0] = bi; }
    }
    __syncthreads();
    // a chunk with no ordered maximum (every logit NaN) keeps its first id as
    // the argmax; its sum is then NaN, which the confidence reports
    const float cmax = smax[0];
    const int carg = (sidx[0] == 0x7fffffff ? 0 : sidx[0]) + base;
    double s = 0.0;
    for (int v = threadIdx.x; v < ncols; v += blockDim.x) s += (double)expf(zr[v] - cmax);
    s = dcu::block_sum(s, sred);
    if (threadIdx.x == 0) {
      NaState t = st[r];
      if (first) {
        t.sum = s; t.mx = cmax; t.arg = carg;
      } else if (cmax > t.mx) {          // chunks come in ascending id order: equal maxima keep the lower id
        t.sum = t.sum * exp((double)t.mx - (double)cmax) + s;
        t.mx = cmax;
        t.arg = carg;
      } else {
        t.sum += s * exp((double)cmax - (double)t.mx);
      }
      st[r] = t;
    }
  }
}

__global__ void k_na_finish(const NaState *__restrict__ st, int m, float *__restrict__ conf,
                            int32_t *__restrict__ argmax) {
  for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < m; r += gridDim.x * blockDim.x) {
    conf[r] = (float)(1.0 / st[r].sum);
    argmax[r] = st[r].arg;
  }
}

int na_fail(int code, const char *msg) {
  dcu::set_global_error(msg);
  return code;
}

}  // namespace

extern "C" int dcu_lm_confidence_noalloc(const void *h_rows, const float *final_norm, const void *lm_head, int32_t m,
                                         int32_t D, int32_t V, int32_t dtype, float rms_eps, float *conf,
                                         int32_t *argmax, dcu_stream_t stream) {
  if (!h_rows || !final_norm || !lm_head || !conf || !argmax || (dtype != DCU_F32 && dtype != DCU_BF16) ||
      m < 0 || D <= 0 || V <= 0 || D % 64 || !(rms_eps > 0.0f))
    return na_fail(DCU_EINVAL, "dcu_lm_confidence_noalloc: bad argument");
  {
    // the row, gain and weight loads are 16-byte vectors; outputs are 4-byte words
    auto mis = [](const void *q, uintptr_t a) { return (reinterpret_cast<uintptr_t>(q) & (a - 1)) != 0; };
    if (mis(h_rows, 16) || mis(final_norm, 16) || mis(lm_head, 16) || mis(conf, 4) || mis(argmax, 4))
      return na_fail(DCU_EINVAL,
                     "dcu_lm_confidence_noalloc: h_rows, final_norm and lm_head must be 16-byte aligned, "
                     "conf and argmax 4-byte aligned");
  }
  if (m > kNaMaxRows || D > kNaMaxD)
    return na_fail(DCU_ECAPACITY, "dcu_lm_confidence_noalloc: at most 256 rows per call and d_model <= 8192");
  if (m == 0) return DCU_OK;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128)
    return na_fail(DCU_ECUDA, "dcu_lm_confidence_noalloc: cudaGetDevice failed");
  void *base = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_na_mutex);
    if (!g_na_ptr[dev]) {
      void *p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, g_na_scratch);
      if (e != cudaSuccess || !p)
        return na_fail(DCU_ECUDA, "dcu_lm_confidence_noalloc: cudaGetSymbolAddress of the scratch array failed");
      g_na_ptr[dev] = p;
    }
    base = g_na_ptr[dev];
  }
  unsigned char *b = static_cast<unsigned char *>(base);
  void *rows = b;
  float *logits = reinterpret_cast<float *>(b + kRowsBytes);
  NaState *st = reinterpret_cast<NaState *>(b + kRowsBytes + kLogitBytes);
  int32_t *rowmap = reinterpret_cast<int32_t *>(b + kRowsBytes + kLogitBytes + kStateBytes);
  int32_t *m_total = rowmap + kNaMaxRows;
  cudaStream_t s = (cudaStream_t)stream;
  const size_t esz = dtype == DCU_BF16 ? 2 : 4;

  k_na_plan<<<1, 256, 0, s>>>(m, rowmap, m_total);
  if (cudaGetLastError() != cudaSuccess) return na_fail(DCU_ECUDA, "dcu_lm_confidence_noalloc: launch failed");
  if (dcu::launch_gather_norm(dtype, rowmap, m_total, m, h_rows, final_norm, rms_eps, D, rows, s) != cudaSuccess)
    return na_fail(DCU_ECUDA, "dcu_lm_confidence_noalloc: gather/norm launch failed");
  for (int v0 = 0, c = 0; v0 < V; v0 += kNaVChunk, ++c) {
    const int nc = (V - v0) < kNaVChunk ? (V - v0) : kNaVChunk;
    dcu::GemmSeg seg{static_cast<const unsigned char *>(lm_head) + (size_t)v0 * D * esz, nc};
    if (dcu::launch_gemm_simt(dtype, rows, D, m_total, m, &seg, 1, D, logits, kNaVChunk, s) != cudaSuccess)
      return na_fail(DCU_ECUDA, "dcu_lm_confidence_noalloc: GEMM launch failed");
    k_na_merge<<<m, 256, 0, s>>>(logits, kNaVChunk, nc, v0, m, c == 0, st);
    if (cudaGetLastError() != cudaSuccess) return na_fail(DCU_ECUDA, "dcu_lm_confidence_noalloc: launch failed");
  }
  k_na_finish<<<(m + 255) / 256, 256, 0, s>>>(st, m, conf, argmax);
  if (cudaGetLastError() != cudaSuccess) return na_fail(DCU_ECUDA, "dcu_lm_confidence_noalloc: launch failed");
  return DCU_OK;
}
