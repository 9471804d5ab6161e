// Attention of the recomputed queries over all N cached keys of their
// sequence (bidirectional, no mask; [DLLM] "研究背景与动机": dLLMs denoise
// with bidirectional attention), one CTA per (query row, head):
// scores in shared memory, exact softmax, then P V.
#include "common.cuh"
#include "kernels.h"

namespace dcu {

namespace {
template <class T>
__global__ void __launch_bounds__(128)
    k_attn_rowhead(const T *__restrict__ Q, const int32_t *__restrict__ rowmap, const int32_t *__restrict__ m_total,
                   int N, int H, int Hkv, int hd, const T *__restrict__ Kc, const T *__restrict__ Vc,
                   T *__restrict__ out, float scale) {
  extern __shared__ float sc[];  // [N]
  __shared__ __align__(16) float q[256];
  __shared__ float redf[32];
  __shared__ double redd[32];
  constexpr int VN = Vec<T>::n;
  const int M = *m_total;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, nw = blockDim.x >> 5;
  for (long long item = blockIdx.x; item < (long long)M * H; item += gridDim.x) {
    const int r = (int)(item / H), h = (int)(item - (long long)r * H);
    const int b = rowmap[r] / N;
    const int kvh = (h * Hkv) / H;
    __syncthreads();
    for (int j = tid; j < hd; j += blockDim.x) q[j] = to_f(Q[((size_t)r * H + h) * hd + j]) * scale;
    __syncthreads();
    const T *Kb = Kc + ((size_t)b * Hkv + kvh) * (size_t)N * hd;
    const T *Vb = Vc + ((size_t)b * Hkv + kvh) * (size_t)N * hd;
    float lmax = -INFINITY;
    for (int key = tid; key < N; key += blockDim.x) {
      const T *kr = Kb + (size_t)key * hd;
      float s = 0.f;
      for (int j = 0; j < hd; j += VN) {
        float kv[VN];
        load_vec(kr + j, kv);
#pragma unroll
        for (int e = 0; e < VN; ++e) s = fmaf(q[j + e], kv[e], s);
      }
      sc[key] = s;
      lmax = fmaxf(lmax, s);
    }
    lmax = warp_max(lmax);
    if (lane == 0) redf[w] = lmax;
    __syncthreads();
    float mx = -INFINITY;
    for (int i = 0; i < nw; ++i) mx = fmaxf(mx, redf[i]);
    double lsum = 0.0;
    for (int key = tid; key < N; key += blockDim.x) {
      const float p = expf(sc[key] - mx);
      sc[key] = p;
      lsum += (double)p;
    }
    const double sum = block_sum(lsum, redd);  // includes a __syncthreads after sc writes
    const float inv = (float)(1.0 / sum);
    for (int t = tid; t < hd; t += blockDim.x) {
      float acc = 0.f;
      for (int key = 0; key < N; ++key) acc = fmaf(sc[key], to_f(Vb[(size_t)key * hd + t]), acc);
      out[((size_t)r * H + h) * hd + t] = from_f<T>(acc * inv);
    }
  }
}
}  // namespace

cudaError_t launch_attention(int dtype, const void *Q, const int32_t *rowmap, const int32_t *m_total, int cap,
                             int N, int H, int Hkv, int hd, const void *Kc, const void *Vc, void *out,
                             cudaStream_t s) {
  if (hd > 256 || N > 16384) return cudaErrorInvalidValue;
  const size_t smem = (size_t)N * sizeof(float);
  static std::atomic<uint64_t> attr_bf16{0}, attr_f32{0};
  if (cudaError_t e = ensure_smem_limit(k_attn_rowhead<bf16>, 16384 * (int)sizeof(float), attr_bf16)) return e;
  if (cudaError_t e = ensure_smem_limit(k_attn_rowhead<float>, 16384 * (int)sizeof(float), attr_f32)) return e;
  long long items = (long long)cap * H;
  int grid = (int)(items < 148 * 16 ? items : 148 * 16);
  if (grid < 1) grid = 1;
  const float scale = 1.0f / sqrtf((float)hd);
  if (dtype == DCU_BF16)
    k_attn_rowhead<bf16><<<grid, 128, smem, s>>>((const bf16 *)Q, rowmap, m_total, N, H, Hkv, hd, (const bf16 *)Kc,
                                                 (const bf16 *)Vc, (bf16 *)out, scale);
  else
    k_attn_rowhead<float><<<grid, 128, smem, s>>>((const float *)Q, rowmap, m_total, N, H, Hkv, hd,
                                                  (const float *)Kc, (const float *)Vc, (float *)out, scale);
  return cudaGetLastError();
}

}  // namespace dcu
