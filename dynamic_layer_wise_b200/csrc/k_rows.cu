// Row-parallel kernels of the DCU step: layer-0 refresh, token dynamics,
// gather + RMSNorm, GEMM epilogues (RoPE + K/V write, residual + RMSNorm,
// SwiGLU, residual + scatter + next-layer dynamics) and the softmax-max of the
// LM head.  One CTA per row (grid-stride), 16-byte vector accesses along the
// row; HBM-bound.
#include "common.cuh"
#include "kernels.h"

namespace dcu {

// Split-K partials of a GEMM output element, summed in split order.
__device__ __forceinline__ float csum(const float *c, size_t sstride, int splits, size_t j) {
  float v = c[j];
  for (int sp = 1; sp < splits; ++sp) v += c[sp * sstride + j];
  return v;
}

static inline int row_grid(int rows_cap) {
  int g = rows_cap < 148 * 16 ? rows_cap : 148 * 16;
  return g > 0 ? g : 1;
}

// ------------------------------------------------------------------ RoPE table
// tab[p][j] = (cos, sin)(p * theta^(-2j/hd)), computed in fp64.
__global__ void k_rope_table(float2 *tab, int max_seq, int hd, double theta) {
  const int half = hd / 2;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < (int64_t)max_seq * half;
       t += (int64_t)gridDim.x * blockDim.x) {
    int p = (int)(t / half), j = (int)(t % half);
    double inv = pow(theta, -(2.0 * j) / (double)hd);
    double a = (double)p * inv;
    tab[t] = make_float2((float)cos(a), (float)sin(a));
  }
}

cudaError_t launch_rope_table(float2 *tab, int max_seq, int hd, float theta, cudaStream_t s) {
  k_rope_table<<<256, 256, 0, s>>>(tab, max_seq, hd, (double)theta);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ dynamics helpers
// Per-thread fp64 partial sums of <g x, g y>, |g x|^2, |g y|^2 and a
// bitwise-equality flag over the thread's vectors of a row.
template <class T>
__device__ __forceinline__ void dyn_accum(const T *x, const T *y, const float *g, int D, double &dot, double &nx,
                                          double &ny, bool &same) {
  constexpr int VN = Vec<T>::n;
  for (int j = threadIdx.x * VN; j < D; j += blockDim.x * VN) {
    float xv[VN], yv[VN];
    uint32_t xb[VN], yb[VN];
    load_vec(x + j, xv, xb);
    load_vec(y + j, yv, yb);
#pragma unroll
    for (int i = 0; i < VN; ++i) {
      same = same && (xb[i] == yb[i]);
      double gg = (double)g[j + i];
      double a = gg * (double)xv[i], b = gg * (double)yv[i];
      dot += a * b;
      nx += a * a;
      ny += b * b;
    }
  }
}

// ------------------------------------------------------------------ layer-0 refresh
// full != 0: H0[r] = E[id] for every row (dense forward).  Otherwise only rows
// whose id changed since the previous call are rewritten, with d0 = distance
// between the new embedding row and the cached H0 row ([DLLM] "关键设计 1").
template <class T>
__global__ void k_embed_refresh(const int32_t *__restrict__ ids, int32_t *__restrict__ prev_ids,
                                const T *__restrict__ embed, T *__restrict__ H0, float *__restrict__ d0,
                                const float *__restrict__ g0, int BN, int D, int V, int full, int32_t *status) {
  __shared__ double red[32];
  constexpr int VN = Vec<T>::n;
  for (int r = blockIdx.x; r < BN; r += gridDim.x) {
    int id = ids[r];
    if (id < 0 || id >= V) {
      if (threadIdx.x == 0) atomicOr(status, DCU_ST_BAD_TOKEN);
      id = id < 0 ? 0 : V - 1;
    }
    const T *e = embed + (size_t)id * D;
    T *h = H0 + (size_t)r * D;
    if (full) {
      for (int j = threadIdx.x * VN; j < D; j += blockDim.x * VN)
        *reinterpret_cast<uint4 *>(h + j) = *reinterpret_cast<const uint4 *>(e + j);
      if (threadIdx.x == 0) { prev_ids[r] = id; d0[r] = 0.f; }
      continue;
    }
    const int old = prev_ids[r];
    if (old == id) {
      if (threadIdx.x == 0) d0[r] = 0.f;
      continue;
    }
    double dot = 0, nx = 0, ny = 0;
    bool same = true;
    dyn_accum<T>(e, h, g0, D, dot, nx, ny, same);
    same = __syncthreads_and(same);
    dot = block_sum(dot, red);
    nx = block_sum(nx, red);
    ny = block_sum(ny, red);
    for (int j = threadIdx.x * VN; j < D; j += blockDim.x * VN)
      *reinterpret_cast<uint4 *>(h + j) = *reinterpret_cast<const uint4 *>(e + j);
    if (threadIdx.x == 0) {
      d0[r] = finish_cosine_distance(dot, nx, ny, same);
      prev_ids[r] = id;
    }
  }
}

cudaError_t launch_embed_refresh(int dtype, const int32_t *ids, int32_t *prev_ids, const void *embed, void *H0,
                                 float *d0, const float *g0, int BN, int D, int V, int full, int32_t *status,
                                 cudaStream_t s) {
  if (BN <= 0) return cudaSuccess;
  if (dtype == DCU_BF16)
    k_embed_refresh<bf16><<<row_grid(BN), 256, 0, s>>>(ids, prev_ids, (const bf16 *)embed, (bf16 *)H0, d0, g0, BN,
                                                        D, V, full, status);
  else
    k_embed_refresh<float><<<row_grid(BN), 256, 0, s>>>(ids, prev_ids, (const float *)embed, (float *)H0, d0, g0,
                                                         BN, D, V, full, status);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ standalone dynamics
template <class T>
__global__ void k_cosine_distance(const T *__restrict__ x, const T *__restrict__ y, const float *__restrict__ g,
                                  int64_t rows, int D, float *__restrict__ d) {
  __shared__ double red[32];
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    double dot = 0, nx = 0, ny = 0;
    bool same = true;
    dyn_accum<T>(x + r * D, y + r * D, g, D, dot, nx, ny, same);
    same = __syncthreads_and(same);
    dot = block_sum(dot, red);
    nx = block_sum(nx, red);
    ny = block_sum(ny, red);
    if (threadIdx.x == 0) d[r] = finish_cosine_distance(dot, nx, ny, same);
  }
}

cudaError_t launch_cosine_distance(int dtype, const void *x, const void *y, const float *g, int64_t rows, int D,
                                   float *d, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  int grid = rows < 148 * 16 ? (int)rows : 148 * 16;
  if (dtype == DCU_BF16)
    k_cosine_distance<bf16><<<grid, 256, 0, s>>>((const bf16 *)x, (const bf16 *)y, g, rows, D, d);
  else
    k_cosine_distance<float><<<grid, 256, 0, s>>>((const float *)x, (const float *)y, g, rows, D, d);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ gather + RMSNorm
// xs[r] = T(H[rowmap[r]] / sqrt(mean(H^2) + eps) * g) for r < *m_total.
template <class T>
__global__ void k_gather_norm(const int32_t *__restrict__ rowmap, const int32_t *__restrict__ m_total,
                              const T *__restrict__ H, const float *__restrict__ g, float eps, int D,
                              T *__restrict__ xs) {
  __shared__ double red[32];
  constexpr int VN = Vec<T>::n;
  const int M = *m_total;
  for (int r = blockIdx.x; r < M; r += gridDim.x) {
    const T *x = H + (size_t)rowmap[r] * D;
    double ss = 0;
    for (int j = threadIdx.x * VN; j < D; j += blockDim.x * VN) {
      float v[VN];
      load_vec(x + j, v);
#pragma unroll
      for (int i = 0; i < VN; ++i) ss += (double)v[i] * (double)v[i];
    }
    ss = block_sum(ss, red);
    const float inv = (float)(1.0 / sqrt(ss / (double)D + (double)eps));
    T *o = xs + (size_t)r * D;
    for (int j = threadIdx.x * VN; j < D; j += blockDim.x * VN) {
      float v[VN];
      load_vec(x + j, v);
#pragma unroll
      for (int i = 0; i < VN; ++i) v[i] = v[i] * inv * g[j + i];
      store_vec(o + j, v);
    }
  }
}

cudaError_t launch_gather_norm(int dtype, const int32_t *rowmap, const int32_t *m_total, int cap, const void *H,
                               const float *g, float eps, int D, void *xs, cudaStream_t s) {
  if (dtype == DCU_BF16)
    k_gather_norm<bf16><<<row_grid(cap), 256, 0, s>>>(rowmap, m_total, (const bf16 *)H, g, eps, D, (bf16 *)xs);
  else
    k_gather_norm<float><<<row_grid(cap), 256, 0, s>>>(rowmap, m_total, (const float *)H, g, eps, D, (float *)xs);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ QKV epilogue
// C row r = [q (H*hd) | k (Hkv*hd) | v (Hkv*hd)].  RoPE (rotate-half) on q and
// k at the row's position; q -> Q[r]; k, v -> the layer's K/V cache at
// (b, kv head, i).
template <class T>
__global__ void k_epi_qkv(const float *__restrict__ C, int ldc, int splits, size_t sstride,
                          const int32_t *__restrict__ rowmap,
                          const int32_t *__restrict__ m_total, int N, int H, int Hkv, int hd,
                          const float2 *__restrict__ rope_tab, int use_rope, T *__restrict__ Q, T *__restrict__ Kc,
                          T *__restrict__ Vc) {
  const int M = *m_total;
  const int half = hd / 2;
  for (int r = blockIdx.x; r < M; r += gridDim.x) {
    const int row = rowmap[r];
    const int b = row / N, i = row - b * N;
    const float *c = C + (size_t)r * ldc;
    for (int t = threadIdx.x; t < (H + Hkv) * half; t += blockDim.x) {
      const int head = t / half, j = t - head * half;
      const int base = head * hd;  // q heads first, then k heads (contiguous in C)
      float a = csum(c, sstride, splits, base + j), bb = csum(c, sstride, splits, base + j + half);
      if (use_rope) {
        float2 cs = rope_tab[(size_t)i * half + j];
        float a2 = a * cs.x - bb * cs.y;
        float b2 = bb * cs.x + a * cs.y;
        a = a2;
        bb = b2;
      }
      T *dst;
      if (head < H) {
        dst = Q + (size_t)r * H * hd + (size_t)head * hd;
      } else {
        const int kvh = head - H;
        dst = Kc + (((size_t)b * Hkv + kvh) * N + i) * hd;
      }
      dst[j] = from_f<T>(a);
      dst[j + half] = from_f<T>(bb);
    }
    const float *cv = c + (size_t)(H + Hkv) * hd;
    for (int t = threadIdx.x; t < Hkv * hd; t += blockDim.x) {
      const int kvh = t / hd, j = t - kvh * hd;
      Vc[(((size_t)b * Hkv + kvh) * N + i) * hd + j] = from_f<T>(csum(cv, sstride, splits, t));
    }
  }
}

cudaError_t launch_epi_qkv(int dtype, const float *C, int ldc, int splits, size_t sstride, const int32_t *rowmap,
                           const int32_t *m_total, int cap, int N, int H, int Hkv, int hd, const float2 *rope_tab,
                           int use_rope, void *Q, void *Kc, void *Vc, cudaStream_t s) {
  if (dtype == DCU_BF16)
    k_epi_qkv<bf16><<<row_grid(cap), 256, 0, s>>>(C, ldc, splits, sstride, rowmap, m_total, N, H, Hkv, hd, rope_tab, use_rope,
                                                   (bf16 *)Q, (bf16 *)Kc, (bf16 *)Vc);
  else
    k_epi_qkv<float><<<row_grid(cap), 256, 0, s>>>(C, ldc, splits, sstride, rowmap, m_total, N, H, Hkv, hd, rope_tab, use_rope,
                                                    (float *)Q, (float *)Kc, (float *)Vc);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ O epilogue
// hmid[r] = H_l[row] + C[r] (fp32); xs[r] = T(RMSNorm(hmid[r]) * g2).
template <class T>
__global__ void k_epi_o(const float *__restrict__ C, int ldc, int splits, size_t sstride,
                        const int32_t *__restrict__ rowmap,
                        const int32_t *__restrict__ m_total, const T *__restrict__ Hl, const float *__restrict__ g2,
                        float eps, int D, float *__restrict__ hmid, T *__restrict__ xs) {
  __shared__ double red[32];
  constexpr int VN = Vec<T>::n;
  const int M = *m_total;
  for (int r = blockIdx.x; r < M; r += gridDim.x) {
    const T *x = Hl + (size_t)rowmap[r] * D;
    const float *c = C + (size_t)r * ldc;
    float *hm = hmid + (size_t)r * D;
    double ss = 0;
    for (int j = threadIdx.x * VN; j < D; j += blockDim.x * VN) {
      float v[VN];
      load_vec(x + j, v);
#pragma unroll
      for (int i = 0; i < VN; ++i) {
        v[i] += csum(c, sstride, splits, j + i);
        hm[j + i] = v[i];
        ss += (double)v[i] * (double)v[i];
      }
    }
    ss = block_sum(ss, red);
    const float inv = (float)(1.0 / sqrt(ss / (double)D + (double)eps));
    T *o = xs + (size_t)r * D;
    for (int j = threadIdx.x * VN; j < D; j += blockDim.x * VN) {
      float v[VN];
#pragma unroll
      for (int i = 0; i < VN; ++i) v[i] = hm[j + i] * inv * g2[j + i];
      store_vec(o + j, v);
    }
  }
}

cudaError_t launch_epi_o(int dtype, const float *C, int ldc, int splits, size_t sstride, const int32_t *rowmap,
                         const int32_t *m_total, int cap, const void *Hl, const float *g2, float eps, int D,
                         float *hmid, void *xs, cudaStream_t s) {
  if (dtype == DCU_BF16)
    k_epi_o<bf16><<<row_grid(cap), 256, 0, s>>>(C, ldc, splits, sstride, rowmap, m_total, (const bf16 *)Hl, g2, eps, D, hmid,
                                                 (bf16 *)xs);
  else
    k_epi_o<float><<<row_grid(cap), 256, 0, s>>>(C, ldc, splits, sstride, rowmap, m_total, (const float *)Hl, g2, eps, D, hmid,
                                                  (float *)xs);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ SwiGLU epilogue
// C row r = [gate (F) | up (F)];  act[r] = T(silu(gate) * up).
template <class T>
__global__ void k_epi_swiglu(const float *__restrict__ C, int ldc, int splits, size_t sstride,
                             const int32_t *__restrict__ m_total, int F,
                             T *__restrict__ act) {
  const int M = *m_total;
  for (int r = blockIdx.x; r < M; r += gridDim.x) {
    const float *c = C + (size_t)r * ldc;
    for (int j = threadIdx.x; j < F; j += blockDim.x) {
      const float gt = csum(c, sstride, splits, j), up = csum(c, sstride, splits, F + j);
      act[(size_t)r * F + j] = from_f<T>(gt / (1.0f + expf(-gt)) * up);
    }
  }
}

cudaError_t launch_epi_swiglu(int dtype, const float *C, int ldc, int splits, size_t sstride, const int32_t *m_total,
                              int cap, int F, void *act, cudaStream_t s) {
  if (dtype == DCU_BF16)
    k_epi_swiglu<bf16><<<row_grid(cap), 256, 0, s>>>(C, ldc, splits, sstride, m_total, F, (bf16 *)act);
  else
    k_epi_swiglu<float><<<row_grid(cap), 256, 0, s>>>(C, ldc, splits, sstride, m_total, F, (float *)act);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ down epilogue + scatter
// new = T(hmid[r] + C[r]); if d_next: d_next[row] = distance(new, H_{l+1}[row])
// ([DLLM] "关键设计 1", computed against the cached row before it is
// overwritten); H_{l+1}[row] = new.
template <class T>
__global__ void k_epi_down_scatter(const float *__restrict__ C, int ldc, int splits, size_t sstride,
                                   const int32_t *__restrict__ rowmap,
                                   const int32_t *__restrict__ m_total, const float *__restrict__ hmid,
                                   T *__restrict__ Hn, const float *__restrict__ g_next, float *__restrict__ d_next,
                                   int D) {
  __shared__ double red[32];
  constexpr int VN = Vec<T>::n;
  const int M = *m_total;
  for (int r = blockIdx.x; r < M; r += gridDim.x) {
    const int row = rowmap[r];
    const float *c = C + (size_t)r * ldc;
    const float *hm = hmid + (size_t)r * D;
    T *dst = Hn + (size_t)row * D;
    double dot = 0, nx = 0, ny = 0;
    bool same = true;
    for (int j = threadIdx.x * VN; j < D; j += blockDim.x * VN) {
      float v[VN];
#pragma unroll
      for (int i = 0; i < VN; ++i) v[i] = hm[j + i] + csum(c, sstride, splits, j + i);
      if (d_next) {
        float ov[VN];
        uint32_t ob[VN];
        load_vec(dst + j, ov, ob);
#pragma unroll
        for (int i = 0; i < VN; ++i) {
          T nt = from_f<T>(v[i]);
          float nv = to_f(nt);
          same = same && (bits_of<T>(nt) == ob[i]);
          double gg = (double)g_next[j + i];
          double a = gg * (double)nv, b = gg * (double)ov[i];
          dot += a * b;
          nx += a * a;
          ny += b * b;
        }
      }
      store_vec(dst + j, v);
    }
    if (d_next) {
      same = __syncthreads_and(same);
      dot = block_sum(dot, red);
      nx = block_sum(nx, red);
      ny = block_sum(ny, red);
      if (threadIdx.x == 0) d_next[row] = finish_cosine_distance(dot, nx, ny, same);
    }
  }
}

cudaError_t launch_epi_down_scatter(int dtype, const float *C, int ldc, int splits, size_t sstride,
                                    const int32_t *rowmap, const int32_t *m_total, int cap, const float *hmid,
                                    void *Hnext, const float *g_next, float *d_next, int D, cudaStream_t s) {
  if (dtype == DCU_BF16)
    k_epi_down_scatter<bf16><<<row_grid(cap), 256, 0, s>>>(C, ldc, splits, sstride, rowmap, m_total, hmid, (bf16 *)Hnext, g_next,
                                                            d_next, D);
  else
    k_epi_down_scatter<float><<<row_grid(cap), 256, 0, s>>>(C, ldc, splits, sstride, rowmap, m_total, hmid, (float *)Hnext, g_next,
                                                             d_next, D);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ softmax-max
// For LM-head row r (position rowmap[r]): c = 1 / sum_v exp(z_v - z_max) and
// the argmax (lowest id among equal maxima) ([FRECHET] "整体框架").
__global__ void k_softmax_max(const float *__restrict__ C, int ldc, const int32_t *__restrict__ rowmap,
                              const int32_t *__restrict__ m_total, int V, float *__restrict__ conf,
                              int32_t *__restrict__ amax) {
  __shared__ float smax[32];
  __shared__ int sidx[32];
  __shared__ double red[32];
  const int M = *m_total;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int r = blockIdx.x; r < M; r += gridDim.x) {
    const float *z = C + (size_t)r * ldc;
    float best = -INFINITY;
    int bi = 0x7fffffff;
    for (int v = threadIdx.x; v < V; v += blockDim.x) {
      float x = z[v];
      if (x > best) { best = x; bi = v; }  // strided ascending: first max of this thread is its lowest id
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      float ob = __shfl_xor_sync(0xffffffffu, best, o);
      int oi = __shfl_xor_sync(0xffffffffu, bi, o);
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
        float ob = __shfl_xor_sync(0xffffffffu, best, o);
        int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ob > best || (ob == best && oi < bi)) { best = ob; bi = oi; }
      }
      if (lane == 0) { smax[0] = best; sidx[0] = bi; }
    }
    __syncthreads();
    const float zmax = smax[0];
    const int arg = sidx[0];
    double sum = 0;
    for (int v = threadIdx.x; v < V; v += blockDim.x) sum += (double)expf(z[v] - zmax);
    sum = block_sum(sum, red);
    if (threadIdx.x == 0) {
      const int row = rowmap[r];
      conf[row] = (float)(1.0 / sum);
      amax[row] = arg;
    }
  }
}

cudaError_t launch_softmax_max(const float *C, int ldc, const int32_t *rowmap, const int32_t *m_total, int cap,
                               int V, float *conf, int32_t *amax, cudaStream_t s) {
  k_softmax_max<<<row_grid(cap), 512, 0, s>>>(C, ldc, rowmap, m_total, V, conf, amax);
  return cudaGetLastError();
}

}  // namespace dcu
