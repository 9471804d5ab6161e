// Adaptive parallel decoding (APD), [DLLM] "关键设计 3": per candidate position
// the confidence concentration c = 1 - (second-highest probability), the
// temporal instability H = 1 - cos(p, p_prev) of the full probability vectors
// of adjacent commit steps, and the threshold update tau <- tau - alpha c +
// beta H.  The commit rule (DCU_APD in k_commit_rule) then unmasks every
// candidate whose confidence reaches its own tau.
#include "common.cuh"
#include "kernels.h"

namespace dcu {

// tau[r] = tau0, has_prev[r] = 0 for r < n (a new generation).
__global__ void k_apd_reset(float *__restrict__ tau, uint8_t *__restrict__ has_prev, int64_t n, float tau0) {
  pdl_enter();
  for (int64_t r = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; r < n; r += (int64_t)gridDim.x * blockDim.x) {
    tau[r] = tau0;
    has_prev[r] = 0;
  }
}

cudaError_t launch_apd_reset(float *tau, uint8_t *has_prev, int64_t n, float tau0, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const int64_t g = (n + 255) / 256;
  launch_pdl(k_apd_reset, (int)(g < 148 * 4 ? g : 148 * 4), 256, 0, s, tau, has_prev, n, tau0);
  return cudaGetLastError();
}

// One CTA per packed candidate row r < *m_total (position pos = rowmap[r]).
// z: this step's logits of the row, at z_cur + (by_pos ? pos : r) * ld_cur;
// with z_copy, the row is also copied to z_copy + pos * V (the next step's
// previous logits).  z_prev + pos * V holds the previous step's logits when
// has_prev[pos].  fp64 sums of float32 exponentials.
__global__ void __launch_bounds__(256)
    k_apd_signals(const float *__restrict__ z_cur, int64_t ld_cur, int by_pos, float *__restrict__ z_copy,
                  const float *__restrict__ z_prev, const int32_t *__restrict__ rowmap,
                  const int32_t *__restrict__ m_total, int V, uint8_t *__restrict__ has_prev, float *__restrict__ tau,
                  float alpha, float beta, float *__restrict__ out_c, float *__restrict__ out_h) {
  pdl_enter();
  __shared__ float s1[32], s2[32];
  __shared__ double red[32];
  const int M = *m_total;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int r = blockIdx.x; r < M; r += gridDim.x) {
    const int pos = rowmap[r];
    const float *z = z_cur + (int64_t)(by_pos ? pos : r) * ld_cur;
    const bool prev = has_prev[pos] != 0;
    const float *zp = z_prev + (int64_t)pos * V;
    // pass 1: the two largest logits (a tie at the top counts twice) and the previous maximum
    float a1 = -INFINITY, a2 = -INFINITY, pm = -INFINITY;
    for (int v = threadIdx.x; v < V; v += blockDim.x) {
      const float x = z[v];
      if (x > a1) {
        a2 = a1;
        a1 = x;
      } else if (x > a2) {
        a2 = x;
      }
      if (prev) pm = fmaxf(pm, zp[v]);
      if (z_copy) z_copy[(int64_t)pos * V + v] = x;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float b1 = __shfl_xor_sync(0xffffffffu, a1, o), b2 = __shfl_xor_sync(0xffffffffu, a2, o);
      const float hi = fmaxf(a1, b1), lo = fmaxf(fminf(a1, b1), fmaxf(a2, b2));
      a1 = hi;
      a2 = lo;
      pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, o));
    }
    __syncthreads();
    if (lane == 0) {
      s1[w] = a1;
      s2[w] = a2;
      red[w] = (double)pm;
    }
    __syncthreads();
    a1 = -INFINITY;
    a2 = -INFINITY;
    pm = -INFINITY;
    for (int i = 0; i < nw; ++i) {
      const float hi = fmaxf(a1, s1[i]), lo = fmaxf(fminf(a1, s1[i]), fmaxf(a2, s2[i]));
      a1 = hi;
      a2 = lo;
      pm = fmaxf(pm, (float)red[i]);
    }
    __syncthreads();
    // pass 2: S = sum e, Q = sum e^2, P = sum e'^2, X = sum e e' with e = exp(z - a1), e' = exp(z' - pm)
    double S = 0.0, Q = 0.0, P = 0.0, X = 0.0;
    for (int v = threadIdx.x; v < V; v += blockDim.x) {
      const double e = (double)expf(z[v] - a1);
      S += e;
      Q += e * e;
      if (prev) {
        const double ep = (double)expf(zp[v] - pm);
        P += ep * ep;
        X += e * ep;
      }
    }
    S = block_sum(S, red);
    Q = block_sum(Q, red);
    P = block_sum(P, red);
    X = block_sum(X, red);
    if (threadIdx.x == 0) {
      const double c = 1.0 - (double)expf(a2 - a1) / S;
      double h = 0.0;
      if (prev && Q > 0.0 && P > 0.0) {
        h = 1.0 - X / (sqrt(Q) * sqrt(P));
        h = h < 0.0 ? 0.0 : (h > 2.0 ? 2.0 : h);
      }
      tau[pos] = (float)((double)tau[pos] - (double)alpha * c + (double)beta * h);
      has_prev[pos] = 1;
      out_c[pos] = (float)c;
      out_h[pos] = (float)h;
    }
  }
}

cudaError_t launch_apd_signals(const float *z_cur, int64_t ld_cur, int by_pos, float *z_copy, const float *z_prev,
                               const int32_t *rowmap, const int32_t *m_total, int cap, int V, uint8_t *has_prev,
                               float *tau, float alpha, float beta, float *out_c, float *out_h, cudaStream_t s) {
  const int grid = cap < 148 * 4 ? (cap > 0 ? cap : 1) : 148 * 4;
  launch_pdl(k_apd_signals, grid, 256, 0, s, z_cur, ld_cur, by_pos, z_copy, z_prev, rowmap, m_total, V, has_prev,
             tau, alpha, beta, out_c, out_h);
  return cudaGetLastError();
}

}  // namespace dcu
