// Row-parallel kernels of the DCU step: layer-0 refresh, token dynamics,
// gather + RMSNorm, GEMM epilogues (RoPE + K/V write, residual + RMSNorm,
// SwiGLU, residual + scatter + next-layer dynamics) and the softmax-max of the
// LM head.  One CTA per row (grid-stride), 16-byte vector accesses along the
// row; HBM-bound.
#include "common.cuh"
#include "gemm_tc.h"
#include "kernels.h"

namespace dcu {

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
                                const float *__restrict__ g0, int BN, int D, int V, int full, int32_t *status,
                                uint8_t *__restrict__ stale0) {
  pdl_enter();
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
      if (stale0 && !same) stale0[r] = 1;  // H_0 row changed: layer 0 has not recomputed it yet
    }
  }
}

cudaError_t launch_embed_refresh(int dtype, const int32_t *ids, int32_t *prev_ids, const void *embed, void *H0,
                                 float *d0, const float *g0, int BN, int D, int V, int full, int32_t *status,
                                 uint8_t *stale0, cudaStream_t s) {
  if (BN <= 0) return cudaSuccess;
  if (dtype == DCU_BF16)
    launch_pdl(k_embed_refresh<bf16>, row_grid(BN), 256, 0, s, ids, prev_ids, (const bf16 *)embed, (bf16 *)H0, d0, g0, BN,
                                                        D, V, full, status, stale0);
  else
    launch_pdl(k_embed_refresh<float>, row_grid(BN), 256, 0, s, ids, prev_ids, (const float *)embed, (float *)H0, d0, g0,
                                                         BN, D, V, full, status, stale0);
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
// xs[r] = T(H[rowmap[r]] / sqrt(mean(H^2) + eps) * g) for r < *m_total.  The
// row stays in registers between the sum of squares and the scaling (rows of
// up to 256 threads x 4 vectors; longer rows are re-read).
template <class T>
__global__ void k_gather_norm(const int32_t *__restrict__ rowmap, const int32_t *__restrict__ m_total,
                              const T *__restrict__ H, const float *__restrict__ g, float eps, int D,
                              T *__restrict__ xs) {
  pdl_enter();
  __shared__ double red[32];
  constexpr int VN = Vec<T>::n;
  constexpr int KEEP = 4;
  const int M = *m_total;
  const int step = blockDim.x * VN;
  for (int r = blockIdx.x; r < M; r += gridDim.x) {
    const T *x = H + (size_t)rowmap[r] * D;
    float keep[KEEP][VN];
    double ss = 0;
#pragma unroll
    for (int q = 0; q < KEEP; ++q) {
      const int j = threadIdx.x * VN + q * step;
      if (j < D) {
        load_vec(x + j, keep[q]);
#pragma unroll
        for (int i = 0; i < VN; ++i) ss += (double)keep[q][i] * (double)keep[q][i];
      }
    }
    for (int j = threadIdx.x * VN + KEEP * step; j < D; j += step) {
      float v[VN];
      load_vec(x + j, v);
#pragma unroll
      for (int i = 0; i < VN; ++i) ss += (double)v[i] * (double)v[i];
    }
    ss = block_sum(ss, red);
    const float inv = (float)(1.0 / sqrt(ss / (double)D + (double)eps));
    T *o = xs + (size_t)r * D;
#pragma unroll
    for (int q = 0; q < KEEP; ++q) {
      const int j = threadIdx.x * VN + q * step;
      if (j < D) {
#pragma unroll
        for (int i = 0; i < VN; ++i) keep[q][i] = keep[q][i] * inv * g[j + i];
        store_vec(o + j, keep[q]);
      }
    }
    for (int j = threadIdx.x * VN + KEEP * step; j < D; j += step) {
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
    launch_pdl(k_gather_norm<bf16>, row_grid(cap), 256, 0, s, rowmap, m_total, (const bf16 *)H, g, eps, D, (bf16 *)xs);
  else
    launch_pdl(k_gather_norm<float>, row_grid(cap), 256, 0, s, rowmap, m_total, (const float *)H, g, eps, D, (float *)xs);
  return cudaGetLastError();
}

// Pieces of column j's 128-wide tile (1 when geo.grid == 0).  The piece tables
// are written when a geometry is first used, long before an epilogue reads them.
__device__ __forceinline__ int slot_count(const SlotGeo &geo, size_t j) {
  return geo.grid <= 0 ? 1 : (geo.nslots ? __ldg(geo.nslots + (j >> 7)) : sk_nslots(geo, (int)(j >> 7)));
}

// 4 consecutive GEMM outputs (j % 4 == 0) summed over their ns pieces in slot
// order; the loads of up to K pieces are all issued before the first add (a
// tile of the 32-tile GEMMs over 148 CTAs has up to 6 pieces).
template <int K = 8>
__device__ __forceinline__ float4 csum4n(const float *c, long long stride, size_t j, int ns) {
  float4 w[K];
#pragma unroll
  for (int sp = 0; sp < K; ++sp)
    if (sp < ns) w[sp] = *reinterpret_cast<const float4 *>(c + (size_t)sp * (size_t)stride + j);
  float4 v = w[0];
#pragma unroll
  for (int sp = 1; sp < K; ++sp)
    if (sp < ns) {
      v.x += w[sp].x;
      v.y += w[sp].y;
      v.z += w[sp].z;
      v.w += w[sp].w;
    }
  for (int sp = K; sp < ns; ++sp) {
    const float4 u = *reinterpret_cast<const float4 *>(c + (size_t)sp * (size_t)stride + j);
    v.x += u.x;
    v.y += u.y;
    v.z += u.z;
    v.w += u.w;
  }
  return v;
}

// The same sum with one load in flight at a time: few registers, for the
// flattened epilogues whose occupancy matters more than one row's latency.
__device__ __forceinline__ float4 csum4(const float *c, const SlotGeo &geo, size_t j) {
  float4 v = *reinterpret_cast<const float4 *>(c + j);
  const int ns = slot_count(geo, j);
  for (int sp = 1; sp < ns; ++sp) {
    const float4 w = *reinterpret_cast<const float4 *>(c + (size_t)sp * (size_t)geo.slot_stride + j);
    v.x += w.x;
    v.y += w.y;
    v.z += w.z;
    v.w += w.w;
  }
  return v;
}

// The row epilogues (O, down) run right after a GEMM under programmatic
// dependent launch.  Only the GEMM's slots come from the launch they wait for;
// the row count, the row plan, the piece tables and the other operands were
// written two or more launches earlier (final once this launch has started),
// so they are loaded before the wait and only the slot loads follow it.

// Two such sums (columns ja and jb of one packed row) with their loads
// interleaved: each column summed in slot order as csum4 does, two loads in
// flight instead of one.
__device__ __forceinline__ void csum4x2(const float *c, const SlotGeo &geo, size_t ja, size_t jb, float4 &va,
                                        float4 &vb) {
  va = *reinterpret_cast<const float4 *>(c + ja);
  vb = *reinterpret_cast<const float4 *>(c + jb);
  const int na = slot_count(geo, ja), nb = slot_count(geo, jb);
  const int n = na > nb ? na : nb;
  for (int sp = 1; sp < n; ++sp) {
    const float *cs = c + (size_t)sp * (size_t)geo.slot_stride;
    if (sp < na) {
      const float4 w = *reinterpret_cast<const float4 *>(cs + ja);
      va.x += w.x;
      va.y += w.y;
      va.z += w.z;
      va.w += w.w;
    }
    if (sp < nb) {
      const float4 w = *reinterpret_cast<const float4 *>(cs + jb);
      vb.x += w.x;
      vb.y += w.y;
      vb.z += w.z;
      vb.w += w.w;
    }
  }
}

template <class T>
__device__ __forceinline__ void store4(T *p, float a, float b, float c, float d);
template <>
__device__ __forceinline__ void store4<float>(float *p, float a, float b, float c, float d) {
  *reinterpret_cast<float4 *>(p) = make_float4(a, b, c, d);
}
template <>
__device__ __forceinline__ void store4<bf16>(bf16 *p, float a, float b, float c, float d) {
  __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t *>(&lo);
  u.y = *reinterpret_cast<uint32_t *>(&hi);
  *reinterpret_cast<uint2 *>(p) = u;
}

// Grid of the flattened (row, 4-column) epilogues: at most 4 CTAs of 256
// threads per SM, so half of each SM's thread slots stay free for the next
// GEMM's CTAs, which programmatic dependent launch schedules while these run.
static inline int flat_grid(long long items_cap) {
  long long g = (items_cap + 255) / 256;
  if (g > 148 * 4) g = 148 * 4;
  return g > 0 ? (int)g : 1;
}

// ------------------------------------------------------------------ QKV epilogue
// C row r = [q (H*hd) | k (Hkv*hd) | v (Hkv*hd)].  RoPE (rotate-half) on q and
// k at the row's position; q -> Q[r]; k, v -> the layer's K/V cache at
// (b, kv head, i).  Work items of 4 consecutive pairs (RoPE) or 4 consecutive
// v values, flattened over all rows so every SM has loads in flight.
template <class T>
__global__ void k_epi_qkv(const float *__restrict__ C, int ldc, const SlotGeo geo,
                          const int32_t *__restrict__ rowmap, const int32_t *__restrict__ m_total, int N, int H,
                          int Hkv, int hd, const float2 *__restrict__ rope_tab, int use_rope, T *__restrict__ Q,
                          T *__restrict__ Kc, T *__restrict__ Vc, uint8_t *__restrict__ stale) {
  const int M = *m_total;
  const int half = hd / 2;
  const int n_rope = (H + Hkv) * half / 4, n_v = Hkv * hd / 4;
  const int per_row = n_rope + n_v;
  // the first item's row and RoPE factors (written long before this launch),
  // loaded before the wait for the QKV GEMM
  const long long it0 = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  int row0 = 0;
  float2 cs0[4];
  if (it0 < (long long)M * per_row) {
    const int r = (int)(it0 / per_row), u = (int)(it0 - (long long)r * per_row);
    row0 = rowmap[r];
    if (u < n_rope && use_rope) {
      const int t = u * 4, head = t / half, j = t - head * half;
      const int i = row0 - (row0 / N) * N;
#pragma unroll
      for (int e = 0; e < 4; ++e) cs0[e] = rope_tab[(size_t)i * half + j + e];
    }
  }
  pdl_enter();
  for (long long it = it0; it < (long long)M * per_row; it += (long long)gridDim.x * blockDim.x) {
    const bool first = it == it0;
    const int r = (int)(it / per_row), u = (int)(it - (long long)r * per_row);
    const int row = first ? row0 : rowmap[r];
    const int b = row / N, i = row - b * N;
    const float *c = C + (size_t)r * ldc;
    if (u < n_rope) {
      const int t = u * 4;
      const int head = t / half, j = t - head * half;
      const int base = head * hd;  // q heads first, then k heads (contiguous in C)
      float4 a, bb;
      csum4x2(c, geo, base + j, base + j + half, a, bb);
      float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {bb.x, bb.y, bb.z, bb.w};
      if (use_rope) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 cs = first ? cs0[e] : rope_tab[(size_t)i * half + j + e];
          const float a2 = av[e] * cs.x - bv[e] * cs.y;
          const float b2 = bv[e] * cs.x + av[e] * cs.y;
          av[e] = a2;
          bv[e] = b2;
        }
      }
      T *dst = head < H ? Q + (size_t)r * H * hd + (size_t)head * hd
                        : Kc + (((size_t)b * Hkv + (head - H)) * N + i) * hd;
      store4<T>(dst + j, av[0], av[1], av[2], av[3]);
      store4<T>(dst + j + half, bv[0], bv[1], bv[2], bv[3]);
    } else {
      const int t = (u - n_rope) * 4;
      const int kvh = t / hd, j = t - kvh * hd;
      if (t == 0 && stale) stale[row] = 0;  // the layer recomputes this row
      const float4 v = csum4(c, geo, (size_t)(H + Hkv) * hd + t);
      store4<T>(Vc + (((size_t)b * Hkv + kvh) * N + i) * hd + j, v.x, v.y, v.z, v.w);
    }
  }
}

cudaError_t launch_epi_qkv(int dtype, const float *C, int ldc, const SlotGeo geo, const int32_t *rowmap,
                           const int32_t *m_total, int cap, int N, int H, int Hkv, int hd, const float2 *rope_tab,
                           int use_rope, void *Q, void *Kc, void *Vc, uint8_t *stale, cudaStream_t s) {
  const long long items = (long long)cap * ((H + Hkv) * (hd / 2) / 4 + Hkv * hd / 4);
  if (dtype == DCU_BF16)
    launch_pdl(k_epi_qkv<bf16>, flat_grid(items), 256, 0, s, C, ldc, geo, rowmap, m_total, N, H, Hkv, hd,
                                                      rope_tab, use_rope, (bf16 *)Q, (bf16 *)Kc, (bf16 *)Vc, stale);
  else
    launch_pdl(k_epi_qkv<float>, flat_grid(items), 256, 0, s, C, ldc, geo, rowmap, m_total, N, H, Hkv, hd,
                                                       rope_tab, use_rope, (float *)Q, (float *)Kc, (float *)Vc, stale);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ O epilogue
// hmid[r] = H_l[row] + C[r] (fp32); xs[r] = T(RMSNorm(hmid[r]) * g2).  One CTA
// of 512 threads per row, 8 consecutive elements per thread per pass.
template <class T>
__global__ void __launch_bounds__(512)
    k_epi_o(const float *__restrict__ C, int ldc, const SlotGeo geo, const int32_t *__restrict__ rowmap,
            const int32_t *__restrict__ m_total, const T *__restrict__ Hl, const float *__restrict__ g2, float eps,
            int D, float *__restrict__ hmid, T *__restrict__ xs) {
  __shared__ double red[32];
  const int M = *m_total;
  const int r0 = blockIdx.x, j0 = threadIdx.x * 8;
  // the first row's operands other than the slots, before the wait
  const bool pre = r0 < M && j0 < D;
  int row0 = 0, ns0 = 1;
  float xv[8], gv[8];
  if (pre) {
    row0 = rowmap[r0];
    const T *x = Hl + (size_t)row0 * D + j0;
    if (Vec<T>::n == 8) {
      load_vec(x, *reinterpret_cast<float(*)[Vec<T>::n]>(xv));
    } else {
      load_vec(x, *reinterpret_cast<float(*)[Vec<T>::n]>(xv));
      load_vec(x + 4, *reinterpret_cast<float(*)[Vec<T>::n]>(xv + 4));
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) gv[e] = g2[j0 + e];
    ns0 = slot_count(geo, j0);
  }
  griddep_wait();
  allow_dependents();
  for (int r = r0; r < M; r += gridDim.x) {
    const bool first = r == r0;
    const int row = first ? row0 : rowmap[r];
    const T *x = Hl + (size_t)row * D;
    const float *c = C + (size_t)r * ldc;
    float *hm = hmid + (size_t)r * D;
    double ss = 0;
    for (int j = j0; j < D; j += blockDim.x * 8) {
      const bool p0 = first && j == j0;
      float v[8];
      if (p0) {
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = xv[e];
      } else if (Vec<T>::n == 8) {
        load_vec(x + j, *reinterpret_cast<float(*)[Vec<T>::n]>(v));
      } else {
        load_vec(x + j, *reinterpret_cast<float(*)[Vec<T>::n]>(v));
        load_vec(x + j + 4, *reinterpret_cast<float(*)[Vec<T>::n]>(v + 4));
      }
      const int ns = p0 ? ns0 : slot_count(geo, j);  // j and j + 4 share their tile
      const float4 c0 = csum4n<6>(c, geo.slot_stride, j, ns), c1 = csum4n<6>(c, geo.slot_stride, j + 4, ns);
      v[0] += c0.x; v[1] += c0.y; v[2] += c0.z; v[3] += c0.w;
      v[4] += c1.x; v[5] += c1.y; v[6] += c1.z; v[7] += c1.w;
      *reinterpret_cast<float4 *>(hm + j) = make_float4(v[0], v[1], v[2], v[3]);
      *reinterpret_cast<float4 *>(hm + j + 4) = make_float4(v[4], v[5], v[6], v[7]);
#pragma unroll
      for (int e = 0; e < 8; ++e) ss += (double)v[e] * (double)v[e];
    }
    ss = block_sum(ss, red);
    const float inv = (float)(1.0 / sqrt(ss / (double)D + (double)eps));
    T *o = xs + (size_t)r * D;
    for (int j = j0; j < D; j += blockDim.x * 8) {
      const float4 h0 = *reinterpret_cast<const float4 *>(hm + j), h1 = *reinterpret_cast<const float4 *>(hm + j + 4);
      float g[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) g[e] = (first && j == j0) ? gv[e] : g2[j + e];
      store4<T>(o + j, h0.x * inv * g[0], h0.y * inv * g[1], h0.z * inv * g[2], h0.w * inv * g[3]);
      store4<T>(o + j + 4, h1.x * inv * g[4], h1.y * inv * g[5], h1.z * inv * g[6], h1.w * inv * g[7]);
    }
  }
}

cudaError_t launch_epi_o(int dtype, const float *C, int ldc, const SlotGeo geo, const int32_t *rowmap,
                         const int32_t *m_total, int cap, const void *Hl, const float *g2, float eps, int D,
                         float *hmid, void *xs, cudaStream_t s) {
  if (dtype == DCU_BF16)
    launch_pdl(k_epi_o<bf16>, row_grid(cap), 512, 0, s, C, ldc, geo, rowmap, m_total, (const bf16 *)Hl, g2, eps, D,
                                                hmid, (bf16 *)xs);
  else
    launch_pdl(k_epi_o<float>, row_grid(cap), 512, 0, s, C, ldc, geo, rowmap, m_total, (const float *)Hl, g2, eps,
                                                 D, hmid, (float *)xs);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ SwiGLU epilogue
// C row r = [gate (F) | up (F)];  act[r] = T(silu(gate) * up), 4 values per work item.
template <class T>
__global__ void k_epi_swiglu(const float *__restrict__ C, int ldc, const SlotGeo geo,
                             const int32_t *__restrict__ m_total, int F, T *__restrict__ act) {
  pdl_enter();
  const int M = *m_total;
  const int per_row = F / 4;
  for (long long it = blockIdx.x * (long long)blockDim.x + threadIdx.x; it < (long long)M * per_row;
       it += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(it / per_row), j = (int)(it - (long long)r * per_row) * 4;
    const float *c = C + (size_t)r * ldc;
    float4 gt, up;
    csum4x2(c, geo, j, (size_t)F + j, gt, up);
    store4<T>(act + (size_t)r * F + j, gt.x / (1.0f + expf(-gt.x)) * up.x, gt.y / (1.0f + expf(-gt.y)) * up.y,
              gt.z / (1.0f + expf(-gt.z)) * up.z, gt.w / (1.0f + expf(-gt.w)) * up.w);
  }
}

cudaError_t launch_epi_swiglu(int dtype, const float *C, int ldc, const SlotGeo geo, const int32_t *m_total,
                              int cap, int F, void *act, cudaStream_t s) {
  const long long items = (long long)cap * (F / 4);
  if (dtype == DCU_BF16)
    launch_pdl(k_epi_swiglu<bf16>, flat_grid(items), 256, 0, s, C, ldc, geo, m_total, F, (bf16 *)act);
  else
    launch_pdl(k_epi_swiglu<float>, flat_grid(items), 256, 0, s, C, ldc, geo, m_total, F, (float *)act);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ down epilogue + scatter
// new = T(hmid[r] + C[r]); if d_next: d_next[row] = distance(new, H_{l+1}[row])
// ([DLLM] "关键设计 1", computed against the cached row before it is
// overwritten); H_{l+1}[row] = new.  512 threads per row, 8 elements each.
template <class T>
__global__ void __launch_bounds__(512)
    k_epi_down_scatter(const float *__restrict__ C, int ldc, const SlotGeo geo,
                       const int32_t *__restrict__ rowmap, const int32_t *__restrict__ m_total,
                       const float *__restrict__ hmid, T *__restrict__ Hn, const float *__restrict__ g_next,
                       float *__restrict__ d_next, uint8_t *__restrict__ stale_next, int D) {
  __shared__ double red[32];
  constexpr int VN = Vec<T>::n;
  const int M = *m_total;
  const int r0 = blockIdx.x, j0 = threadIdx.x * 8;
  // the first row's operands other than the slots, before the wait: hmid (the
  // O epilogue's, three launches back) and the cached H_{l+1} row that the
  // distance compares against (only this launch rewrites it)
  const bool pre = r0 < M && j0 < D;
  int row0 = 0, ns0 = 1;
  float4 h0p = make_float4(0.f, 0.f, 0.f, 0.f), h1p = h0p;
  float ovp[8];
  uint32_t obp[8];
  if (pre) {
    row0 = rowmap[r0];
    ns0 = slot_count(geo, j0);
    const float *hm = hmid + (size_t)r0 * D;
    h0p = *reinterpret_cast<const float4 *>(hm + j0);
    h1p = *reinterpret_cast<const float4 *>(hm + j0 + 4);
    if (d_next) {
      const T *dst = Hn + (size_t)row0 * D;
#pragma unroll
      for (int q = 0; q < 8; q += VN)
        load_vec(dst + j0 + q, *reinterpret_cast<float(*)[VN]>(ovp + q), *reinterpret_cast<uint32_t(*)[VN]>(obp + q));
    }
  }
  griddep_wait();
  allow_dependents();
  for (int r = r0; r < M; r += gridDim.x) {
    const bool first = r == r0;
    const int row = first ? row0 : rowmap[r];
    const float *c = C + (size_t)r * ldc;
    const float *hm = hmid + (size_t)r * D;
    T *dst = Hn + (size_t)row * D;
    double dot = 0, nx = 0, ny = 0;
    bool same = true;
    for (int j = j0; j < D; j += blockDim.x * 8) {
      const bool p0 = first && j == j0;
      const int ns = p0 ? ns0 : slot_count(geo, j);  // j and j + 4 share their tile
      const float4 c0 = csum4n<6>(c, geo.slot_stride, j, ns), c1 = csum4n<6>(c, geo.slot_stride, j + 4, ns);
      const float4 h0 = p0 ? h0p : *reinterpret_cast<const float4 *>(hm + j);
      const float4 h1 = p0 ? h1p : *reinterpret_cast<const float4 *>(hm + j + 4);
      float v[8] = {h0.x + c0.x, h0.y + c0.y, h0.z + c0.z, h0.w + c0.w,
                    h1.x + c1.x, h1.y + c1.y, h1.z + c1.z, h1.w + c1.w};
      if (d_next) {
        float ov[8];
        uint32_t ob[8];
        if (p0) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            ov[e] = ovp[e];
            ob[e] = obp[e];
          }
        } else {
#pragma unroll
          for (int q = 0; q < 8; q += VN)
            load_vec(dst + j + q, *reinterpret_cast<float(*)[VN]>(ov + q), *reinterpret_cast<uint32_t(*)[VN]>(ob + q));
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const T nt = from_f<T>(v[e]);
          const float nv = to_f(nt);
          same = same && (bits_of<T>(nt) == ob[e]);
          const double gg = (double)g_next[j + e];
          const double a = gg * (double)nv, b = gg * (double)ov[e];
          dot += a * b;
          nx += a * a;
          ny += b * b;
        }
      }
#pragma unroll
      for (int q = 0; q < 8; q += VN) store_vec(dst + j + q, *reinterpret_cast<float(*)[VN]>(v + q));
    }
    if (d_next) {
      same = __syncthreads_and(same);
      dot = block_sum(dot, red);
      nx = block_sum(nx, red);
      ny = block_sum(ny, red);
      if (threadIdx.x == 0) {
        d_next[row] = finish_cosine_distance(dot, nx, ny, same);
        if (stale_next && !same) stale_next[row] = 1;  // H_{l+1} row changed
      }
    }
  }
}

cudaError_t launch_epi_down_scatter(int dtype, const float *C, int ldc, const SlotGeo geo,
                                    const int32_t *rowmap, const int32_t *m_total, int cap, const float *hmid,
                                    void *Hnext, const float *g_next, float *d_next, uint8_t *stale_next, int D,
                                    cudaStream_t s) {
  if (dtype == DCU_BF16)
    launch_pdl(k_epi_down_scatter<bf16>, row_grid(cap), 512, 0, s, C, ldc, geo, rowmap, m_total, hmid,
                                                            (bf16 *)Hnext, g_next, d_next, stale_next, D);
  else
    launch_pdl(k_epi_down_scatter<float>, row_grid(cap), 512, 0, s, C, ldc, geo, rowmap, m_total, hmid,
                                                             (float *)Hnext, g_next, d_next, stale_next, D);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ Value dynamics (select_from = "v")
// For packed stale row r (position rowmap[r] = b * N + i): the recomputed Value
// v = sum of the GEMM's slots over the Hkv * hd columns, rounded to the cache
// dtype, against the cached Value row (all kv heads): d[row] = 1 - cos(v,
// v_cached) in fp64 with the equal-row / zero rules ([DLLM] "关键设计 1", the
// Value comparison it contrasts with the input proxy).  One CTA per row.
template <class T>
__global__ void __launch_bounds__(256)
    k_value_dist(const float *__restrict__ C, int ldc, const SlotGeo geo, const int32_t *__restrict__ rowmap,
                 const int32_t *__restrict__ m_total, int N, int Hkv, int hd, const T *__restrict__ Vc,
                 float *__restrict__ d) {
  pdl_enter();
  __shared__ double red[32];
  const int M = *m_total;
  const int W = Hkv * hd;
  for (int r = blockIdx.x; r < M; r += gridDim.x) {
    const int row = rowmap[r];
    const int b = row / N, i = row - b * N;
    const float *c = C + (size_t)r * ldc;
    double dot = 0, nx = 0, ny = 0;
    bool same = true;
    for (int j = threadIdx.x * 4; j < W; j += blockDim.x * 4) {
      const float4 v = csum4(c, geo, (size_t)j);
      const int kvh = j / hd, jj = j - kvh * hd;
      const T *cv = Vc + (((size_t)b * Hkv + kvh) * N + i) * hd + jj;
      const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const T nt = from_f<T>(vv[e]);
        const T ot = cv[e];
        same = same && (bits_of<T>(nt) == bits_of<T>(ot));
        const double a = (double)to_f(nt), o = (double)to_f(ot);
        dot += a * o;
        nx += a * a;
        ny += o * o;
      }
    }
    same = __syncthreads_and(same);
    dot = block_sum(dot, red);
    nx = block_sum(nx, red);
    ny = block_sum(ny, red);
    if (threadIdx.x == 0) d[row] = finish_cosine_distance(dot, nx, ny, same);
  }
}

cudaError_t launch_value_dist(int dtype, const float *C, int ldc, const SlotGeo geo, const int32_t *rowmap,
                              const int32_t *m_total, int cap, int N, int Hkv, int hd, const void *Vc, float *d,
                              cudaStream_t s) {
  if (dtype == DCU_BF16)
    launch_pdl(k_value_dist<bf16>, row_grid(cap), 256, 0, s, C, ldc, geo, rowmap, m_total, N, Hkv, hd,
               (const bf16 *)Vc, d);
  else
    launch_pdl(k_value_dist<float>, row_grid(cap), 256, 0, s, C, ldc, geo, rowmap, m_total, N, Hkv, hd,
               (const float *)Vc, d);
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
