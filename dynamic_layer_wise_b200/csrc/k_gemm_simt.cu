// CUDA-core GEMM C[m][n] = sum_k X[m][k] * W[n][k] (fp32 accumulate) for the
// float32 model and for small shapes: 64x64 output tiles, BK = 16, 256
// threads with 4x4 register tiles.  The row count M is read from the device,
// so one launch serves any recompute set size inside a captured graph.
#include "common.cuh"
#include "kernels.h"

namespace dcu {

namespace {
constexpr int BM = 64, BN = 64, BK = 16;

struct SegTable {
  const void *W[4];
  int row0[5];
  int nseg;
};

template <class T>
__device__ __forceinline__ void load4(const T *p, float (&v)[4]);
template <>
__device__ __forceinline__ void load4<float>(const float *p, float (&v)[4]) {
  float4 u = *reinterpret_cast<const float4 *>(p);
  v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
}
template <>
__device__ __forceinline__ void load4<bf16>(const bf16 *p, float (&v)[4]) {
  uint2 u = *reinterpret_cast<const uint2 *>(p);
  const bf16 *e = reinterpret_cast<const bf16 *>(&u);
  v[0] = __bfloat162float(e[0]); v[1] = __bfloat162float(e[1]);
  v[2] = __bfloat162float(e[2]); v[3] = __bfloat162float(e[3]);
}

template <class T>
__global__ void __launch_bounds__(256) k_gemm_simt(const T *__restrict__ X, int ldx, const int32_t *__restrict__ m_total,
                                                   int m_host, SegTable segs, int ntot, int K, float *__restrict__ C,
                                                   int ldc) {
  __shared__ __align__(16) float As[BK][BM + 4];
  __shared__ __align__(16) float Bs[BK][BN + 4];
  const int M = m_total ? *m_total : m_host;
  const int m_tiles = (M + BM - 1) / BM;
  const int n_tiles = (ntot + BN - 1) / BN;
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  // loader mapping: 64 rows x 16 k = 256 groups of 4 consecutive k
  const int lrow = tid >> 2, lk = (tid & 3) * 4;

  for (int w = blockIdx.x; w < m_tiles * n_tiles; w += gridDim.x) {
    const int nt = w / m_tiles, mt = w - nt * m_tiles;
    const int m0 = mt * BM, n0 = nt * BN;
    // segment of this n tile (segments before the last have rows % BN == 0)
    int sg = 0;
    while (sg + 1 < segs.nseg && n0 >= segs.row0[sg + 1]) ++sg;
    const T *W = reinterpret_cast<const T *>(segs.W[sg]);
    const int wrow0 = segs.row0[sg], wrows = segs.row0[sg + 1] - segs.row0[sg];

    float acc[4][4] = {};
    const int xm = m0 + lrow;
    const int wn = n0 + lrow - wrow0;
    const bool xok = xm < M;
    const bool wok = (n0 + lrow) < ntot && wn < wrows;
    const T *xp = X + (size_t)(xok ? xm : 0) * ldx + lk;
    const T *wp = W + (size_t)(wok ? wn : 0) * K + lk;
    for (int k0 = 0; k0 < K; k0 += BK) {
      float xv[4] = {0.f, 0.f, 0.f, 0.f}, wv[4] = {0.f, 0.f, 0.f, 0.f};
      if (xok) load4<T>(xp + k0, xv);
      if (wok) load4<T>(wp + k0, wv);
      __syncthreads();
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        As[lk + e][lrow] = xv[e];
        Bs[lk + e][lrow] = wv[e];
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < BK; ++kk) {
        float4 a = *reinterpret_cast<const float4 *>(&As[kk][ty * 4]);
        float4 b = *reinterpret_cast<const float4 *>(&Bs[kk][tx * 4]);
        float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int m = m0 + ty * 4 + i;
      if (m >= M) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int n = n0 + tx * 4 + j;
        if (n < ntot) C[(size_t)m * ldc + n] = acc[i][j];
      }
    }
    __syncthreads();
  }
}
}  // namespace

cudaError_t launch_gemm_simt(int dtype, const void *X, int ldx, const int32_t *m_total, int m_cap,
                             const GemmSeg *segs, int nseg, int K, float *C, int ldc, cudaStream_t s) {
  if (m_cap <= 0) return cudaSuccess;
  if (nseg < 1 || nseg > 4 || (K % BK) != 0) return cudaErrorInvalidValue;
  SegTable t{};
  t.nseg = nseg;
  int r = 0;
  for (int i = 0; i < nseg; ++i) {
    t.W[i] = segs[i].W;
    t.row0[i] = r;
    r += segs[i].rows;
  }
  t.row0[nseg] = r;
  const int n_tiles = (r + BN - 1) / BN;
  const long long cap_tiles = (long long)n_tiles * ((m_cap + BM - 1) / BM);
  int grid = (int)(cap_tiles < 148 * 8 ? cap_tiles : 148 * 8);
  if (grid < 1) grid = 1;
  if (dtype == DCU_BF16)
    k_gemm_simt<bf16><<<grid, 256, 0, s>>>((const bf16 *)X, ldx, m_total, m_cap, t, r, K, C, ldc);
  else
    k_gemm_simt<float><<<grid, 256, 0, s>>>((const float *)X, ldx, m_total, m_cap, t, r, K, C, ldc);
  return cudaGetLastError();
}

}  // namespace dcu
