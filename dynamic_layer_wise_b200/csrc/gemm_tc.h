// Host interface of the tcgen05 GEMM (internal).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dcu {

// Kernel parameters (passed as a __grid_constant__ so the tensor maps can be
// addressed by TMA).  Output column of segment s, row r: seg_col0[s] + r.
struct TcParams {
  CUtensorMap a[3];        // weight segments, bf16 [rows][K], box 64 x 128, 128-byte swizzle
  CUtensorMap b;           // packed activations, bf16 [cap][K], box 64 x BN, 128-byte swizzle
  int seg_tile0[4];        // first 128-row tile of segment s; seg_tile0[nseg] = n_tiles
  int seg_col0[3];         // first output column of segment s
  int seg_rows[3];         // rows of segment s
  int nseg, n_tiles, kblocks, splits, ldc;
  const int32_t *m_total;  // device row count M (or null: m_host)
  int m_host;
  float *ws;               // partials [splits][cap][ldc]
  long long split_stride;  // elements between two splits' partials
  int32_t *status;         // device status word (DCU_ST_TIMEOUT)
};

template <int BN>
struct TcCfg {
  static constexpr int STAGES = BN <= 64 ? 8 : (BN <= 128 ? 6 : 4);
  static constexpr uint32_t A_BYTES = 128u * 64u * 2u;
  static constexpr uint32_t B_BYTES = (uint32_t)BN * 64u * 2u;
  static constexpr size_t SMEM = (size_t)STAGES * (A_BYTES + B_BYTES) + 1024;
};

// Row-major bf16 matrix [outer][inner] with row pitch row_bytes, box
// box_inner x box_outer, 128-byte swizzle.  False if the driver entry point is
// missing or the encoding is rejected.
bool encode_tmap_bf16(CUtensorMap *map, const void *ptr, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                      uint32_t box_inner, uint32_t box_outer);
int choose_splits(int n_tiles, int kblocks, int passes, int num_sms);
cudaError_t launch_gemm_tc(const TcParams &p, int bn, int grid, cudaStream_t s);

}  // namespace dcu
