// Host interface of the tcgen05 GEMM (internal).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dcu {

constexpr int kTcMaxA = 16;                 // deepest weight-tile ring
constexpr int kTcMaxB = 4;                  // deepest activation-tile ring
constexpr int kTcThreads = 224;             // 7 warps: W producer, MMA, 4 epilogue, X producer
constexpr uint32_t kTcABytes = 128u * 128u;  // weight tile: 128 rows x 64 bf16
constexpr size_t kTcSmem = 220u * 1024u;     // dynamic shared memory per CTA (one CTA per SM)

// Stream-K schedule: the flattened (tile, k block) space of one token pass,
// T = n_tiles * kblocks, is cut into G contiguous ranges [c*T/G, (c+1)*T/G)
// (with tile_aligned the cut points are rounded down to whole tiles).  A tile
// is computed in nslots pieces, one per CTA whose range meets it; piece j is
// stored in slot j, so a consumer sums slots 0..nslots-1 of the tile in slot
// order and the result does not depend on CTA scheduling.
struct SlotGeo {
  int n_tiles, kblocks, grid, tile_aligned;
  long long slot_stride;        // elements between two slots (cap * ldc)
  const int32_t *nslots = nullptr;  // device table [n_tiles] of sk_nslots (consumers), or null
};

// (Every product below is at most n_tiles * kblocks * grid; when that fits in
// 32 bits -- every shape of these models -- the divisions run in 32-bit
// arithmetic, which the GPU does natively, with the same results.)
__host__ __device__ inline bool sk_small(const SlotGeo &g) {
  return (unsigned long long)g.n_tiles * (unsigned)g.kblocks * (unsigned)g.grid < (1ull << 32);
}
__host__ __device__ inline long long sk_begin(const SlotGeo &g, int c) {
  if (sk_small(g)) {
    if (g.tile_aligned) return (long long)((unsigned)g.n_tiles * (unsigned)c / (unsigned)g.grid * (unsigned)g.kblocks);
    return (long long)((unsigned)g.n_tiles * (unsigned)g.kblocks * (unsigned)c / (unsigned)g.grid);
  }
  if (g.tile_aligned) return (long long)g.n_tiles * c / g.grid * g.kblocks;
  return (long long)g.n_tiles * g.kblocks * c / g.grid;
}
// CTA whose range holds flattened index x
__host__ __device__ inline int sk_owner(const SlotGeo &g, long long x) {
  const long long T = (long long)g.n_tiles * g.kblocks;
  int c = sk_small(g) ? (int)((unsigned)x * (unsigned)g.grid / (unsigned)T) : (int)((x * (long long)g.grid) / T);
  if (c >= g.grid) c = g.grid - 1;
  while (c + 1 < g.grid && sk_begin(g, c + 1) <= x) ++c;
  while (c > 0 && sk_begin(g, c) > x) --c;
  return c;
}
__host__ __device__ inline int sk_first(const SlotGeo &g, int tile) { return sk_owner(g, (long long)tile * g.kblocks); }
__host__ __device__ inline int sk_nslots(const SlotGeo &g, int tile) {
  return sk_owner(g, (long long)(tile + 1) * g.kblocks - 1) - sk_first(g, tile) + 1;
}

// Epilogue kinds.  EPI_NONE: the pieces stay in their slots (separate
// epilogue kernels sum them).  EPI_LMHEAD: softmax statistics of the LM head.
// The other four are the layer epilogues of a chained launch (see TcParams):
//   EPI_QKV   RoPE (rotate-half) on q and k, q -> Q[r], k / v -> the K/V cache
//   EPI_O     hmid = H_l[row] + o (float); xs = bf16(RMSNorm(hmid) * g2)
//   EPI_GU    act = bf16(silu(gate) * up)
//   EPI_DOWN  new = hmid + down -> H_{l+1}[row] (scatter), next-layer d and
//             stale flag against the cached row before it is overwritten
enum { EPI_NONE = 0, EPI_LMHEAD = 1, EPI_QKV = 2, EPI_O = 3, EPI_GU = 4, EPI_DOWN = 5 };
constexpr int kTcMaxPhases = 3;

// Arguments of the chained epilogues.
struct EpiArgs {
  const int32_t *rowmap;   // packed row -> b * N + i
  int N;                   // sequence length
  // EPI_QKV
  int H, Hkv, hd, use_rope;
  const float2 *rope_tab;  // [max_seq][hd / 2] (cos, sin)
  void *Q, *Kc, *Vc;       // Q [cap][H * hd]; the layer's K / V cache [B][Hkv][N][hd]
  uint8_t *stale_l;        // cleared at the recomputed rows (may be null)
  // EPI_O / EPI_GU / EPI_DOWN
  int D, F;
  float eps;
  const void *Hl;          // layer input rows [B * N][D]
  const float *g2;         // FFN norm gain [D]
  float *hmid;             // [cap][D]
  void *xs;                // [cap][D] bf16, gate|up operand
  void *act;               // [cap][F] bf16, down operand
  void *Hn;                // H_{l+1} rows [B * N][D]
  const float *g_next;     // next layer's attention-norm gain (null: no d)
  float *d_next;           // next layer's d [B * N] (null: no d)
  uint8_t *stale_next;     // set at rows whose H_{l+1} content changed (may be null)
};

// One GEMM of a launch: out[slot][m][n] = the piece `slot` of
// sum_k X[m][k] * W[n][k] over the concatenated weight segments (output
// column of segment s, row r: seg_col0[s] + r; every segment but the last has
// rows % 128 == 0, so column n lies in tile n / 128).
struct TcPhase {
  CUtensorMap a[3];        // weight segments, bf16 [rows][K], box 64 x 128, 128-byte swizzle
  CUtensorMap b;           // packed activations, bf16 [cap][K], box 64 x b_rows, 128-byte swizzle
  int seg_tile0[4];        // first 128-row tile of segment s; seg_tile0[nseg] = n_tiles
  int seg_col0[3];         // first output column of segment s
  int seg_rows[3];         // rows of segment s
  int nseg, ldc;
  SlotGeo geo;             // n_tiles, kblocks, grid, tile_aligned, slot stride, piece table
  int epi;                 // chained launches: the epilogue run after this phase
};

// Kernel parameters (passed as a __grid_constant__ so the tensor maps can be
// addressed by TMA).  A launch runs nphase GEMMs over the same packed rows.
// chain = 0: one GEMM (nphase = 1), its pieces in slots, or the LM head
// (epi_mode 1).  chain = 1 (a cooperative launch, one CTA per SM): after each
// phase every CTA meets a grid barrier, the phase's epilogue runs spread over
// all CTAs, a second barrier publishes its outputs, and the next phase's
// activation loads wait for that barrier while its weight loads have been
// streaming all along.  bar: 2 * nphase counters, zero before the launch.
struct TcParams {
  TcPhase ph[kTcMaxPhases];
  int nphase;
  int chain;
  int32_t *bar;
  int b_rows;              // rows of the activation box: the token pass (BN) or fewer when cap < BN
  // Pass sweep (chain = 0; layer GEMMs and the LM head): when M spans more than one token pass,
  // up to `sweep` passes share each weight tile while it is in shared memory
  // (one activation box per pass in a stage, one TMEM accumulator per pass),
  // so the weights stream from HBM once per group of passes instead of once
  // per pass.  0 or 1: every pass re-streams the weights.  launch_gemm_tc
  // lowers it to what TMEM (512 columns) and the shared memory hold.
  int sweep;
  const int32_t *m_total;  // device row count M (or null: m_host)
  int m_host;
  float *out;              // slots [slot][cap][ldc] (every phase uses the same buffer in turn)
  int32_t *status;         // device status word (DCU_ST_TIMEOUT) or null
  uint32_t smem_bytes;
  // epi_mode 1 (LM head, tile_aligned, BN = 256, one segment): the tokens are
  // the MMA M dimension and the weight tile (128 vocabulary rows) is N; instead
  // of storing logits, CTA c writes per token m its softmax statistics over the
  // vocabulary rows of its whole range: smx[c][m] = (max, sum of exp(z - max)),
  // smx_arg[c][m] = lowest id reaching the max; row pitch ldm.
  int epi_mode;
  float2 *smx;
  int32_t *smx_arg;
  int ldm;
  // epi_mode 1 with zout: the logits of token m are also stored at
  // zout[zrow[m] * ldz + v] (fp32; the next commit's previous logits for APD)
  float *zout;
  const int32_t *zrow;
  int64_t ldz;
  // Prefetch of the next GEMM's weights: after its last TMA load, CTA c
  // prefetches into L2 the first nx_count (tile, k block) units of the ranges
  // of CTAs c, c + grid, ... of the next GEMM's stream-K geometry nx_geo over
  // its weight segments nx_a (0: off).  The next GEMM then finds them in L2.
  CUtensorMap nx_a[3];
  int nx_seg_tile0[4];
  int nx_nseg;
  SlotGeo nx_geo;
  int nx_count;
  EpiArgs e;               // chained epilogues
};

// Row-major bf16 matrix [outer][inner] with row pitch row_bytes, box
// box_inner x box_outer, 128-byte swizzle.  False if the driver entry point is
// missing or the encoding is rejected.
bool encode_tmap_bf16(CUtensorMap *map, const void *ptr, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                      uint32_t box_inner, uint32_t box_outer);
// bn: token rows per pass (128 or 256); the grid is p.ph[0].geo.grid CTAs (a
// cooperative launch when p.chain).
cudaError_t launch_gemm_tc(TcParams p, int bn, cudaStream_t s);
// Most pieces a tile can be cut into under the stream-K split over `grid` CTAs.
int tc_max_slots(int n_tiles, int grid);
// Merges the per-CTA softmax statistics of the LM head (epi_mode 1, n_parts =
// the GEMM's grid): for packed row r (position rowmap[r]), conf =
// 1 / sum_c s_c exp(m_c - M), argmax = the lowest id reaching M = max_c m_c.
cudaError_t launch_lm_combine(const float2 *smx, const int32_t *smx_arg, int n_tiles, int ldm,
                              const int32_t *rowmap, const int32_t *m_total, int cap, float *conf, int32_t *amax,
                              cudaStream_t s);

}  // namespace dcu
