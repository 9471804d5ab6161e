// tcgen05 (5th-generation tensor core) GEMM for the bf16 recompute projections,
// FFN and LM head:  ws[split][m][n] = sum_{k in split} X[m][k] * W[n][k].
//
// Swap-AB: the weight rows are the MMA M dimension (128-row tiles, K-major,
// TMA-loaded with the 128-byte swizzle) and the selected tokens are the MMA N
// dimension (a BN-row K-major tile of the packed activations), so a recompute
// set of ~65 rows still drives full 128-row tensor-core instructions while
// every weight byte is read from HBM once.  Accumulators live in TMEM.
//
// Warp roles (224 threads, one CTA per SM, persistent over work units):
//   warp 0      weight producer (one lane): deep ring of 16 KB W tiles; it
//               starts before the previous launch has finished (weights are
//               never written by a kernel)
//   warp 6      activation producer (one lane): shallow ring of X tiles (from
//               L2, one TMA box of the whole token pass per stage), after the
//               programmatic-dependency wait
//   warp 1      TMEM allocator + MMA issuer (one lane): 4 x tcgen05.mma (K=16)
//               per 64-wide k block, tcgen05.commit frees both smem stages
//   warps 2..5  epilogue: tcgen05.ld of the 128 x BN fp32 tile, coalesced
//               stores of the split-K partial (32 lanes = 32 consecutive n)
// A work unit is (weight tile, k split, token pass); the row count M is read
// from the device, so one launch serves any recompute-set size inside a graph.
// Every mbarrier wait is bounded: on expiry the CTA sets DCU_ST_TIMEOUT,
// drains its own copies / MMAs in flight, frees TMEM and exits.
#include <cuda.h>

#include "common.cuh"
#include "gemm_tc.h"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace dcu {
namespace {

struct Frag {
  int tile, kb0, kb1, seg, arow, slot;
};

// Fragment iterator over this CTA's stream-K range, pass by pass.
struct FragIter {
  long long pos, end;
  int pass;
};

__device__ __forceinline__ bool next_frag(const TcParams &p, int passes, FragIter &it, Frag &f) {
  while (it.pos >= it.end) {
    if (++it.pass >= passes) return false;
    it.pos = sk_begin(p.geo, blockIdx.x);
  }
  const int KB = p.geo.kblocks;
  const int t = (int)(it.pos / KB);
  const int kb0 = (int)(it.pos - (long long)t * KB);
  const long long left = it.end - it.pos;
  const int kb1 = (int)((long long)kb0 + left < KB ? kb0 + left : KB);
  it.pos += kb1 - kb0;
  f.tile = t;
  f.kb0 = kb0;
  f.kb1 = kb1;
  int seg = 0;
  while (seg + 1 < p.nseg && t >= p.seg_tile0[seg + 1]) ++seg;
  f.seg = seg;
  f.arow = (t - p.seg_tile0[seg]) * 128;
  f.slot = (int)blockIdx.x - sk_first(p.geo, t);
  return true;
}



// Position in this CTA's (fragment, k block) sequence.
struct KCursor {
  FragIter it;
  Frag f;
  int kb, m0, nb;
  bool valid;
  __device__ __forceinline__ void load_frag(int BN, int M) {
    kb = f.kb0;
    m0 = it.pass * BN;
    nb = (min(BN, M - m0) + 15) / 16;
  }
  __device__ __forceinline__ void start(const TcParams &p, int passes, long long b, long long e, int BN, int M) {
    it = FragIter{b, e, 0};
    valid = next_frag(p, passes, it, f);
    if (valid) load_frag(BN, M);
  }
  __device__ __forceinline__ void advance(const TcParams &p, int passes, int BN, int M) {
    if (++kb < f.kb1) return;
    valid = next_frag(p, passes, it, f);
    if (valid) load_frag(BN, M);
  }
};

template <int BN>
__global__ void __launch_bounds__(kTcThreads, 1) k_gemm_tc(const __grid_constant__ TcParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[2 * kTcMaxA + 2 * kTcMaxB + 5];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  // The row count is written by the select / plan kernel two launches before
  // this one, so it is final even while the previous launch still runs.
  const int M = p.m_total ? *p.m_total : p.m_host;
  if (M <= 0) return;
  const int passes = (M + BN - 1) / BN;
  const long long my_begin = sk_begin(p.geo, blockIdx.x), my_end = sk_begin(p.geo, blockIdx.x + 1);
  if (my_begin >= my_end) return;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Two rings: weight tiles (16 KB, from HBM) and activation tiles (16-row
  // boxes of the rows actually loaded, from L2).  The activation ring only has
  // to cover the L2 latency, so most of shared memory holds weight tiles in
  // flight.
  const uint32_t b_bytes = (uint32_t)p.b_rows * 128u;            // one TMA box per stage
  const uint32_t b_stage = (b_bytes + 1023u) & ~1023u;             // 1024-byte aligned stages
  const int SB = b_stage > 16384u ? 3 : 4;
  int SA = (int)((p.smem_bytes - 1024u - (uint32_t)SB * b_stage) / kTcABytes);
  SA = SA > kTcMaxA ? kTcMaxA : SA;
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t bbase = sbase + (uint32_t)SA * kTcABytes;
  const uint32_t bar0 = smem_u32(bars);
  // two TMEM accumulators (columns [0, BN) and [BN, 2 BN)) alternate between fragments
#define FULL_A(s) (bar0 + 8u * (uint32_t)(s))
#define EMPTY_A(s) (bar0 + 8u * (uint32_t)(kTcMaxA + (s)))
#define FULL_B(s) (bar0 + 8u * (uint32_t)(2 * kTcMaxA + (s)))
#define EMPTY_B(s) (bar0 + 8u * (uint32_t)(2 * kTcMaxA + kTcMaxB + (s)))
  const uint32_t tfull0 = bar0 + 8u * (uint32_t)(2 * kTcMaxA + 2 * kTcMaxB), tempty0 = tfull0 + 16u,
                 drain = tfull0 + 32u;
#define TFULL(a) (tfull0 + 8u * (uint32_t)(a))
#define TEMPTY(a) (tempty0 + 8u * (uint32_t)(a))
#define STAGE_A(s) (sbase + (uint32_t)(s) * kTcABytes)
#define STAGE_B(s) (bbase + (uint32_t)(s) * b_stage)

  if (threadIdx.x == 0) {
    for (int s = 0; s < SA; ++s) {
      mbar_init(FULL_A(s), 1);
      mbar_init(EMPTY_A(s), 1);
    }
    for (int s = 0; s < SB; ++s) {
      mbar_init(FULL_B(s), 1);
      mbar_init(EMPTY_B(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(TFULL(a), 1);
      mbar_init(TEMPTY(a), 4);
    }
    mbar_init(drain, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_slot), 2 * BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  volatile int *abort_v = &abort_flag;

  if (warp == 0) {
    // weight producer: the weights are never written by a kernel, so the ring
    // fills before (and while) the previous launch finishes
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();  // weights stream through once
      uint32_t fill_parity[kTcMaxA];
      bool used[kTcMaxA];
      for (int s = 0; s < kTcMaxA; ++s) used[s] = false;
      KCursor ca;
      ca.start(p, passes, my_begin, my_end, BN, M);
      // L2 prefetch cursor, pf_ahead tiles past the ring (the first SA loads
      // are issued at once, so it starts at tile SA)
      KCursor cp;
      cp.start(p, passes, my_begin, my_end, BN, M);
      const int look = p.pf_ahead > 0 ? SA + p.pf_ahead : 0;
      int cp_idx = 0;
      if (look > 0)
        while (cp.valid && cp_idx < SA) {
          cp.advance(p, passes, BN, M);
          ++cp_idx;
        }
      int stage = 0, ld_idx = 0;
      uint32_t phase = 0;
      bool ok = true;
      while (ca.valid) {
        while (look > 0 && cp.valid && cp_idx <= ld_idx + look) {
          tma_prefetch_2d(&p.a[cp.f.seg], cp.kb * 64, cp.f.arow);
          cp.advance(p, passes, BN, M);
          ++cp_idx;
        }
        if (!wait_bounded(EMPTY_A(stage), phase ^ 1u, abort_v, p.status)) {
          ok = false;
          break;
        }
        mbar_expect_tx(FULL_A(stage), kTcABytes);
        tma_load_2d(STAGE_A(stage), &p.a[ca.f.seg], ca.kb * 64, ca.f.arow, FULL_A(stage), pol_w);
        used[stage] = true;
        fill_parity[stage] = phase;
        ca.advance(p, passes, BN, M);
        ++ld_idx;
        if (++stage == SA) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) {
        for (int s = 0; s < SA; ++s)
          if (used[s]) wait_drain(FULL_A(s), fill_parity[s]);
      } else if (p.nx_count > 0) {
        // the next GEMM's first weight tiles into L2 (fire and forget)
        const int nkb = p.nx_geo.kblocks;
        for (int c = blockIdx.x; c < p.nx_geo.grid; c += gridDim.x) {
          const long long b = sk_begin(p.nx_geo, c), e0 = sk_begin(p.nx_geo, c + 1);
          const long long e = e0 < b + p.nx_count ? e0 : b + p.nx_count;
          for (long long x = b; x < e; ++x) {
            const int t = (int)(x / nkb), kb = (int)(x - (long long)t * nkb);
            int seg = 0;
            while (seg + 1 < p.nx_nseg && t >= p.nx_seg_tile0[seg + 1]) ++seg;
            tma_prefetch_2d(&p.nx_a[seg], kb * 64, (t - p.nx_seg_tile0[seg]) * 128);
          }
        }
      }
    }
  } else if (warp == 6) {
    // activation producer: the packed rows are written by the previous launch
    if (lane == 0) {
      griddep_wait();
      allow_dependents();  // the next kernel may be scheduled (it waits for this grid)
      const uint64_t pol_x = policy_evict_last();  // activations are re-read by every tile
      uint32_t fill_parity[kTcMaxB];
      bool used[kTcMaxB];
      for (int s = 0; s < kTcMaxB; ++s) used[s] = false;
      KCursor cb;
      cb.start(p, passes, my_begin, my_end, BN, M);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      while (cb.valid) {
        if (!wait_bounded(EMPTY_B(stage), phase ^ 1u, abort_v, p.status)) {
          ok = false;
          break;
        }
        // the whole token pass in one box: TMA throughput is bound by the number
        // of copies, not their bytes (rows past the packed count are never read
        // by the MMA; rows past the buffer are zero-filled)
        mbar_expect_tx(FULL_B(stage), b_bytes);
        tma_load_2d(STAGE_B(stage), &p.b, cb.kb * 64, cb.m0, FULL_B(stage), pol_x);
        used[stage] = true;
        fill_parity[stage] = phase;
        cb.advance(p, passes, BN, M);
        if (++stage == SB) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok)
        for (int s = 0; s < SB; ++s)
          if (used[s]) wait_drain(FULL_B(s), fill_parity[s]);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int sa = 0, sb = 0;
      uint32_t pa = 0, pb = 0, nfrag = 0;
      const uint32_t idesc_lm = idesc_bf16(128, 128);
      bool ok = true, issued = false;
      FragIter it{my_begin, my_end, 0};
      Frag f;
      while (ok && next_frag(p, passes, it, f)) {
        const int mrows = min(BN, M - it.pass * BN);
        const uint32_t idesc = idesc_bf16(128, (mrows + 15) & ~15);
        const int lm_halves = mrows > 128 ? 2 : 1;
        const uint32_t acc = nfrag & 1u, use = nfrag >> 1;
        const uint32_t dtm = tmem + acc * (uint32_t)BN;
        if (!wait_bounded(TEMPTY(acc), (use & 1u) ^ 1u, abort_v, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = f.kb0; kb < f.kb1; ++kb) {
          if (!wait_bounded(FULL_A(sa), pa, abort_v, p.status) || !wait_bounded(FULL_B(sb), pb, abort_v, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = sw128_desc(STAGE_A(sa));
          const uint64_t bd = sw128_desc(STAGE_B(sb));
          if (p.epi_mode == 1) {
            // LM head: tokens are the MMA M dimension (one or two 128-row halves of
            // the activation box), the tile's 128 vocabulary rows are N
            for (int mt = 0; mt < lm_halves; ++mt) {
              const uint64_t xd = sw128_desc(STAGE_B(sb) + (uint32_t)mt * 16384u);
#pragma unroll
              for (int k = 0; k < 4; ++k)
                tc_mma(dtm + (uint32_t)(mt * 128), xd + (uint64_t)(2 * k), ad + (uint64_t)(2 * k), idesc_lm,
                       (kb > f.kb0 || k > 0) ? 1u : 0u);
            }
          } else {
#pragma unroll
            for (int k = 0; k < 4; ++k)  // 4 x K=16 (32 bytes) inside the 128-byte swizzle atom
              tc_mma(dtm, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k), idesc, (kb > f.kb0 || k > 0) ? 1u : 0u);
          }
          issued = true;
          tc_commit(EMPTY_A(sa));  // both stages are free once these MMAs have read them
          tc_commit(EMPTY_B(sb));
          if (++sa == SA) {
            sa = 0;
            pa ^= 1u;
          }
          if (++sb == SB) {
            sb = 0;
            pb ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(TFULL(acc));
        ++nfrag;
      }
      if (!ok && issued) {
        tc_commit(drain);
        wait_drain(drain, 0);
      }
    }
  } else if (warp >= 2 && warp <= 5) {
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    uint32_t nfrag = 0;
    FragIter it{my_begin, my_end, 0};
    Frag f;
    float lm_max[2] = {-INFINITY, -INFINITY};
    double lm_sum[2] = {0.0, 0.0};  // fp64 running sums: ~1000 terms per CTA
    int lm_arg[2] = {0x7fffffff, 0x7fffffff};
    int lm_pass = 0;
    // LM head: this CTA's statistics of the pass's tokens over its vocabulary range
    auto lm_flush = [&](int pass) {
      for (int mt = 0; mt < 2; ++mt) {
        const int m = pass * BN + mt * 128 + q * 32 + lane;
        if (m < M) {
          const size_t o = (size_t)blockIdx.x * p.ldm + (size_t)m;
          p.smx[o] = make_float2(lm_max[mt], (float)lm_sum[mt]);
          p.smx_arg[o] = lm_arg[mt];
        }
        lm_max[mt] = -INFINITY;
        lm_sum[mt] = 0.0;
        lm_arg[mt] = 0x7fffffff;
      }
    };
    while (next_frag(p, passes, it, f)) {
      const int m0 = it.pass * BN;
      const int mrows = min(BN, M - m0);
      const uint32_t acc = nfrag & 1u, use = nfrag >> 1;
      const uint32_t tacc = tmem + acc * (uint32_t)BN + ((uint32_t)(q * 32) << 16);
      if (!__all_sync(0xffffffffu, wait_bounded(TFULL(acc), use & 1u, abort_v, p.status))) break;
      tc_fence_after();
      const int rin = f.arow + q * 32 + lane;  // row within the weight segment
      const bool col_ok = rin < p.seg_rows[f.seg];
      const size_t col = (size_t)(p.seg_col0[f.seg] + rin);
      if (p.epi_mode == 1) {
        // LM head: this thread owns token m = mt * 128 + (TMEM lane) and folds the
        // tile's 128 logits into its running (max, sum of exp, lowest argmax);
        // tiles arrive in increasing vocabulary order, so on equal maxima the
        // earlier (lower) id is kept
        const int vbase = f.tile * 128;
        if (it.pass != lm_pass) {
          lm_flush(lm_pass);
          lm_pass = it.pass;
        }
        for (int mt = 0; mt < (mrows > 128 ? 2 : 1); ++mt) {
          const uint32_t tm = tmem + acc * (uint32_t)BN + (uint32_t)(mt * 128) + ((uint32_t)(q * 32) << 16);
          float &RM = lm_max[mt];
          double &RS = lm_sum[mt];
          int &RI = lm_arg[mt];
          for (int c = 0; c < 128; c += 16) {
            float v[16];
            tmem_ld16(tm + (uint32_t)c, v);
            float cm = -INFINITY;
            int cj = 0;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const bool ok = vbase + c + j < p.seg_rows[0];
              v[j] = ok ? v[j] : -INFINITY;
              if (v[j] > cm) { cm = v[j]; cj = j; }
            }
            // no divergent exit from this loop: tmem_ld16 is warp-collective
            if (cm > RM) {
              RS = (RM == -INFINITY) ? 0.0 : RS * (double)expf(RM - cm);
              RM = cm;
              RI = vbase + c + cj;
            }
            if (RM != -INFINITY) {
              float e = 0.f;
#pragma unroll
              for (int j = 0; j < 16; ++j) e += expf(v[j] - RM);
              RS += (double)e;
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(TEMPTY(acc));
        ++nfrag;
        continue;
      }
      float *dst = p.out + (size_t)f.slot * (size_t)p.geo.slot_stride + col;
      for (int c = 0; c < mrows; c += 16) {
        float v[16];
        tmem_ld16(tacc + (uint32_t)c, v);
        if (col_ok) {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (c + j < mrows) dst[(size_t)(m0 + c + j) * p.ldc] = v[j];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(TEMPTY(acc));  // the accumulator may be reused from here on
      ++nfrag;
    }
    if (p.epi_mode == 1) lm_flush(lm_pass);
  }
#undef FULL_A
#undef EMPTY_A
#undef FULL_B
#undef EMPTY_B
#undef TFULL
#undef TEMPTY
#undef STAGE_A
#undef STAGE_B
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * BN);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  // looked up once per process (a thread-safe static): the driver entry point
  // does not depend on the device
  static const EncodeTiledFn fn = [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(p);
    return (EncodeTiledFn) nullptr;
  }();
  return fn;
}

}  // namespace

bool encode_tmap_bf16(CUtensorMap *map, const void *ptr, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                      uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN>
static cudaError_t launch_bn(const TcParams &p, int grid, cudaStream_t s) {
  static std::atomic<uint64_t> smem_set{0};
  if (cudaError_t e = ensure_smem_limit(k_gemm_tc<BN>, (int)kTcSmem, smem_set)) return e;
  // programmatic dependent launch: the CTAs may start while the previous kernel
  // finishes; they wait (griddepcontrol.wait) before reading its outputs
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = kTcSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_gemm_tc<BN>, p);
}

cudaError_t launch_gemm_tc(TcParams p, int bn, cudaStream_t s) {
  const int grid = p.geo.grid;
  if (grid <= 0) return cudaSuccess;
  if (p.b_rows <= 0 || p.b_rows > bn || p.b_rows % 16 != 0) return cudaErrorInvalidValue;
  p.smem_bytes = (uint32_t)kTcSmem;
  if (bn == 128) return launch_bn<128>(p, grid, s);
  if (bn == 256) return launch_bn<256>(p, grid, s);
  return cudaErrorInvalidValue;
}

int tc_max_slots(int n_tiles, int grid) { return (grid + n_tiles - 1) / n_tiles + 1; }

namespace {
__global__ void __launch_bounds__(512) k_lm_combine(const float2 *__restrict__ smx, const int32_t *__restrict__ arg,
                                                    int n_tiles, int ldm, const int32_t *__restrict__ rowmap,
                                                    const int32_t *__restrict__ m_total, float *__restrict__ conf,
                                                    int32_t *__restrict__ amax) {
  pdl_enter();
  __shared__ float sm[32];
  __shared__ int si[32];
  __shared__ double sd[32];
  const int M = *m_total;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int r = blockIdx.x; r < M; r += gridDim.x) {
    float mx = -INFINITY;
    int ix = 0x7fffffff;
    for (int t = threadIdx.x; t < n_tiles; t += blockDim.x) {
      const float2 v = smx[(size_t)t * ldm + r];
      const int i = arg[(size_t)t * ldm + r];
      if (v.x > mx || (v.x == mx && i < ix)) { mx = v.x; ix = i; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float om = __shfl_xor_sync(0xffffffffu, mx, o);
      const int oi = __shfl_xor_sync(0xffffffffu, ix, o);
      if (om > mx || (om == mx && oi < ix)) { mx = om; ix = oi; }
    }
    __syncthreads();
    if (lane == 0) { sm[w] = mx; si[w] = ix; }
    __syncthreads();
    mx = -INFINITY;
    ix = 0x7fffffff;
    for (int i = 0; i < nw; ++i)
      if (sm[i] > mx || (sm[i] == mx && si[i] < ix)) { mx = sm[i]; ix = si[i]; }
    double sum = 0.0;
    for (int t = threadIdx.x; t < n_tiles; t += blockDim.x) {
      const float2 v = smx[(size_t)t * ldm + r];
      if (v.x != -INFINITY) sum += (double)v.y * exp((double)v.x - (double)mx);
    }
    sum = block_sum(sum, sd);
    if (threadIdx.x == 0) {
      const int row = rowmap[r];
      conf[row] = (float)(1.0 / sum);
      amax[row] = ix;
    }
  }
}
}  // namespace

cudaError_t launch_lm_combine(const float2 *smx, const int32_t *smx_arg, int n_tiles, int ldm,
                              const int32_t *rowmap, const int32_t *m_total, int cap, float *conf, int32_t *amax,
                              cudaStream_t s) {
  const int grid = cap < 148 * 8 ? cap : 148 * 8;
  launch_pdl(k_lm_combine, grid > 0 ? grid : 1, 512, 0, s, smx, smx_arg, n_tiles, ldm, rowmap, m_total, conf, amax);
  return cudaGetLastError();
}

}  // namespace dcu
