// tcgen05 (5th-generation tensor core) GEMM for the bf16 recompute projections,
// FFN and LM head:  ws[split][m][n] = sum_{k in split} X[m][k] * W[n][k].
//
// Swap-AB: the weight rows are the MMA M dimension (128-row tiles, K-major,
// TMA-loaded with the 128-byte swizzle) and the selected tokens are the MMA N
// dimension (a BN-row K-major tile of the packed activations), so a recompute
// set of ~65 rows still drives full 128-row tensor-core instructions while
// every weight byte is read from HBM once.  Accumulators live in TMEM.
//
// Warp roles (192 threads, one CTA per SM, persistent over work units):
//   warp 0      TMA producer (one lane): STAGES-deep ring of (W tile, X tile)
//   warp 1      TMEM allocator + MMA issuer (one lane): 4 x tcgen05.mma (K=16)
//               per 64-wide k block, tcgen05.commit frees the smem stage
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

namespace dcu {
namespace {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y, uint32_t bar,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 TMEM lanes x 16 consecutive 32-bit columns: thread i of the warp gets lane
// (base lane + i), columns col..col+15.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  // the registers are only valid after wait::ld; tie them to it
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15])
               :
               : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor of a K-major tile with the 128-byte swizzle:
// start address >> 4 in bits [0,14), leading byte offset 0 (unused for this
// layout), stride byte offset 1024 (8 rows x 128 B) >> 4 in bits [32,46), the
// fixed descriptor version 1 at bit 46, swizzle mode 2 (128 B) in bits [61,64).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) |
         ((uint64_t)2 << 61);
}

// Instruction descriptor, kind::f16: fp32 accumulator (bits 4-5 = 1), A and B
// bf16 (bits 7-9 = 1, 10-12 = 1), both K-major, N >> 3 in bits 17-22,
// M >> 4 in bits 24-28.
__device__ __forceinline__ uint32_t idesc_bf16(int m, int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

constexpr uint32_t kSpinLimit = 1u << 25;

__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                             int32_t *status) {
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 255u && *abort_flag) return false;
    if (it >= kSpinLimit) {
      *abort_flag = 1;
      if (status) atomicOr(status, DCU_ST_TIMEOUT);
      return false;
    }
  }
}

// Drain wait on the abort path: bounded, ignores the abort flag.
__device__ __forceinline__ void wait_drain(uint32_t bar, uint32_t parity) {
  for (uint32_t it = 0; it < (1u << 22); ++it)
    if (mbar_try_wait(bar, parity)) return;
}

struct Unit {
  int tile, split, pass, seg, arow, kb0, kb1, m0;
};

__device__ __forceinline__ Unit decode_unit(const TcParams &p, int u, int passes) {
  Unit w;
  w.pass = u % passes;
  const int ts = u / passes;
  w.split = ts % p.splits;
  w.tile = ts / p.splits;
  w.kb0 = (int)((long long)w.split * p.kblocks / p.splits);
  w.kb1 = (int)((long long)(w.split + 1) * p.kblocks / p.splits);
  int seg = 0;
  while (seg + 1 < p.nseg && w.tile >= p.seg_tile0[seg + 1]) ++seg;
  w.seg = seg;
  w.arow = (w.tile - p.seg_tile0[seg]) * 128;
  return w;
}

template <int BN>
__global__ void __launch_bounds__(192, 1) k_gemm_tc(const __grid_constant__ TcParams p) {
  using C = TcCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[2 * C::STAGES + 3];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const int M = p.m_total ? *p.m_total : p.m_host;
  if (M <= 0) return;
  const int passes = (M + BN - 1) / BN;
  const int n_units = p.n_tiles * p.splits * passes;
  if ((int)blockIdx.x >= n_units) return;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sA = sbase, sB = sbase + C::STAGES * C::A_BYTES;
  const uint32_t bar0 = smem_u32(bars);
  const uint32_t tfull = bar0 + 8u * (2 * C::STAGES), tempty = tfull + 8u, drain = tfull + 16u;
#define FULL(s) (bar0 + 8u * (uint32_t)(s))
#define EMPTY(s) (bar0 + 8u * (uint32_t)(C::STAGES + (s)))

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(FULL(s), 1);
      mbar_init(EMPTY(s), 1);
    }
    mbar_init(tfull, 1);
    mbar_init(tempty, 4);
    mbar_init(drain, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_slot), BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  volatile int *abort_v = &abort_flag;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();  // weights stream through once
      const uint64_t pol_x = policy_evict_last();   // activations are re-read by every tile
      uint32_t fill_parity[C::STAGES];
      bool used[C::STAGES];
      for (int s = 0; s < C::STAGES; ++s) used[s] = false;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const Unit w = decode_unit(p, u, passes);
        const int m0 = w.pass * BN;
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!wait_bounded(EMPTY(stage), phase ^ 1u, abort_v, p.status)) {
            ok = false;
            break;
          }
          mbar_expect_tx(FULL(stage), C::A_BYTES + C::B_BYTES);
          tma_load_2d(sA + stage * C::A_BYTES, &p.a[w.seg], kb * 64, w.arow, FULL(stage), pol_w);
          tma_load_2d(sB + stage * C::B_BYTES, &p.b, kb * 64, m0, FULL(stage), pol_x);
          used[stage] = true;
          fill_parity[stage] = phase;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok)
        for (int s = 0; s < C::STAGES; ++s)
          if (used[s]) wait_drain(FULL(s), fill_parity[s]);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, tphase = 0;
      bool ok = true, issued = false;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const Unit w = decode_unit(p, u, passes);
        const int mrows = min(BN, M - w.pass * BN);
        const uint32_t idesc = idesc_bf16(128, (mrows + 15) & ~15);
        if (!wait_bounded(tempty, tphase ^ 1u, abort_v, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!wait_bounded(FULL(stage), phase, abort_v, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = sw128_desc(sA + stage * C::A_BYTES);
          const uint64_t bd = sw128_desc(sB + stage * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < 4; ++k)  // 4 x K=16 (32 bytes) inside the 128-byte swizzle atom
            tc_mma(tmem, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k), idesc, (kb > w.kb0 || k > 0) ? 1u : 0u);
          issued = true;
          tc_commit(EMPTY(stage));
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(tfull);
        tphase ^= 1u;
      }
      if (!ok && issued) {
        tc_commit(drain);
        wait_drain(drain, 0);
      }
    }
  } else {
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    uint32_t tphase = 0;
    for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
      const Unit w = decode_unit(p, u, passes);
      const int m0 = w.pass * BN;
      const int mrows = min(BN, M - m0);
      if (!wait_bounded(tfull, tphase, abort_v, p.status)) break;
      tc_fence_after();
      const int rin = w.arow + q * 32 + lane;  // row within the weight segment
      const bool col_ok = rin < p.seg_rows[w.seg];
      float *dst = p.ws + (size_t)w.split * (size_t)p.split_stride + (size_t)(p.seg_col0[w.seg] + rin);
      for (int c = 0; c < mrows; c += 16) {
        float v[16];
        tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)c, v);
        if (col_ok) {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (c + j < mrows) dst[(size_t)(m0 + c + j) * p.ldc] = v[j];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty);
      tphase ^= 1u;
    }
  }
#undef FULL
#undef EMPTY
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, BN);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
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

int choose_splits(int n_tiles, int kblocks, int passes, int num_sms) {
  // minimise (waves x k blocks per unit + per-unit epilogue cost), ties to fewer splits
  double best = 1e30;
  int best_s = 1;
  for (int s = 1; s <= 16 && s <= kblocks; ++s) {
    const long long units = (long long)n_tiles * s * passes;
    const long long waves = (units + num_sms - 1) / num_sms;
    const double cost = (double)waves * ((double)((kblocks + s - 1) / s) + 2.0);
    if (cost < best - 1e-9) {
      best = cost;
      best_s = s;
    }
  }
  return best_s;
}

template <int BN>
static cudaError_t launch_bn(const TcParams &p, int grid, cudaStream_t s) {
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(k_gemm_tc<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)TcCfg<BN>::SMEM);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  k_gemm_tc<BN><<<grid, 192, TcCfg<BN>::SMEM, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_gemm_tc(const TcParams &p, int bn, int grid, cudaStream_t s) {
  if (bn == 64) return launch_bn<64>(p, grid, s);
  if (bn == 128) return launch_bn<128>(p, grid, s);
  if (bn == 256) return launch_bn<256>(p, grid, s);
  return cudaErrorInvalidValue;
}

}  // namespace dcu
