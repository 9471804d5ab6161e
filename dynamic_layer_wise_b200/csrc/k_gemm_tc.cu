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
//               never written by a kernel) and runs through every phase
//   warp 6      activation producer (one lane): shallow ring of X tiles (from
//               L2, one TMA box of the whole token pass per stage), after the
//               programmatic-dependency wait (phase 0) or the grid barrier that
//               publishes the previous phase's epilogue (chained phases)
//   warp 1      TMEM allocator + MMA issuer (one lane): 4 x tcgen05.mma (K=16)
//               per 64-wide k block, tcgen05.commit frees both smem stages
//   warps 2..5  epilogue: tcgen05.ld of the 128 x BN fp32 tile, coalesced
//               stores of the split-K partial (32 lanes = 32 consecutive n);
//               in a chained launch also the grid barriers and their share of
//               each phase's epilogue (128 threads, named barrier 1)
// A work unit is (weight tile, k split, token pass); the row count M is read
// from the device, so one launch serves any recompute-set size inside a graph.
// Every mbarrier wait and grid barrier is bounded: on expiry the CTA sets
// DCU_ST_TIMEOUT, drains its own copies / MMAs in flight, frees TMEM and exits.
#include <cuda.h>

#include "common.cuh"
#include "gemm_tc.h"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace dcu {
namespace {

struct Frag {
  int tile, kb0, kb1, seg, arow, slot;
  int col0, rows;  // first output column and row count of the fragment's weight segment
};

// The fields of a phase that the per-fragment bookkeeping reads, copied out of
// the kernel parameters with constant indices.  (Indexing the parameter
// struct with a run-time phase number, or its small arrays with a run-time
// segment number, turns every access into a generic load from parameter
// memory; at the start of a CTA those dependent loads cost microseconds.)
struct PhaseLite {
  SlotGeo geo;
  int nseg, ldc;
  int t1, t2, t3;   // seg_tile0[1..3]
  int c0, c1, c2;   // seg_col0[0..2]
  int r0, r1, r2;   // seg_rows[0..2]
};

__device__ __forceinline__ void copy_phase(const TcPhase &q, PhaseLite &l) {
  l.geo = q.geo;
  l.nseg = q.nseg;
  l.ldc = q.ldc;
  l.t1 = q.seg_tile0[1];
  l.t2 = q.seg_tile0[2];
  l.t3 = q.seg_tile0[3];
  l.c0 = q.seg_col0[0];
  l.c1 = q.seg_col0[1];
  l.c2 = q.seg_col0[2];
  l.r0 = q.seg_rows[0];
  l.r1 = q.seg_rows[1];
  l.r2 = q.seg_rows[2];
}

__device__ __forceinline__ PhaseLite phase_lite(const TcParams &p, int ph) {
  PhaseLite l;
  if (ph == 0)
    copy_phase(p.ph[0], l);
  else if (ph == 1)
    copy_phase(p.ph[1], l);
  else
    copy_phase(p.ph[2], l);
  return l;
}

// Fragment iterator over this CTA's stream-K range of one phase, group by
// group of token passes (a group is one pass unless the launch sweeps).
struct FragIter {
  long long pos, end;
  int pass, ph;
  PhaseLite l;
};

__device__ __forceinline__ FragIter frag_begin(const TcParams &p, int ph) {
  FragIter it;
  it.l = phase_lite(p, ph);
  const SlotGeo &g = it.l.geo;
  it.ph = ph;
  it.pass = 0;
  if ((int)blockIdx.x < g.grid) {
    it.pos = sk_begin(g, blockIdx.x);
    it.end = sk_begin(g, blockIdx.x + 1);
  } else {  // more CTAs than this phase has ranges
    it.pos = it.end = 0;
  }
  return it;
}

// kSlot: also find the fragment's output slot (a search over the stream-K
// ranges that only the epilogue needs; the loaders and the MMA skip it).
template <bool kSlot>
__device__ __forceinline__ bool next_frag(const TcParams &p, int ngroups, FragIter &it, Frag &f) {
  const PhaseLite &q = it.l;
  if ((int)blockIdx.x >= q.geo.grid) return false;  // no range in this phase
  while (it.pos >= it.end) {
    if (++it.pass >= ngroups) return false;
    it.pos = sk_begin(q.geo, blockIdx.x);
  }
  const int KB = q.geo.kblocks;
  const int t = sk_small(q.geo) ? (int)((unsigned)it.pos / (unsigned)KB) : (int)(it.pos / KB);
  const int kb0 = (int)(it.pos - (long long)t * KB);
  const long long left = it.end - it.pos;
  const int kb1 = (int)((long long)kb0 + left < KB ? kb0 + left : KB);
  it.pos += kb1 - kb0;
  f.tile = t;
  f.kb0 = kb0;
  f.kb1 = kb1;
  // segment of tile t (segment starts ascend): selects with constant indices
  int seg = 0, tile0 = 0, col0 = q.c0, rows = q.r0;
  if (q.nseg > 1 && t >= q.t1) { seg = 1; tile0 = q.t1; col0 = q.c1; rows = q.r1; }
  if (q.nseg > 2 && t >= q.t2) { seg = 2; tile0 = q.t2; col0 = q.c2; rows = q.r2; }
  f.seg = seg;
  f.arow = (t - tile0) * 128;
  f.col0 = col0;
  f.rows = rows;
  if (kSlot) f.slot = (int)blockIdx.x - sk_first(q.geo, t);
  return true;
}

// Position in this CTA's (phase, fragment, k block) sequence; m0 is the first
// row of the fragment's group of token passes (grows rows per group).
struct KCursor {
  FragIter it;
  Frag f;
  int kb, m0;
  bool valid;
  // it0: this CTA's iterator of phase ph, fresh from frag_begin
  __device__ __forceinline__ void start(const TcParams &p, const FragIter &it0, int ngroups, int grows) {
    it = it0;
    valid = next_frag<false>(p, ngroups, it, f);
    if (valid) {
      kb = f.kb0;
      m0 = it.pass * grows;
    }
  }
  __device__ __forceinline__ void advance(const TcParams &p, int ngroups, int grows) {
    if (++kb < f.kb1) return;
    valid = next_frag<false>(p, ngroups, it, f);
    if (valid) {
      kb = f.kb0;
      m0 = it.pass * grows;
    }
  }
};

// ------------------------------------------------------------------ chained launches

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ int ld_acquire(const int32_t *p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Spins (bounded by wall-clock time) until *ctr reaches target.
__device__ __forceinline__ bool spin_count(const int32_t *ctr, int target, volatile int *abort_flag,
                                           int32_t *status) {
  const uint64_t t0 = global_ns();
  for (uint32_t it = 0;; ++it) {
    if (ld_acquire(ctr) >= target) return true;
    if ((it & 15u) == 15u) {
      if (*abort_flag) return false;
      if (global_ns() - t0 > kWaitLimitNs) {
        *abort_flag = 1;
        if (status) atomicOr(status, DCU_ST_TIMEOUT);
        return false;
      }
    }
    __nanosleep(128);
  }
}

// Grid barrier of the epilogue warps (all 128 threads of every CTA call it):
// the CTA's earlier global stores are published, one arrival per CTA, then
// every CTA waits for all gridDim.x arrivals.  False if the wait gave up.
__device__ __forceinline__ bool grid_sync(int32_t *ctr, int ew, int lane, volatile int *abort_flag,
                                          int32_t *status, int *s_flag) {
  __threadfence();
  epi_bar();
  if (ew == 0 && lane == 0) {
    atomicAdd(ctr, 1);
    *s_flag = spin_count(ctr, (int)gridDim.x, abort_flag, status) ? 1 : 0;
  }
  epi_bar();
  const bool ok = *s_flag != 0;
  __threadfence();
  return ok;
}

// Sum of the 128 epilogue threads' values (fixed tree; every thread gets it).
__device__ __forceinline__ double sum128(double v, double *red, int ew, int lane) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  epi_bar();
  if (lane == 0) red[ew] = v;
  epi_bar();
  return (red[0] + red[1]) + (red[2] + red[3]);
}

// 4 consecutive outputs of packed row r: the pieces of their tile summed in
// slot order (read through L2: other CTAs of this launch wrote them).
__device__ __forceinline__ float4 slot_sum4(const TcParams &p, const TcPhase &q, int r, int col) {
  const float *c = p.out + (size_t)r * q.ldc + col;
  float4 v = __ldcg(reinterpret_cast<const float4 *>(c));
  const int ns = __ldg(q.geo.nslots + (col >> 7));
  for (int sp = 1; sp < ns; ++sp) {
    const float4 w = __ldcg(reinterpret_cast<const float4 *>(c + (size_t)sp * (size_t)q.geo.slot_stride));
    v.x += w.x;
    v.y += w.y;
    v.z += w.z;
    v.w += w.w;
  }
  return v;
}

__device__ __forceinline__ uint2 pack_bf16x4(float a, float b, float c, float d) {
  const __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
  uint2 u;
  u.x = *reinterpret_cast<const uint32_t *>(&lo);
  u.y = *reinterpret_cast<const uint32_t *>(&hi);
  return u;
}

// EPI_QKV, items of 4 consecutive RoPE pairs or 4 v values over all rows.
__device__ void epi_qkv(const TcParams &p, const TcPhase &q, int M, int t128) {
  const EpiArgs &e = p.e;
  const int H = e.H, Hkv = e.Hkv, hd = e.hd, half = hd / 2, N = e.N;
  const int n_rope = (H + Hkv) * half / 4, n_v = Hkv * hd / 4;
  const int per_row = n_rope + n_v;
  bf16 *Q = static_cast<bf16 *>(e.Q), *Kc = static_cast<bf16 *>(e.Kc), *Vc = static_cast<bf16 *>(e.Vc);
  for (long long it = (long long)blockIdx.x * 128 + t128; it < (long long)M * per_row; it += (long long)gridDim.x * 128) {
    const int r = (int)(it / per_row), u = (int)(it - (long long)r * per_row);
    const int row = e.rowmap[r];
    const int b = row / N, i = row - b * N;
    if (u < n_rope) {
      const int t = u * 4;
      const int head = t / half, j = t - head * half;
      const int base = head * hd;  // q heads first, then k heads (contiguous in the output)
      const float4 a = slot_sum4(p, q, r, base + j), bb = slot_sum4(p, q, r, base + j + half);
      float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {bb.x, bb.y, bb.z, bb.w};
      if (e.use_rope) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 cs = e.rope_tab[(size_t)i * half + j + k];
          const float a2 = av[k] * cs.x - bv[k] * cs.y;
          const float b2 = bv[k] * cs.x + av[k] * cs.y;
          av[k] = a2;
          bv[k] = b2;
        }
      }
      bf16 *dst = head < H ? Q + (size_t)r * H * hd + (size_t)head * hd
                           : Kc + (((size_t)b * Hkv + (head - H)) * N + i) * hd;
      *reinterpret_cast<uint2 *>(dst + j) = pack_bf16x4(av[0], av[1], av[2], av[3]);
      *reinterpret_cast<uint2 *>(dst + j + half) = pack_bf16x4(bv[0], bv[1], bv[2], bv[3]);
    } else {
      const int t = (u - n_rope) * 4;
      const int kvh = t / hd, j = t - kvh * hd;
      if (t == 0 && e.stale_l) e.stale_l[row] = 0;  // the layer recomputes this row
      const float4 v = slot_sum4(p, q, r, (H + Hkv) * hd + t);
      *reinterpret_cast<uint2 *>(Vc + (((size_t)b * Hkv + kvh) * N + i) * hd + j) = pack_bf16x4(v.x, v.y, v.z, v.w);
    }
  }
}

// EPI_O, one row per CTA: hmid = H_l[row] + o; xs = bf16(hmid / rms(hmid) * g2).
__device__ void epi_o(const TcParams &p, const TcPhase &q, int M, int t128, int ew, int lane, double *red) {
  const EpiArgs &e = p.e;
  const int D = e.D;
  const bf16 *Hl = static_cast<const bf16 *>(e.Hl);
  bf16 *xs = static_cast<bf16 *>(e.xs);
  for (int r = blockIdx.x; r < M; r += gridDim.x) {
    const bf16 *x = Hl + (size_t)e.rowmap[r] * D;
    float *hm = e.hmid + (size_t)r * D;
    double ss = 0;
    for (int j = t128 * 8; j < D; j += 128 * 8) {
      float v[8];
      load_vec(x + j, v);
      const float4 c0 = slot_sum4(p, q, r, j), c1 = slot_sum4(p, q, r, j + 4);
      v[0] += c0.x; v[1] += c0.y; v[2] += c0.z; v[3] += c0.w;
      v[4] += c1.x; v[5] += c1.y; v[6] += c1.z; v[7] += c1.w;
      *reinterpret_cast<float4 *>(hm + j) = make_float4(v[0], v[1], v[2], v[3]);
      *reinterpret_cast<float4 *>(hm + j + 4) = make_float4(v[4], v[5], v[6], v[7]);
#pragma unroll
      for (int k = 0; k < 8; ++k) ss += (double)v[k] * (double)v[k];
    }
    ss = sum128(ss, red, ew, lane);
    const float inv = (float)(1.0 / sqrt(ss / (double)D + (double)e.eps));
    bf16 *o = xs + (size_t)r * D;
    for (int j = t128 * 8; j < D; j += 128 * 8) {
      const float4 h0 = *reinterpret_cast<const float4 *>(hm + j), h1 = *reinterpret_cast<const float4 *>(hm + j + 4);
      const float *g = e.g2 + j;
      *reinterpret_cast<uint2 *>(o + j) =
          pack_bf16x4(h0.x * inv * g[0], h0.y * inv * g[1], h0.z * inv * g[2], h0.w * inv * g[3]);
      *reinterpret_cast<uint2 *>(o + j + 4) =
          pack_bf16x4(h1.x * inv * g[4], h1.y * inv * g[5], h1.z * inv * g[6], h1.w * inv * g[7]);
    }
  }
}

// EPI_GU, items of 4 consecutive columns over all rows: act = silu(gate) * up.
__device__ void epi_gu(const TcParams &p, const TcPhase &q, int M, int t128) {
  const EpiArgs &e = p.e;
  const int F = e.F, per_row = F / 4;
  bf16 *act = static_cast<bf16 *>(e.act);
  for (long long it = (long long)blockIdx.x * 128 + t128; it < (long long)M * per_row; it += (long long)gridDim.x * 128) {
    const int r = (int)(it / per_row), j = (int)(it - (long long)r * per_row) * 4;
    const float4 gt = slot_sum4(p, q, r, j), up = slot_sum4(p, q, r, F + j);
    *reinterpret_cast<uint2 *>(act + (size_t)r * F + j) =
        pack_bf16x4(gt.x / (1.0f + expf(-gt.x)) * up.x, gt.y / (1.0f + expf(-gt.y)) * up.y,
                    gt.z / (1.0f + expf(-gt.z)) * up.z, gt.w / (1.0f + expf(-gt.w)) * up.w);
  }
}

// EPI_DOWN, one row per CTA: new = bf16(hmid + down); with d_next, the next
// layer's distance against the cached row (before it is overwritten) and the
// stale flag; H_{l+1}[row] = new.
__device__ void epi_down(const TcParams &p, const TcPhase &q, int M, int t128, int ew, int lane, double *red,
                         int *s_flag) {
  const EpiArgs &e = p.e;
  const int D = e.D;
  bf16 *Hn = static_cast<bf16 *>(e.Hn);
  const bool want_d = e.d_next != nullptr;
  for (int r = blockIdx.x; r < M; r += gridDim.x) {
    const int row = e.rowmap[r];
    const float *hm = e.hmid + (size_t)r * D;
    bf16 *dst = Hn + (size_t)row * D;
    double dot = 0, nx = 0, ny = 0;
    bool same = true;
    for (int j = t128 * 8; j < D; j += 128 * 8) {
      const float4 c0 = slot_sum4(p, q, r, j), c1 = slot_sum4(p, q, r, j + 4);
      const float4 h0 = __ldcg(reinterpret_cast<const float4 *>(hm + j)),
                   h1 = __ldcg(reinterpret_cast<const float4 *>(hm + j + 4));
      float v[8] = {h0.x + c0.x, h0.y + c0.y, h0.z + c0.z, h0.w + c0.w,
                    h1.x + c1.x, h1.y + c1.y, h1.z + c1.z, h1.w + c1.w};
      if (want_d) {
        float ov[8];
        uint32_t ob[8];
        load_vec(dst + j, ov, ob);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const bf16 nt = __float2bfloat16_rn(v[k]);
          const float nv = __bfloat162float(nt);
          same = same && ((uint32_t)__bfloat16_as_ushort(nt) == ob[k]);
          const double gg = (double)e.g_next[j + k];
          const double a = gg * (double)nv, b = gg * (double)ov[k];
          dot += a * b;
          nx += a * a;
          ny += b * b;
        }
      }
      store_vec(dst + j, v);
    }
    if (want_d) {
      epi_bar();
      if (ew == 0 && lane == 0) *s_flag = 1;
      epi_bar();
      if (!same) *s_flag = 0;
      dot = sum128(dot, red, ew, lane);
      nx = sum128(nx, red, ew, lane);
      ny = sum128(ny, red, ew, lane);
      const bool all_same = *s_flag != 0;
      if (ew == 0 && lane == 0) {
        e.d_next[row] = finish_cosine_distance(dot, nx, ny, all_same);
        if (e.stale_next && !all_same) e.stale_next[row] = 1;  // H_{l+1} row changed
      }
      epi_bar();
    }
  }
}

// MODE (compile time, so each instantiation carries only its own code paths
// and stays small in the instruction cache): kPlain -- stream-K pieces into
// slots; kSweep -- the same with the pass sweep (sweep > 1); kLmHead --
// epi_mode EPI_LMHEAD; kChained -- chained phases (chain != 0).
enum { kPlain = 0, kLmHead = 1, kChained = 2, kSweep = 3 };

template <int BN, int MODE>
__global__ void __launch_bounds__(kTcThreads, 1) k_gemm_tc(const __grid_constant__ TcParams p) {
  constexpr bool kChain = MODE == kChained, kLm = MODE == kLmHead, kSw = MODE == kSweep;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[2 * kTcMaxA + 2 * kTcMaxB + 5];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ int s_epi_ok[4], s_flag, s_same;
  __shared__ double s_red[4];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // this CTA's stream-K range of the first phase (every role starts from it)
  const FragIter it_first = frag_begin(p, 0);
  if (!kChain && it_first.pos >= it_first.end) return;  // a CTA without work may leave (no barrier waits for it)
  // the first loads' tensor maps into the descriptor cache while the CTA sets up
  if (threadIdx.x == 0) {
    for (int s = 0; s < p.ph[0].nseg; ++s) prefetch_tmap(&p.ph[0].a[s]);
    prefetch_tmap(&p.ph[0].b);
  }
  // The row count is written by the select / plan kernel two launches before
  // this one, so it is final even while the previous launch still runs; its
  // load overlaps the set-up below and is checked after it.
  const int M = p.m_total ? *p.m_total : p.m_host;
  // Two rings: weight tiles (16 KB, from HBM) and activation tiles (one TMA
  // box of the token pass per stage, from L2).  The activation ring only has
  // to cover the L2 latency, so most of shared memory holds weight tiles in
  // flight.
  // Shared memory: the weight ring, then the activation region.  With a pass
  // sweep an activation stage holds G boxes, one per token pass of the group;
  // the region is sized for the launch's largest G, so the weight ring's depth
  // does not depend on M (the weight producer starts before M is loaded) and
  // only the activation ring's depth follows G.  (The LM head, which runs
  // once per step, sizes it from M itself: a set within one pass keeps the
  // deeper weight ring.)
  const uint32_t b_bytes = (uint32_t)p.b_rows * 128u;            // one TMA box per token pass
  const uint32_t b_stage = (b_bytes + 1023u) & ~1023u;             // 1024-byte aligned boxes
  const int gmax = kSw ? p.sweep : (kLm && p.sweep > 1 && M > BN ? p.sweep : 1);
  const uint32_t x_region = gmax > 1 ? 2u * (uint32_t)gmax * b_stage : (b_stage > 16384u ? 3u : 4u) * b_stage;
  int SA = (int)((p.smem_bytes - 1024u - x_region) / kTcABytes);
  SA = SA > kTcMaxA ? kTcMaxA : SA;
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t bbase = sbase + (uint32_t)SA * kTcABytes;
  const uint32_t bar0 = smem_u32(bars);
  // TMEM: one accumulator of G x BN columns per fragment, two alternating
  // between fragments while they fit (always for G = 1)
  const uint32_t tcols = (kSw || kLm) ? 512u : 2u * (uint32_t)BN;
#define FULL_A(s) (bar0 + 8u * (uint32_t)(s))
#define EMPTY_A(s) (bar0 + 8u * (uint32_t)(kTcMaxA + (s)))
#define FULL_B(s) (bar0 + 8u * (uint32_t)(2 * kTcMaxA + (s)))
#define EMPTY_B(s) (bar0 + 8u * (uint32_t)(2 * kTcMaxA + kTcMaxB + (s)))
  const uint32_t tfull0 = bar0 + 8u * (uint32_t)(2 * kTcMaxA + 2 * kTcMaxB), tempty0 = tfull0 + 16u,
                 drain = tfull0 + 32u;
#define TFULL(a) (tfull0 + 8u * (uint32_t)(a))
#define TEMPTY(a) (tempty0 + 8u * (uint32_t)(a))
#define STAGE_A(s) (sbase + (uint32_t)(s) * kTcABytes)
#define STAGE_B(s) (bbase + (uint32_t)(s) * x_stage)

  if (threadIdx.x == 0) {
    for (int s = 0; s < SA; ++s) {
      mbar_init(FULL_A(s), 1);
      mbar_init(EMPTY_A(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(TFULL(a), 1);
      mbar_init(TEMPTY(a), 4);
    }
    for (int s = 0; s < kTcMaxB; ++s) {  // every stage: the depth follows G, known once M is
      mbar_init(FULL_B(s), 1);
      mbar_init(EMPTY_B(s), 1);
    }
    mbar_init(drain, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_slot), tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  volatile int *abort_v = &abort_flag;
  if (M <= 0) {  // nothing to multiply (uniform: every CTA of the launch leaves here, or none)
    if (warp == 1) tmem_dealloc(tmem, tcols);
    return;
  }
  const int passes = (M + BN - 1) / BN;
  // G token passes per weight tile (a group); the fragment iterators walk groups
  const int G = (kSw || kLm) ? min(passes, gmax) : 1;
  const int ngroups = (passes + G - 1) / G, grows = G * BN;
  const bool dbuf = 2u * (uint32_t)grows <= tcols;  // two accumulators alternate
  const uint32_t x_stage = (uint32_t)G * b_stage;
  const int SB = min(kTcMaxB, (int)(x_region / x_stage));

  if (warp == 0) {
    // weight producer: the weights are never written by a kernel, so the ring
    // fills before (and while) the previous launch or phase finishes
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();  // weights stream through once
      uint32_t used = 0, fill_parity = 0;  // per stage bit: loaded at least once / parity of its last fill
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int ph = 0; ph < p.nphase && ok; ++ph) {
        KCursor ca;
        ca.start(p, ph == 0 ? it_first : frag_begin(p, ph), ngroups, grows);
        while (ca.valid) {
          if (!wait_bounded(EMPTY_A(stage), phase ^ 1u, abort_v, p.status)) {
            ok = false;
            break;
          }
          mbar_expect_tx(FULL_A(stage), kTcABytes);
          tma_load_2d(STAGE_A(stage), &p.ph[ph].a[ca.f.seg], ca.kb * 64, ca.f.arow, FULL_A(stage), pol_w);
          used |= 1u << stage;
          fill_parity = (fill_parity & ~(1u << stage)) | (phase << stage);
          ca.advance(p, ngroups, grows);
          if (++stage == SA) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        for (int s = 0; s < SA; ++s)
          if ((used >> s) & 1u) wait_drain(FULL_A(s), (fill_parity >> s) & 1u);
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
    // (phase 0) or by the previous phase's epilogue (chained phases)
    if (lane == 0) {
      const uint64_t pol_x = policy_evict_last();  // activations are re-read by every tile
      KCursor cb0;  // the first phase's cursor, ready before the wait
      cb0.start(p, it_first, ngroups, grows);
      griddep_wait();
      allow_dependents();  // the next kernel may be scheduled (it waits for this grid)
      uint32_t used = 0, fill_parity = 0;  // per stage bit: loaded at least once / parity of its last fill
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int ph = 0; ph < p.nphase && ok; ++ph) {
        if (kChain && ph > 0) {
          // the barrier after phase ph - 1's epilogue: its outputs are this phase's operand
          if (!spin_count(p.bar + 2 * (ph - 1) + 1, (int)gridDim.x, abort_v, p.status)) {
            ok = false;
            break;
          }
          fence_proxy_async_global();  // generic-proxy stores of other CTAs, read next by TMA
        }
        KCursor cb = cb0;
        if (ph > 0) cb.start(p, frag_begin(p, ph), ngroups, grows);
        while (cb.valid) {
          if (!wait_bounded(EMPTY_B(stage), phase ^ 1u, abort_v, p.status)) {
            ok = false;
            break;
          }
          // the whole token pass in one box: TMA throughput is bound by the number
          // of copies, not their bytes (rows past the packed count are never read
          // by the MMA; rows past the buffer are zero-filled)
          if ((!kSw && !kLm) || G == 1) {
            mbar_expect_tx(FULL_B(stage), b_bytes);
            tma_load_2d(STAGE_B(stage), &p.ph[ph].b, cb.kb * 64, cb.m0, FULL_B(stage), pol_x);
          } else {  // one box per token pass of the group
            const int npg = min(G, passes - cb.it.pass * G);
            mbar_expect_tx(FULL_B(stage), (uint32_t)npg * b_bytes);
            for (int q = 0; q < npg; ++q)
              tma_load_2d(STAGE_B(stage) + (uint32_t)q * b_stage, &p.ph[ph].b, cb.kb * 64, cb.m0 + q * BN,
                          FULL_B(stage), pol_x);
          }
          used |= 1u << stage;
          fill_parity = (fill_parity & ~(1u << stage)) | (phase << stage);
          cb.advance(p, ngroups, grows);
          if (++stage == SB) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok)
        for (int s = 0; s < SB; ++s)
          if ((used >> s) & 1u) wait_drain(FULL_B(s), (fill_parity >> s) & 1u);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int sa = 0, sb = 0;
      uint32_t pa = 0, pb = 0, nfrag = 0;
      const uint32_t idesc_lm = idesc_bf16(128, 128);
      bool ok = true, issued = false;
      for (int ph = 0; ph < p.nphase && ok; ++ph) {
        FragIter it = ph == 0 ? it_first : frag_begin(p, ph);
        Frag f;
        while (ok && next_frag<false>(p, ngroups, it, f)) {
          const int mrows = min(BN, M - it.pass * grows);  // rows of the group's first pass
          const uint32_t idesc = idesc_bf16(128, (mrows + 15) & ~15);
          const int npg = min(G, passes - it.pass * G);
          const uint32_t acc = dbuf ? (nfrag & 1u) : 0u, use = dbuf ? nfrag >> 1 : nfrag;
          const uint32_t dtm = tmem + acc * (uint32_t)grows;
          if (!wait_bounded(TEMPTY(acc), (use & 1u) ^ 1u, abort_v, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int kb = f.kb0; kb < f.kb1; ++kb) {
            if (!wait_bounded(FULL_A(sa), pa, abort_v, p.status) ||
                !wait_bounded(FULL_B(sb), pb, abort_v, p.status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t ad = sw128_desc(STAGE_A(sa));
            const uint64_t bd = sw128_desc(STAGE_B(sb));
            if (kLm) {
              // LM head: tokens are the MMA M dimension (one or two 128-row halves of
              // each pass's activation box), the tile's 128 vocabulary rows are N;
              // pass q of the group accumulates at columns q * BN
              for (int q = 0; q < npg; ++q) {
                const int mq = min(BN, M - it.pass * grows - q * BN);
                for (int mt = 0; mt < (mq > 128 ? 2 : 1); ++mt) {
                  const uint64_t xd = sw128_desc(STAGE_B(sb) + (uint32_t)q * b_stage + (uint32_t)mt * 16384u);
#pragma unroll
                  for (int k = 0; k < 4; ++k)
                    tc_mma(dtm + (uint32_t)(q * BN + mt * 128), xd + (uint64_t)(2 * k), ad + (uint64_t)(2 * k),
                           idesc_lm, (kb > f.kb0 || k > 0) ? 1u : 0u);
                }
              }
            } else {
#pragma unroll
              for (int k = 0; k < 4; ++k)  // 4 x K=16 (32 bytes) inside the 128-byte swizzle atom
                tc_mma(dtm, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k), idesc, (kb > f.kb0 || k > 0) ? 1u : 0u);
              // the group's further passes: their boxes follow in the stage, their
              // accumulators in TMEM
              for (int q = 1; kSw && q < npg; ++q) {
                const int mq = min(BN, M - it.pass * grows - q * BN);
                const uint32_t idq = idesc_bf16(128, (mq + 15) & ~15);
                const uint64_t bq = sw128_desc(STAGE_B(sb) + (uint32_t)q * b_stage);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                  tc_mma(dtm + (uint32_t)(q * BN), ad + (uint64_t)(2 * k), bq + (uint64_t)(2 * k), idq,
                         (kb > f.kb0 || k > 0) ? 1u : 0u);
              }
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
      }
      if (!ok && issued) {
        tc_commit(drain);
        wait_drain(drain, 0);
      }
    }
  } else if (warp >= 2 && warp <= 5) {
    const int q4 = warp & 3;  // TMEM lane quarter this warp may access
    const int ew = warp - 2, t128 = threadIdx.x - 64;
    uint32_t nfrag = 0;
    // LM head: per (pass of the group, 128-token half) running statistics
    constexpr int kLmSlots = kLm ? 4 : 1;  // a group holds at most 2 passes of the 256-row box
    float lm_max[kLmSlots];
    double lm_sum[kLmSlots];  // fp64 running sums: ~1000 terms per CTA
    int lm_arg[kLmSlots];
#pragma unroll
    for (int i = 0; i < kLmSlots; ++i) {
      lm_max[i] = -INFINITY;
      lm_sum[i] = 0.0;
      lm_arg[i] = 0x7fffffff;
    }
    int lm_group = 0;
    // LM head: this CTA's statistics of the group's tokens over its vocabulary range
    auto lm_flush = [&](int group) {
#pragma unroll
      for (int i = 0; i < kLmSlots; ++i) {
        const int m = (group * G + (i >> 1)) * BN + (i & 1) * 128 + q4 * 32 + lane;
        if ((i >> 1) < G && m < M) {
          const size_t o = (size_t)blockIdx.x * p.ldm + (size_t)m;
          p.smx[o] = make_float2(lm_max[i], (float)lm_sum[i]);
          p.smx_arg[o] = lm_arg[i];
        }
        lm_max[i] = -INFINITY;
        lm_sum[i] = 0.0;
        lm_arg[i] = 0x7fffffff;
      }
    };
    bool alive = true;
    for (int ph = 0; ph < p.nphase && alive; ++ph) {
      const TcPhase &q = p.ph[ph];
      FragIter it = ph == 0 ? it_first : frag_begin(p, ph);
      Frag f;
      while (next_frag<true>(p, ngroups, it, f)) {
        const int mg = it.pass * grows;  // first row of the group
        const uint32_t acc = dbuf ? (nfrag & 1u) : 0u, use = dbuf ? nfrag >> 1 : nfrag;
        const uint32_t tacc = tmem + acc * (uint32_t)grows + ((uint32_t)(q4 * 32) << 16);
        bool okw = __all_sync(0xffffffffu, wait_bounded(TFULL(acc), use & 1u, abort_v, p.status));
        if (kChain) {
          // the 4 warps meet at named barriers below: they leave together or not at all
          if (lane == 0) s_epi_ok[ew] = okw ? 1 : 0;
          epi_bar();
          okw = (s_epi_ok[0] & s_epi_ok[1] & s_epi_ok[2] & s_epi_ok[3]) != 0;
          epi_bar();
        }
        if (!okw) {
          alive = false;
          break;
        }
        tc_fence_after();
        const int rin = f.arow + q4 * 32 + lane;  // row within the weight segment
        const bool col_ok = rin < f.rows;
        const size_t col = (size_t)(f.col0 + rin);
        if (kLm) {
          // LM head: this thread owns token m = mt * 128 + (TMEM lane) and folds the
          // tile's 128 logits into its running (max, sum of exp, lowest argmax);
          // tiles arrive in increasing vocabulary order, so on equal maxima the
          // earlier (lower) id is kept
          const int vbase = f.tile * 128;
          if (it.pass != lm_group) {
            lm_flush(lm_group);
            lm_group = it.pass;
          }
#pragma unroll
          for (int i = 0; i < kLmSlots; ++i) {  // (pass q = i / 2 of the group, half mt = i % 2)
            const int q = i >> 1, mt = i & 1;
            const int mq = min(BN, M - mg - q * BN);  // rows of pass q (<= 0 past the group's passes)
            if (q >= G || mt * 128 >= mq) continue;   // warp-uniform
            const uint32_t tm =
                tmem + acc * (uint32_t)grows + (uint32_t)(q * BN + mt * 128) + ((uint32_t)(q4 * 32) << 16);
            float &RM = lm_max[i];
            double &RS = lm_sum[i];
            int &RI = lm_arg[i];
            const int tok = mg + q * BN + mt * 128 + q4 * 32 + lane;
            float *zdst = (p.zout && tok < M) ? p.zout + (int64_t)p.zrow[tok] * p.ldz + vbase : nullptr;
            for (int c = 0; c < 128; c += 16) {
              float v[16];
              tmem_ld16(tm + (uint32_t)c, v);
              if (zdst) {
#pragma unroll
                for (int j = 0; j < 16; ++j)
                  if (vbase + c + j < f.rows) zdst[c + j] = v[j];
              }
              float cm = -INFINITY;
              int cj = 0;
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const bool ok = vbase + c + j < f.rows;
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
        float *dst = p.out + (size_t)f.slot * (size_t)it.l.geo.slot_stride + col;
        const size_t ldc = (size_t)it.l.ldc;
        const int mend = min(M, mg + grows);  // the group's rows: [mg, mend), pass q at columns q * BN
        for (int c = 0; c < mend - mg; c += 16) {
          float v[16];
          tmem_ld16(tacc + (uint32_t)c, v);
          if (col_ok) {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (mg + c + j < mend) dst[(size_t)(mg + c + j) * ldc] = v[j];
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(TEMPTY(acc));  // the accumulator may be reused from here on
        ++nfrag;
      }
      if (!alive || !kChain) continue;
      // chained launch: every piece of this phase is stored once all CTAs are here
      if (!grid_sync(p.bar + 2 * ph, ew, lane, abort_v, p.status, &s_flag)) {
        alive = false;
        break;
      }
      if (q.epi == EPI_QKV)
        epi_qkv(p, q, M, t128);
      else if (q.epi == EPI_O)
        epi_o(p, q, M, t128, ew, lane, s_red);
      else if (q.epi == EPI_GU)
        epi_gu(p, q, M, t128);
      else if (q.epi == EPI_DOWN)
        epi_down(p, q, M, t128, ew, lane, s_red, &s_same);
      // the epilogue's outputs are the next phase's operand
      if (ph + 1 < p.nphase && !grid_sync(p.bar + 2 * ph + 1, ew, lane, abort_v, p.status, &s_flag)) {
        alive = false;
        break;
      }
    }
    if (kLm) lm_flush(lm_group);
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
    tmem_dealloc(tmem, tcols);
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

template <int BN, int MODE>
static cudaError_t launch_bn(const TcParams &p, int grid, cudaStream_t s) {
  static std::atomic<uint64_t> smem_set{0};
  if (cudaError_t e = ensure_smem_limit(k_gemm_tc<BN, MODE>, (int)kTcSmem, smem_set)) return e;
  prefer_max_smem(reinterpret_cast<const void *>(k_gemm_tc<BN, MODE>));
  // programmatic dependent launch: the CTAs may start while the previous kernel
  // finishes; they wait (griddepcontrol.wait) before reading its outputs
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = p.smem_bytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  // chained phases meet at grid barriers: every CTA must be resident at once
  attr[1].id = cudaLaunchAttributeCooperative;
  attr[1].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.chain == 1 ? 2 : 1;  // chain 2: programmatic launch only (all CTAs fit one per SM)
  return cudaLaunchKernelEx(&cfg, k_gemm_tc<BN, MODE>, p);
}

template <int BN>
static cudaError_t launch_mode(const TcParams &p, int grid, cudaStream_t s) {
  if (p.chain) return launch_bn<BN, kChained>(p, grid, s);
  if (p.epi_mode == EPI_LMHEAD) return launch_bn<BN, kLmHead>(p, grid, s);
  if (p.sweep > 1) return launch_bn<BN, kSweep>(p, grid, s);
  return launch_bn<BN, kPlain>(p, grid, s);
}

cudaError_t launch_gemm_tc(TcParams p, int bn, cudaStream_t s) {
  int grid = p.ph[0].geo.grid;
  if (p.nphase < 1 || p.nphase > kTcMaxPhases) return cudaErrorInvalidValue;
  for (int i = 1; i < p.nphase; ++i) grid = p.ph[i].geo.grid > grid ? p.ph[i].geo.grid : grid;
  if (grid <= 0) return cudaSuccess;
  if (p.chain && !p.bar) return cudaErrorInvalidValue;
  if (p.chain && p.epi_mode == EPI_LMHEAD) return cudaErrorInvalidValue;
  if (p.b_rows <= 0 || p.b_rows > bn || p.b_rows % 16 != 0) return cudaErrorInvalidValue;
  // dynamic shared memory: the default fills the SM; a smaller ring (at least
  // the activation stages and 4 weight tiles) leaves room for the CTAs of the
  // neighbouring small kernels, so this launch's CTAs become resident (and
  // start their weight stream) while those still run
  {
    const uint32_t b_stage = ((uint32_t)p.b_rows * 128u + 1023u) & ~1023u;
    const uint32_t need = 1024u + (b_stage > 16384u ? 3u : 4u) * b_stage + 4u * kTcABytes;
    if (p.smem_bytes == 0 || p.smem_bytes > (uint32_t)kTcSmem) p.smem_bytes = (uint32_t)kTcSmem;
    if (p.smem_bytes < need) p.smem_bytes = need;
    // pass sweep: G passes' accumulators in 512 TMEM columns, and two stages of
    // G activation boxes beside at least 4 weight tiles in shared memory
    int g = p.chain ? 0 : p.sweep;
    if (g > 512 / bn) g = 512 / bn;
    while (g > 1 && 1024u + 2u * (uint32_t)g * b_stage + 4u * kTcABytes > p.smem_bytes) --g;
    p.sweep = g > 1 ? g : 0;
  }
  if (bn == 128) return launch_mode<128>(p, grid, s);
  if (bn == 256) return launch_mode<256>(p, grid, s);
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
