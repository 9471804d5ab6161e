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

// ------------------------------------------------------------------ fused epilogues
// Run by the 4 epilogue warps (128 threads, named barrier 1) of the CTA that
// stored a tile's last piece.  The rows are processed in chunks staged in
// shared memory (two buffers, one mbarrier each): one thread issues a bulk
// copy per (row, piece) and per extra row slice, the 4 warps consume the
// chunk one row per warp at a time, lane l owning the tile's columns
// 4l .. 4l + 3, while the next chunk is in flight.

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ uint2 pack_bf16x4(float a, float b, float c, float d, uint32_t (&bits)[4]) {
  const __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
  uint2 u;
  u.x = *reinterpret_cast<const uint32_t *>(&lo);
  u.y = *reinterpret_cast<const uint32_t *>(&hi);
  bits[0] = u.x & 0xffffu;
  bits[1] = u.x >> 16;
  bits[2] = u.y & 0xffffu;
  bits[3] = u.y >> 16;
  return u;
}

__device__ __forceinline__ void unpack_bf16x4(uint2 u, float (&v)[4], uint32_t (&bits)[4]) {
  bits[0] = u.x & 0xffffu;
  bits[1] = u.x >> 16;
  bits[2] = u.y & 0xffffu;
  bits[3] = u.y >> 16;
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(bits[i] << 16);
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Shared-memory staging of the fix-ups.
struct FixStage {
  uint32_t sbase;   // smem address of buffer 0 (buffer 1 follows)
  uint8_t *gbase;   // generic address of buffer 0
  uint32_t bytes;   // per buffer
  uint32_t bar;     // mbarriers of buffers 0 and 1 (8 bytes apart)
  uint32_t uses[2]; // completed phases waited per buffer (the same in every thread)
  int *rows;        // smem [BN]: global row (rowmap) of each packed row of the tile's pass
  int32_t *status;
  volatile int *abort;
};

// Arrival of this CTA at a counter (after its global stores): true for the
// arrival that makes it reach `total` (that CTA resets it).  All 128 epilogue
// threads call it; only they use named barrier 1.
__device__ __forceinline__ bool epi_arrive(int32_t *cnt, int total, int *s_flag, int ew, int lane) {
  __threadfence();
  epi_bar();
  if (ew == 0 && lane == 0) {
    const int old = atomicAdd(cnt, 1);
    const int last = (old == total - 1);
    if (last) *cnt = 0;  // every arrival has happened: reset for the next launch
    *s_flag = last;
  }
  epi_bar();
  const bool last = *s_flag != 0;
  if (last) {
    __threadfence();
    fence_proxy_async_global();  // the other CTAs' stores, next read by bulk copies
  }
  return last;
}

// Rows [0, mrows) of a pass in chunks of floor(bytes / row_bytes) rows: issue(r,
// dst, bar) (one thread) copies packed row r's data to smem address dst;
// compute(r, src) (one warp) consumes it from generic address src.
template <class Issue, class Compute>
__device__ __forceinline__ void staged_rows(FixStage &st, int mrows, uint32_t row_bytes, int ew, int lane,
                                            Issue issue, Compute compute) {
  const int R = max(1, min(mrows, (int)(st.bytes / row_bytes)));
  const int nch = (mrows + R - 1) / R;
  auto post = [&](int c) {
    const int b = c & 1, r0 = c * R, r1 = min(mrows, r0 + R);
    const uint32_t bar = st.bar + 8u * (uint32_t)b;
    mbar_expect_tx(bar, (uint32_t)(r1 - r0) * row_bytes);
    for (int r = r0; r < r1; ++r) issue(r, st.sbase + (uint32_t)b * st.bytes + (uint32_t)(r - r0) * row_bytes, bar);
  };
  if (ew == 0 && lane == 0) post(0);
  for (int c = 0; c < nch; ++c) {
    const int b = c & 1;
    // buffer b ^ 1 was released by the barrier that ended chunk c - 1
    if (c + 1 < nch && ew == 0 && lane == 0) post(c + 1);
    const uint32_t bar = st.bar + 8u * (uint32_t)b, par = st.uses[b] & 1u;
    if (!wait_bounded(bar, par, st.abort, st.status)) wait_drain(bar, par);  // the copies land before reuse
    ++st.uses[b];
    const int r0 = c * R, r1 = min(mrows, r0 + R);
    for (int r = r0 + ew; r < r1; r += 4) compute(r, st.gbase + (size_t)b * st.bytes + (size_t)(r - r0) * row_bytes);
    epi_bar();
  }
}

__device__ __forceinline__ float4 piece_sum(const uint8_t *src, int ns, int lane) {
  float4 v = reinterpret_cast<const float4 *>(src)[lane];
  for (int sp = 1; sp < ns; ++sp) {
    const float4 w = reinterpret_cast<const float4 *>(src + sp * 512)[lane];
    v.x += w.x;
    v.y += w.y;
    v.z += w.z;
    v.w += w.w;
  }
  return v;
}

// the ns pieces of packed row pr, 128 fp32 columns from output column col0
__device__ __forceinline__ void issue_pieces(const TcParams &p, int ns, int pr, size_t col0, uint32_t dst, uint32_t bar) {
  for (int sp = 0; sp < ns; ++sp)
    bulk_g2s(dst + 512u * (uint32_t)sp, p.out + (size_t)sp * (size_t)p.geo.slot_stride + (size_t)pr * p.ldc + col0, 512,
             bar);
}

// EPI_QKV on tile t of segment seg (0 q, 1 k, 2 v).
__device__ void fix_qkv(const TcParams &p, FixStage &st, int t, int seg, int m0, int mrows, int ns, int ew,
                        int lane) {
  const EpiArgs &e = p.e;
  const int hd = e.hd, half = hd >> 1;
  const int tcol0 = (t - p.seg_tile0[seg]) * 128;
  const int tcol = tcol0 + lane * 4;  // column within the segment
  const int head = tcol / hd, j4 = tcol - head * hd;
  const bool first = j4 < half;
  const int jr = first ? j4 : j4 - half;  // rotation index of the 4 pairs
  const int xl = half >> 2;               // lane distance to the partner half
  const size_t col0 = (size_t)p.seg_col0[seg] + (size_t)tcol0;
  const bool rot = seg < 2 && e.use_rope;
  bf16 *Q = static_cast<bf16 *>(e.Q), *Kc = static_cast<bf16 *>(e.Kc), *Vc = static_cast<bf16 *>(e.Vc);
  staged_rows(
      st, mrows, 512u * (uint32_t)ns, ew, lane,
      [&](int r, uint32_t dst, uint32_t bar) { issue_pieces(p, ns, m0 + r, col0, dst, bar); },
      [&](int r, const uint8_t *src) {
        const int pr = m0 + r;
        float4 v = piece_sum(src, ns, lane);
        const int row = st.rows[r];
        const int b = row / e.N, i = row - b * e.N;
        if (rot) {
          const float o[4] = {__shfl_xor_sync(0xffffffffu, v.x, xl), __shfl_xor_sync(0xffffffffu, v.y, xl),
                              __shfl_xor_sync(0xffffffffu, v.z, xl), __shfl_xor_sync(0xffffffffu, v.w, xl)};
          float a[4] = {v.x, v.y, v.z, v.w};
          const float2 *cs = e.rope_tab + (size_t)i * half + jr;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 c = cs[k];
            a[k] = first ? a[k] * c.x - o[k] * c.y : a[k] * c.x + o[k] * c.y;
          }
          v = make_float4(a[0], a[1], a[2], a[3]);
        }
        if (seg == 2 && tcol == 0 && e.stale_l) e.stale_l[row] = 0;  // the layer recomputes this row
        bf16 *dst = seg == 0 ? Q + (size_t)pr * e.H * hd + (size_t)head * hd
                             : (seg == 1 ? Kc : Vc) + (((size_t)b * e.Hkv + head) * e.N + i) * hd;
        uint32_t bits[4];
        *reinterpret_cast<uint2 *>(dst + j4) = pack_bf16x4(v.x, v.y, v.z, v.w, bits);
      });
}

// EPI_O on tile t (columns t * 128 .. of D).
__device__ void fix_o(const TcParams &p, FixStage &st, int t, int m0, int mrows, int ns, int ew, int lane) {
  const EpiArgs &e = p.e;
  const int col0 = t * 128, col = col0 + lane * 4;
  const bf16 *Hl = static_cast<const bf16 *>(e.Hl);
  bf16 *u = static_cast<bf16 *>(e.u);
  const float4 g = *reinterpret_cast<const float4 *>(e.g2 + col);
  const uint32_t pb = 512u * (uint32_t)ns;
  staged_rows(
      st, mrows, pb + 256u, ew, lane,
      [&](int r, uint32_t dst, uint32_t bar) {
        issue_pieces(p, ns, m0 + r, (size_t)col0, dst, bar);
        bulk_g2s(dst + pb, Hl + (size_t)st.rows[r] * e.D + col0, 256, bar);
      },
      [&](int r, const uint8_t *src) {
        const int pr = m0 + r;
        const float4 v = piece_sum(src, ns, lane);
        float x[4];
        uint32_t xb[4];
        unpack_bf16x4(reinterpret_cast<const uint2 *>(src + pb)[lane], x, xb);
        const float4 hm = make_float4(x[0] + v.x, x[1] + v.y, x[2] + v.z, x[3] + v.w);
        *reinterpret_cast<float4 *>(e.hmid + (size_t)pr * e.D + col) = hm;
        uint32_t bits[4];
        *reinterpret_cast<uint2 *>(u + (size_t)pr * e.D + col) =
            pack_bf16x4(hm.x * g.x, hm.y * g.y, hm.z * g.z, hm.w * g.w, bits);
        double ss = (double)hm.x * (double)hm.x + (double)hm.y * (double)hm.y + (double)hm.z * (double)hm.z +
                    (double)hm.w * (double)hm.w;
        ss = warp_sum_d(ss);
        if (lane == 0) e.ssq[(size_t)pr * e.ssq_ld + t] = ss;
      });
}

// EPI_GU on tile t: gate tiles are [0, F/128), up tiles [F/128, 2F/128).
__device__ void fix_gu(const TcParams &p, FixStage &st, int t, int pass, int m0, int mrows, int ns, int ew,
                       int lane, int *s_flag) {
  const EpiArgs &e = p.e;
  const int ft = e.F / 128, ntd = e.D / 128;
  const int col0 = t * 128, col = col0 + lane * 4;  // column of [gate | up]
  const uint32_t pb = 512u * (uint32_t)ns, sb = 8u * (uint32_t)e.ssq_ld;
  staged_rows(
      st, mrows, pb + sb, ew, lane,
      [&](int r, uint32_t dst, uint32_t bar) {
        issue_pieces(p, ns, m0 + r, (size_t)col0, dst, bar);
        bulk_g2s(dst + pb, e.ssq + (size_t)(m0 + r) * e.ssq_ld, sb, bar);
      },
      [&](int r, const uint8_t *src) {
        const int pr = m0 + r;
        float4 v = piece_sum(src, ns, lane);
        const double *sq = reinterpret_cast<const double *>(src + pb);
        double ss = 0.0;
        for (int k = lane; k < ntd; k += 32) ss += sq[k];
        ss = warp_sum_d(ss);
        const float inv = (float)(1.0 / sqrt(ss / (double)e.D + (double)e.eps));
        v.x *= inv;
        v.y *= inv;
        v.z *= inv;
        v.w *= inv;
        *reinterpret_cast<float4 *>(p.out + (size_t)pr * p.ldc + col) = v;  // slot 0 now holds the result
      });
  const int pair = t < ft ? t : t - ft;
  if (!epi_arrive(e.pass_cnt + (size_t)pass * ft + pair, 2, s_flag, ew, lane)) return;
  // second tile of the pair: act = silu(gate) * up over the pair's 128 columns
  const int j0 = pair * 128, j = j0 + lane * 4;
  bf16 *act = static_cast<bf16 *>(e.act);
  staged_rows(
      st, mrows, 1024u, ew, lane,
      [&](int r, uint32_t dst, uint32_t bar) {
        const float *row = p.out + (size_t)(m0 + r) * p.ldc;
        bulk_g2s(dst, row + j0, 512, bar);
        bulk_g2s(dst + 512u, row + e.F + j0, 512, bar);
      },
      [&](int r, const uint8_t *src) {
        const float4 gt = reinterpret_cast<const float4 *>(src)[lane];
        const float4 up = reinterpret_cast<const float4 *>(src + 512)[lane];
        uint32_t bits[4];
        *reinterpret_cast<uint2 *>(act + (size_t)(m0 + r) * e.F + j) =
            pack_bf16x4(gt.x / (1.0f + expf(-gt.x)) * up.x, gt.y / (1.0f + expf(-gt.y)) * up.y,
                        gt.z / (1.0f + expf(-gt.z)) * up.z, gt.w / (1.0f + expf(-gt.w)) * up.w, bits);
      });
}

// EPI_DOWN on tile t (columns t * 128 .. of D).
__device__ void fix_down(const TcParams &p, FixStage &st, int t, int pass, int m0, int mrows, int ns, int ew,
                         int lane, int *s_flag) {
  const EpiArgs &e = p.e;
  const int ntd = e.D / 128;
  const int col0 = t * 128, col = col0 + lane * 4;
  const bool want_d = e.d_next != nullptr;
  bf16 *Hn = static_cast<bf16 *>(e.Hn);
  float gg[4] = {0.f, 0.f, 0.f, 0.f};
  if (want_d) {
    const float4 g = *reinterpret_cast<const float4 *>(e.g_next + col);
    gg[0] = g.x;
    gg[1] = g.y;
    gg[2] = g.z;
    gg[3] = g.w;
  }
  const uint32_t pb = 512u * (uint32_t)ns;
  staged_rows(
      st, mrows, pb + 512u + 256u, ew, lane,
      [&](int r, uint32_t dst, uint32_t bar) {
        issue_pieces(p, ns, m0 + r, (size_t)col0, dst, bar);
        bulk_g2s(dst + pb, e.hmid + (size_t)(m0 + r) * e.D + col0, 512, bar);
        bulk_g2s(dst + pb + 512u, Hn + (size_t)st.rows[r] * e.D + col0, 256, bar);  // the cached row
      },
      [&](int r, const uint8_t *src) {
        const int pr = m0 + r;
        const float4 v = piece_sum(src, ns, lane);
        const float4 hm = reinterpret_cast<const float4 *>(src + pb)[lane];
        float nv[4] = {hm.x + v.x, hm.y + v.y, hm.z + v.z, hm.w + v.w};
        uint32_t nb[4];
        const uint2 packed = pack_bf16x4(nv[0], nv[1], nv[2], nv[3], nb);
        if (want_d) {
          float ov[4];
          uint32_t ob[4];
          unpack_bf16x4(reinterpret_cast<const uint2 *>(src + pb + 512)[lane], ov, ob);
          double dot = 0.0, nx = 0.0, ny = 0.0;
          bool same = true;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            same = same && (nb[k] == ob[k]);
            const double a = (double)gg[k] * (double)__uint_as_float(nb[k] << 16), b = (double)gg[k] * (double)ov[k];
            dot += a * b;
            nx += a * a;
            ny += b * b;
          }
          dot = warp_sum_d(dot);
          nx = warp_sum_d(nx);
          ny = warp_sum_d(ny);
          same = __all_sync(0xffffffffu, same);
          if (lane == 0) {
            double *o = e.dpart + ((size_t)pr * ntd + t) * 4;
            o[0] = dot;
            o[1] = nx;
            o[2] = ny;
            o[3] = same ? 1.0 : 0.0;
          }
        }
        *reinterpret_cast<uint2 *>(Hn + (size_t)st.rows[r] * e.D + col) = packed;
      });
  if (!want_d) return;
  if (!epi_arrive(e.pass_cnt + pass, ntd, s_flag, ew, lane)) return;
  // last tile of the pass: the next-layer d of every row of the pass
  staged_rows(
      st, mrows, 32u * (uint32_t)ntd, ew, lane,
      [&](int r, uint32_t dst, uint32_t bar) {
        bulk_g2s(dst, e.dpart + (size_t)(m0 + r) * ntd * 4, 32u * (uint32_t)ntd, bar);
      },
      [&](int r, const uint8_t *src) {
        const double *o = reinterpret_cast<const double *>(src);
        double dot = 0.0, nx = 0.0, ny = 0.0;
        bool same = true;
        for (int k = lane; k < ntd; k += 32) {
          dot += o[4 * k];
          nx += o[4 * k + 1];
          ny += o[4 * k + 2];
          same = same && (o[4 * k + 3] != 0.0);
        }
        dot = warp_sum_d(dot);
        nx = warp_sum_d(nx);
        ny = warp_sum_d(ny);
        same = __all_sync(0xffffffffu, same);
        if (lane == 0) {
          const int row = st.rows[r];
          e.d_next[row] = finish_cosine_distance(dot, nx, ny, same);
          if (e.stale_next && !same) e.stale_next[row] = 1;  // H_{l+1} row changed
        }
      });
}

template <int BN>
__global__ void __launch_bounds__(kTcThreads, 1) k_gemm_tc(const __grid_constant__ TcParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[2 * kTcMaxA + 2 * kTcMaxB + 7];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ int s_epi_ok[4], s_epi_flag;
  __shared__ int s_rows[256];  // fused epilogues: global rows of the pass being fixed up

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
  // fused epilogues: two fix-up staging buffers after the rings (the weight
  // ring keeps >= 6 stages, which the pure weight stream needs)
  const uint32_t fix_bytes = p.epi_mode >= EPI_QKV ? 2u * kFixBuf : 0u;
  int SA = (int)((p.smem_bytes - 1024u - (uint32_t)SB * b_stage - fix_bytes) / kTcABytes);
  SA = SA > kTcMaxA ? kTcMaxA : SA;
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t bbase = sbase + (uint32_t)SA * kTcABytes;
  const uint32_t fbase = bbase + (uint32_t)SB * b_stage;
  const uint32_t bar0 = smem_u32(bars);
  // two TMEM accumulators (columns [0, BN) and [BN, 2 BN)) alternate between fragments
#define FULL_A(s) (bar0 + 8u * (uint32_t)(s))
#define EMPTY_A(s) (bar0 + 8u * (uint32_t)(kTcMaxA + (s)))
#define FULL_B(s) (bar0 + 8u * (uint32_t)(2 * kTcMaxA + (s)))
#define EMPTY_B(s) (bar0 + 8u * (uint32_t)(2 * kTcMaxA + kTcMaxB + (s)))
  const uint32_t tfull0 = bar0 + 8u * (uint32_t)(2 * kTcMaxA + 2 * kTcMaxB), tempty0 = tfull0 + 16u,
                 drain = tfull0 + 32u, fixbar = tfull0 + 40u;
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
    mbar_init(fixbar, 1);
    mbar_init(fixbar + 8u, 1);
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
    const bool fused = p.epi_mode >= EPI_QKV;
    const int ew = warp - 2;  // epilogue warp 0..3 (row interleave of the fused epilogues)
    FixStage st;
    st.sbase = fbase;
    st.gbase = smem_raw + (fbase - smem_u32(smem_raw));
    st.bytes = kFixBuf;
    st.bar = fixbar;
    st.uses[0] = st.uses[1] = 0;
    st.rows = s_rows;
    st.status = p.status;
    st.abort = abort_v;
    // the fused epilogues read what the previous launches wrote (H_l rows, the
    // row sums of squares, hmid): wait for them like the activation producer
    if (fused) griddep_wait();
    while (next_frag(p, passes, it, f)) {
      const int m0 = it.pass * BN;
      const int mrows = min(BN, M - m0);
      const uint32_t acc = nfrag & 1u, use = nfrag >> 1;
      const uint32_t tacc = tmem + acc * (uint32_t)BN + ((uint32_t)(q * 32) << 16);
      bool okw = __all_sync(0xffffffffu, wait_bounded(TFULL(acc), use & 1u, abort_v, p.status));
      if (fused) {
        // the 4 warps meet at named barriers below: they leave together or not at all
        if (lane == 0) s_epi_ok[ew] = okw ? 1 : 0;
        epi_bar();
        okw = (s_epi_ok[0] & s_epi_ok[1] & s_epi_ok[2] & s_epi_ok[3]) != 0;
      }
      if (!okw) break;
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
          const int tok = it.pass * BN + mt * 128 + q * 32 + lane;
          float *zdst = (p.zout && tok < M) ? p.zout + (int64_t)p.zrow[tok] * p.ldz + vbase : nullptr;
          for (int c = 0; c < 128; c += 16) {
            float v[16];
            tmem_ld16(tm + (uint32_t)c, v);
            if (zdst) {
#pragma unroll
              for (int j = 0; j < 16; ++j)
                if (vbase + c + j < p.seg_rows[0]) zdst[c + j] = v[j];
            }
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
      if (fused) {
        const int ns = sk_nslots(p.geo, f.tile);
        if (epi_arrive(p.e.tile_cnt + (size_t)it.pass * p.geo.n_tiles + f.tile, ns, &s_epi_flag, ew, lane)) {
          for (int r = threadIdx.x - 64; r < mrows; r += 128) s_rows[r] = p.e.rowmap[m0 + r];
          epi_bar();
          if (p.epi_mode == EPI_QKV)
            fix_qkv(p, st, f.tile, f.seg, m0, mrows, ns, ew, lane);
          else if (p.epi_mode == EPI_O)
            fix_o(p, st, f.tile, m0, mrows, ns, ew, lane);
          else if (p.epi_mode == EPI_GU)
            fix_gu(p, st, f.tile, it.pass, m0, mrows, ns, ew, lane, &s_epi_flag);
          else
            fix_down(p, st, f.tile, it.pass, m0, mrows, ns, ew, lane, &s_epi_flag);
        }
      }
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
  prefer_max_smem(reinterpret_cast<const void *>(k_gemm_tc<BN>));
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
