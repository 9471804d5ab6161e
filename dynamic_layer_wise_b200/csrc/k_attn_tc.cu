// Attention of the recomputed queries over all N cached keys of their
// sequence (bidirectional, unmasked; [DLLM] "研究背景与动机") on the 5th-gen
// tensor cores.
//
// One CTA per (sequence b, kv head, key split, tile of 128 queries); a query
// is a (packed row, query head) pair of the kv head's GQA group and owns one
// TMEM lane.  The split's keys are walked in chunks of 128:
//
//   warp 0   TMA producer: K and V chunks (128 keys x hd, 128-byte swizzle)
//            into two rings (a K stage is free once S_j is computed, a V
//            stage once P_j V_j is accumulated)
//   warp 1   MMA issuer (one thread): S_j = Q K_j^T into one of two TMEM S
//            buffers (M = 128 queries, N = 128 keys, K = hd), and
//            O += P_j V_j (M = 128, N = hd, K = 128 keys) with P_j read from
//            tensor memory and V the B operand in MN-major form, straight
//            from its TMA layout
//   warps 2-17 softmax, four warpgroups: thread = (query row, one of four
//            32-key parts of the chunk); reads its part of the S row from
//            TMEM, combines the row max with the other parts' threads, keeps
//            the running max and its share of the sum (log2 domain), rescales
//            its quarter of the O row in TMEM when the max grows, writes its
//            part of P (bf16 pairs) into one of two TMEM P buffers, and
//            finally stores its quarter of O
//
// S_{j+1} is computed while the softmax of chunk j runs, and P_j has a TMEM
// buffer of its own, so the softmax of chunk j + 1 does not wait for P_j V_j
// unless the running max moved and O must be rescaled.  With one key split
// the CTA normalises and stores bf16 rows.  With several, the splits of one
// (sequence, kv head, query tile) run as one thread-block cluster: each CTA
// stages its (O, max, sum) rows in its own shared memory and, after a cluster
// barrier, merges a slice of the rows by reading its siblings' rows through
// distributed shared memory (summed in split order: deterministic).
// Every mbarrier wait is bounded by wall-clock time; on expiry the CTA sets
// DCU_ST_TIMEOUT, drains its copies and MMAs in flight, frees TMEM and exits.
#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace dcu {
namespace {

constexpr int kQT = 128;      // queries per tile (TMEM lanes)
constexpr int kKC = 128;      // keys per chunk (S columns)
constexpr int kParts = 4;                     // softmax warpgroups: key parts of a chunk
constexpr int kPartKeys = kKC / kParts;        // keys of a part (32)
constexpr int kSoftThreads = 128 * kParts;     // softmax threads
constexpr int kThreads = 64 + kSoftThreads;   // warps: TMA, MMA, 4 x kParts softmax

template <int HD>
struct TcAttnCfg {
  static constexpr uint32_t kQBytes = (uint32_t)kQT * HD * 2;      // Q tile, HD / 64 swizzle blocks of 16 KB
  static constexpr uint32_t kKVBytes = (uint32_t)kKC * HD * 2;     // K (or V) of one chunk
  static constexpr int kKStages = HD == 128 ? 3 : 4;               // K ring depth
  static constexpr int kVStages = HD == 128 ? 2 : 4;               // V ring depth
  static constexpr uint32_t kSmem = kQBytes + (kKStages + kVStages) * kKVBytes + 1024;  // + alignment slack
  // S buffers [0, 128), [128, 256); O [256, 256 + HD); P buffers (128 keys
  // as bf16 pairs) [384, 448), [448, 512)
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kPCol = 384;
  static_assert(256 + HD <= kPCol, "O and the P buffers overlap");
};

struct TcAttnArgs {
  CUtensorMap kmap, vmap;   // the layer's K / V as [B*Hkv*N rows][hd], box 64 x 128, 128-byte swizzle
  const bf16 *Q;            // [cap][H][hd]
  bf16 *out;                // [cap][H][hd]
  const int32_t *seq_off;   // [B + 1] packed-row offsets of the sequences
  int32_t *status;          // device status word (DCU_ST_TIMEOUT)
  int B, N, H, Hkv, splits, kc, qt_grid;
  float scale_log2;         // log2(e) / sqrt(hd)
};

// Byte offset of the 16-byte chunk c (elements 8c .. 8c+7 along K) of row r in a
// K-major operand tile of 128 rows written in the 128-byte swizzle layout TMA
// produces: 64-element column blocks of 128 rows x 128 B, chunk c' = c ^ (r & 7).
__device__ __forceinline__ uint32_t sw128_off(int r, int c) {
  return (uint32_t)(c >> 3) * 16384u + (uint32_t)r * 128u + ((uint32_t)((c & 7) ^ (r & 7)) << 4);
}

__device__ __forceinline__ void cp_async16_z(uint32_t dst, const void *src, bool valid) {
  const int n = valid ? 16 : 0;  // zero-fill when invalid
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// Cluster-wide barrier (all threads of every CTA of the cluster; arrive has
// release and wait acquire semantics for shared memory of the cluster).
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ float4 ld_dsmem_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ float2 ld_dsmem_f2(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared::cluster.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ void tmem_wait_tie(uint32_t (&r)[32]) { tmem_wait_ld_tie32(r); }
__device__ __forceinline__ void tmem_wait_tie(uint32_t (&r)[64]) { tmem_wait_ld_tie64(r); }
__device__ __forceinline__ void tmem_wait_tie(uint32_t (&r)[128]) { tmem_wait_ld_tie128(r); }

// 2^x by the SFU's approximate base-2 exponential (PTX ex2.approx.ftz.f32:
// relative error about 2^-22, results below 2^-126 flush to 0); P is rounded
// to bf16 right after, so the approximation is far inside that rounding.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

template <int HD>
__global__ void __launch_bounds__(kThreads, 1) k_attn_tc(const __grid_constant__ TcAttnArgs a) {
  using C = TcAttnCfg<HD>;
  constexpr uint32_t kStagePitch = (uint32_t)HD * 4u + 16u;  // staged O row (fp32), padded against bank conflicts
  extern __shared__ __align__(16) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[4 * 4 + 2 + 2 + 1 + 1 + 1 + 1];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ float s_w[kQT][8];     // split weights of the merge
  __shared__ float2 s_ml[kQT];      // this split's (max, sum) per query row
  __shared__ float s_mx[2][kParts][kQT];  // [chunk parity][part] chunk max per row (row-group exchange)
  __shared__ float s_l[kParts][kQT];      // [part] share of the row sum

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int item = blockIdx.x;
  const int per_b = a.Hkv * a.splits * a.qt_grid;
  const int b = item / per_b;
  item -= b * per_b;
  const int qt0 = item / (a.Hkv * a.splits);
  item -= qt0 * a.Hkv * a.splits;
  const int kvh = item / a.splits, ks = item - kvh * a.splits;
  const int k_begin = ks * a.kc;
  // (CTA-uniform exits before any barrier or TMEM use)
  if (b >= a.B || k_begin >= a.N) {
    pdl_enter();
    return;
  }
  const int k_end = min(a.N, k_begin + a.kc);
  const int nch = (k_end - k_begin + kKC - 1) / kKC;

  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  // kv_s: the K ring, then the V ring (after the last chunk of a tile, the
  // staging area of the cluster merge)
  const uint32_t q_s = sbase, kv_s = sbase + C::kQBytes, v_s = kv_s + (uint32_t)C::kKStages * C::kKVBytes;
  const uint32_t bar0 = smem_u32(bars);
#define K_FULL(s) (bar0 + 8u * (uint32_t)(s))
#define K_EMPTY(s) (bar0 + 8u * (uint32_t)(4 + (s)))
#define V_FULL(s) (bar0 + 8u * (uint32_t)(8 + (s)))
#define V_EMPTY(s) (bar0 + 8u * (uint32_t)(12 + (s)))
#define S_FULL(i) (bar0 + 8u * (uint32_t)(16 + (i)))
  // P_FULL per S / P buffer: the softmax warps are not in step with one
  // another (only the two of a row pair are), and a warp may finish P_{j+1}
  // before a slower one finishes P_j; with one barrier for both, such early
  // arrivals would count towards chunk j's phase.  A warp reaches P_{j+2}
  // only after every warp's P_j (S_{j+2} follows P_j V_j), so per buffer the
  // phases stay in order.
#define P_FULL(i) (bar0 + 8u * (uint32_t)(18 + (i)))
  // O_DONE: once per chunk, after P_j V_j (the rescale waits); O_FINAL: once
  // per query tile, after its last P V.  The softmax skips O_DONE phases, so
  // its wait for the tile's last chunk could alias an older phase; O_FINAL
  // cannot.
  const uint32_t O_DONE = bar0 + 8u * 20u, DRAIN = bar0 + 8u * 21u, Q_FULL = bar0 + 8u * 22u,
                 O_FINAL = bar0 + 8u * 23u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kKStages; ++s) {
      mbar_init(K_FULL(s), 1);
      mbar_init(K_EMPTY(s), 1);
    }
    for (int s = 0; s < C::kVStages; ++s) {
      mbar_init(V_FULL(s), 1);
      mbar_init(V_EMPTY(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(S_FULL(i), 1);
      mbar_init(P_FULL(i), kSoftThreads / 32);  // one arrive per softmax warp
    }
    mbar_init(O_DONE, 1);
    mbar_init(O_FINAL, 1);
    mbar_init(DRAIN, 1);
    mbar_init(Q_FULL, kSoftThreads / 32);  // one arrive per softmax warp
    abort_flag = 0;
    fence_barrier_init();
  }
  // This split's first K / V chunks into L2 while the previous launch (the QKV
  // epilogue, which rewrites only the recomputed rows) still runs; L2 stays
  // coherent with those writes, so the loads after the wait see them.
  if (threadIdx.x == 0) {
    prefetch_tmap(&a.kmap);
    prefetch_tmap(&a.vmap);
    const int y0 = (b * a.Hkv + kvh) * a.N + k_begin;
    const int npf = nch < 4 ? nch : 4;
    for (int j = 0; j < npf; ++j)
#pragma unroll
      for (int h = 0; h < HD / 64; ++h) {
        tma_prefetch_2d(&a.kmap, h * 64, y0 + j * kKC);
        tma_prefetch_2d(&a.vmap, h * 64, y0 + j * kKC);
      }
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  volatile int *abort_v = &abort_flag;

  // Q, K and V are written by the previous launches (the QKV epilogue)
  griddep_wait();
  allow_dependents();

  const int G = a.H / a.Hkv;
  const int row0 = a.seq_off[b], nq = (a.seq_off[b + 1] - row0) * G;
  const int rowbase = (b * a.Hkv + kvh) * a.N;  // first K / V row of this (sequence, kv head)
  uint32_t cbase = 0;                            // chunks this CTA has walked before the current tile

  uint32_t ntile = 0;                            // query tiles this CTA has walked
  for (int qt = qt0; qt * kQT < nq; qt += a.qt_grid, ++ntile) {
    // after a timed-out wait (read after the barrier that ends every tile:
    // uniform in the CTA) a lone CTA stops; the CTAs of a cluster keep walking
    // the tiles, every wait now failing at once, so their cluster barriers match
    if (a.splits == 1 && *abort_v) break;
    if (warp == 0) {
      // ---- TMA producers: lane 0 fills the K ring, lane 1 the V ring, so a K
      // load never queues behind a V stage still held by P V
      if (lane < 2) {
        const bool is_v = lane == 1;
        const uint32_t stages = is_v ? (uint32_t)C::kVStages : (uint32_t)C::kKStages;
        const uint32_t ring = is_v ? v_s : kv_s;
        const uint32_t full0 = is_v ? V_FULL(0) : K_FULL(0), empty0 = is_v ? V_EMPTY(0) : K_EMPTY(0);
        const CUtensorMap *map = is_v ? &a.vmap : &a.kmap;
        bool ok = true;
        uint32_t issued = 0;
        const uint64_t pol = policy_evict_normal();
        for (int j = 0; j < nch; ++j) {
          const uint32_t g = cbase + (uint32_t)j, st = g % stages;
          const int y = rowbase + k_begin + j * kKC;  // rows past the split are masked, past the tensor zero
          if (!wait_bounded(empty0 + 8u * st, ((g / stages) & 1u) ^ 1u, abort_v, a.status)) {
            ok = false;
            break;
          }
          mbar_expect_tx(full0 + 8u * st, C::kKVBytes);
#pragma unroll
          for (int h = 0; h < HD / 64; ++h)
            tma_load_2d(ring + st * C::kKVBytes + (uint32_t)h * 16384u, map, h * 64, y, full0 + 8u * st, pol);
          ++issued;
        }
        if (!ok) {  // wait, bounded, for the copies this tile still has in flight
          for (uint32_t j = 0; j < issued; ++j) {
            const uint32_t g = cbase + j;
            wait_drain(full0 + 8u * (g % stages), (g / stages) & 1u);
          }
        }
      }
    } else if (warp == 1) {
      // ---- MMA issuer
      if (lane == 0) {
        const uint32_t idesc_s = idesc_bf16(kQT, kKC);
        const uint32_t idesc_o = idesc_bf16_bmn(kQT, HD);
        const uint32_t o_tm = tmem + 256u;
        bool ok = true, any = false;
        // P_i from its TMEM buffer (16 keys = 8 columns per K step), V_i from its
        // stage.  The softmax writes P_{i+2} into the same buffer only after
        // S_{i+2}, whose commit follows the completion of these MMAs.
        auto issue_pv = [&](int i) -> bool {
          const uint32_t g = cbase + (uint32_t)i, vs = g % C::kVStages;
          if (!wait_bounded(P_FULL(g & 1u), (g >> 1) & 1u, abort_v, a.status) ||
              !wait_bounded(V_FULL(vs), (g / C::kVStages) & 1u, abort_v, a.status))
            return false;
          tc_fence_after();
          const uint32_t vb = v_s + vs * C::kKVBytes, p_tm = tmem + C::kPCol + (g & 1u) * 64u;
#pragma unroll
          for (int kk = 0; kk < kKC / 16; ++kk) {
            const uint64_t vd = sw128_mn_desc(vb + (uint32_t)kk * 2048u, 16384u);
            tc_mma_ts(o_tm, p_tm + (uint32_t)(kk * 8), vd, idesc_o, (i > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(V_EMPTY(vs));  // the stage may be refilled once these MMAs have read it
          tc_commit(O_DONE);
          return true;
        };
        if (!wait_bounded(Q_FULL, ntile & 1u, abort_v, a.status)) ok = false;
        tc_fence_after();
        // S_j's buffer was last read by the softmax of chunk j - 2, which had
        // finished (P_FULL) before P_{j-2} V_{j-2}, issued before these
        for (int j = 0; j < nch && ok; ++j) {
          const uint32_t g = cbase + (uint32_t)j, ks = g % C::kKStages, sb = g & 1u;
          if (!wait_bounded(K_FULL(ks), (g / C::kKStages) & 1u, abort_v, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t kb = kv_s + ks * C::kKVBytes;
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint64_t qd = sw128_desc(q_s + (uint32_t)(kk >> 2) * 16384u) + (uint64_t)(2 * (kk & 3));
            const uint64_t kd = sw128_desc(kb + (uint32_t)(kk >> 2) * 16384u) + (uint64_t)(2 * (kk & 3));
            tc_mma(tmem + sb * (uint32_t)kKC, qd, kd, idesc_s, kk > 0 ? 1u : 0u);
          }
          any = true;
          tc_commit(K_EMPTY(ks));
          tc_commit(S_FULL(sb));
          if (j >= 1 && !issue_pv(j - 1)) ok = false;
        }
        if (ok && !issue_pv(nch - 1)) ok = false;
        if (ok) tc_commit(O_FINAL);  // every P V of the tile is accumulated
        if (!ok && any) {
          tc_commit(DRAIN);
          wait_drain(DRAIN, 0);
        }
      }
    } else {
      // ---- softmax: kParts warpgroups; thread = (query row = TMEM lane, part
      // of the key columns).  Warp w takes keys [32 p, 32 p + 32) of every
      // chunk, p = (w - 2) / 4; the kParts warps w = 2 + 4 p + (w % 4) share
      // the rows 32 (w % 4) .. and combine their row max (and at the end their
      // sums) through shared memory at a named barrier of the row group.
      constexpr int OC = HD / kParts;          // O columns of a part
      const int q4 = warp & 3;
      const int qi = q4 * 32 + lane;
      const int pt = (warp - 2) >> 2;          // key part
      const int st_id = threadIdx.x - 64;      // 0 .. kSoftThreads - 1
      const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
      const uint32_t o_tm = tmem + 256u + lane_off + (uint32_t)(pt * OC);  // this part's O columns
      const float sc = a.scale_log2;
      auto group_sync = [&]() { asm volatile("bar.sync %0, %1;" ::"r"(1 + q4), "r"(32 * kParts) : "memory"); };
      // Q tile -> shared memory (the softmax threads; zero rows past nq),
      // while the producers already stream K / V
      for (int c = st_id; c < kQT * (HD / 8); c += kSoftThreads) {
        const int qr = c / (HD / 8), ch = c - qr * (HD / 8);
        const int q = qt * kQT + qr;
        const bool ok = q < nq;
        const int r = row0 + (ok ? q / G : 0), h = kvh * G + (ok ? q % G : 0);
        cp_async16_z(q_s + sw128_off(qr, ch), a.Q + ((size_t)r * a.H + h) * HD + ch * 8, ok);
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
      asm volatile("cp.async.wait_group 0;" ::: "memory");
      fence_proxy_async_smem();  // the MMA reads Q through the async proxy
      __syncwarp();
      if (lane == 0) mbar_arrive(Q_FULL);
      float m_run = -INFINITY, l_run = 0.f;  // l_run: this part's share of the row sum
      bool alive = true;
      // Every softmax warp walks all nch chunks and meets its row group at each
      // named barrier, also after a timed-out wait (it then skips the work), so
      // the named barriers always match.
      for (int j = 0; j < nch; ++j) {
        const uint32_t g = cbase + (uint32_t)j, sb = g & 1u;
        if (alive) alive = __all_sync(0xffffffffu, wait_bounded(S_FULL(sb), (g >> 1) & 1u, abort_v, a.status));
        const int nvalid = min(kKC, k_end - (k_begin + j * kKC)) - pt * kPartKeys;  // valid keys of this part
        float sv[kPartKeys];
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if (alive) {
          tc_fence_after();
          uint32_t sr[kPartKeys];
          tmem_ld32_issue(tmem + sb * (uint32_t)kKC + lane_off + (uint32_t)(pt * kPartKeys), sr);
          tmem_wait_ld_tie32(sr);
          if (nvalid >= kPartKeys) {  // a full part (every chunk but a ragged last one)
#pragma unroll
            for (int c = 0; c < kPartKeys; ++c) {
              sv[c] = __uint_as_float(sr[c]);
              mx[c & 3] = fmaxf(mx[c & 3], sv[c]);
            }
          } else {
#pragma unroll
            for (int c = 0; c < kPartKeys; ++c) {
              sv[c] = c < nvalid ? __uint_as_float(sr[c]) : -INFINITY;
              mx[c & 3] = fmaxf(mx[c & 3], sv[c]);
            }
          }
        }
        // raw S here; the scale (> 0) commutes with the max and enters the exponent below
        float mc = sc * fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        s_mx[j & 1][pt][qi] = mc;
        group_sync();
#pragma unroll
        for (int o = 0; o < kParts; ++o) mc = fmaxf(mc, s_mx[j & 1][o][qi]);  // the row's chunk max
        if (!alive) continue;
        // The running max only moves when the chunk's max exceeds it by more than
        // 8 (log2 units): P then stays below 2^8 and most chunks need no O
        // rescale.  The result is exact either way (P, the sums and O share m_run).
        const bool grow = mc > m_run + 8.f;  // always on the first chunk (m_run = -inf)
        const float m_new = grow ? mc : m_run;
        const float alpha = grow ? (m_run == -INFINITY ? 0.f : ex2_approx(m_run - m_new)) : 1.f;
        // a rescale of O needs P_{j-1} V_{j-1} accumulated first (P_j has a
        // buffer of its own, so otherwise nothing waits for it).  The parity
        // wait is exact: P_j V_j cannot complete before this warp's P_FULL
        // arrival below, and S_j (seen above) completed after P_{j-2} V_{j-2},
        // issued before it, so O_DONE has completed chunk j - 2 or j - 1.
        if (j >= 1 && __any_sync(0xffffffffu, grow)) {  // warp-uniform: tcgen05.ld / st are collective
          alive = __all_sync(0xffffffffu, wait_bounded(O_DONE, (g - 1u) & 1u, abort_v, a.status));
          if (!alive) continue;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < OC / 16; ++c) {  // this part's OC columns, 16 at a time
            float ov[16];
            tmem_ld16(o_tm + (uint32_t)(c * 16), ov);
#pragma unroll
            for (int e = 0; e < 16; ++e) ov[e] *= alpha;
            tmem_st16(o_tm + (uint32_t)(c * 16), ov);
          }
          tmem_wait_st();
        }
        m_run = m_new;
        // P = 2^(s - m) of this part's valid keys (0 past them), as bf16 pairs:
        // keys 32 pt + 2c, 32 pt + 2c + 1 in column 16 pt + c of P buffer j % 2
        // (the K-major A operand of P_j V_j in tensor memory)
        float ps[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t pk[kPartKeys / 2];
#pragma unroll
        for (int c = 0; c < kPartKeys / 2; ++c) {
          const float p0 = ex2_approx(fmaf(sv[2 * c], sc, -m_new));
          const float p1 = ex2_approx(fmaf(sv[2 * c + 1], sc, -m_new));
          ps[c & 3] += p0 + p1;
          pk[c] = pack2_bf16(p0, p1);
        }
        tmem_st16u(tmem + C::kPCol + sb * 64u + lane_off + (uint32_t)(pt * (kPartKeys / 2)), pk);
        l_run = l_run * alpha + ((ps[0] + ps[1]) + (ps[2] + ps[3]));
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(P_FULL(sb));
      }
      if (alive) alive = __all_sync(0xffffffffu, wait_bounded(O_FINAL, ntile & 1u, abort_v, a.status));
      // the row sum: the parts' shares in part order
      s_l[pt][qi] = l_run;
      group_sync();
      float l_row = 0.f;
#pragma unroll
      for (int o = 0; o < kParts; ++o) l_row += s_l[o][qi];
      if (alive) {
        tc_fence_after();
        float orr[OC];
#pragma unroll
        for (int c = 0; c < OC / 16; ++c) tmem_ld16(o_tm + (uint32_t)(c * 16), *reinterpret_cast<float(*)[16]>(orr + 16 * c));
        const int q = qt * kQT + qi;
        if (q < nq) {
          const int r = row0 + q / G, h = kvh * G + q % G;
          const size_t qidx = (size_t)r * a.H + h;
          if (a.splits == 1) {
            const float inv = 1.f / l_row;
            uint4 *dst = reinterpret_cast<uint4 *>(a.out + qidx * HD + pt * OC);
#pragma unroll
            for (int c = 0; c < OC / 8; ++c)
              dst[c] = make_uint4(pack2_bf16(orr[8 * c] * inv, orr[8 * c + 1] * inv),
                                  pack2_bf16(orr[8 * c + 2] * inv, orr[8 * c + 3] * inv),
                                  pack2_bf16(orr[8 * c + 4] * inv, orr[8 * c + 5] * inv),
                                  pack2_bf16(orr[8 * c + 6] * inv, orr[8 * c + 7] * inv));
          } else {
            // this split's (O, max, sum) of the row, staged in this CTA's shared
            // memory for the cluster merge (the K / V rings are idle by now)
            const uint32_t dst = kv_s + (uint32_t)qi * kStagePitch + (uint32_t)(pt * OC) * 4u;
#pragma unroll
            for (int c = 0; c < OC / 4; ++c)
              st_shared_v4(dst + (uint32_t)c * 16u, __float_as_uint(orr[4 * c]), __float_as_uint(orr[4 * c + 1]),
                           __float_as_uint(orr[4 * c + 2]), __float_as_uint(orr[4 * c + 3]));
            if (pt == 0) s_ml[qi] = make_float2(m_run, l_row);
          }
        }
      }
      tc_fence_before();
    }
    __syncthreads();
    // ---- split merge inside the cluster (the CTAs of one (sequence, kv head,
    // query tile) are the key splits, cluster rank = split): once every CTA has
    // staged its rows, CTA ks merges rows [ks R, ks R + R) of the tile,
    // out = sum_s w_s O_s with w_s = 2^(m_s - M) / sum_s' 2^(m_s' - M) l_s',
    // reading the siblings' shared memory; summed in split order.
    if (a.splits > 1) {
      cluster_sync();  // every CTA's rows are staged (release / acquire)
      const int nqt = min(kQT, nq - qt * kQT);
      const int R = (nqt + a.splits - 1) / a.splits;
      const int t0 = ks * R, t1 = min(nqt, t0 + R);
      const uint32_t ml_base = smem_u32(s_ml);
      if (threadIdx.x < t1 - t0) {
        const int t = t0 + threadIdx.x;
        float2 ml[8];
        float M = -INFINITY;
#pragma unroll
        for (int sp = 0; sp < 8; ++sp)
          if (sp < a.splits) {
            ml[sp] = ld_dsmem_f2(mapa_shared(ml_base + (uint32_t)t * 8u, (uint32_t)sp));
            M = fmaxf(M, ml[sp].x);
          }
        float L = 0.f;
#pragma unroll
        for (int sp = 0; sp < 8; ++sp)
          if (sp < a.splits) L += ml[sp].y * ex2_approx(ml[sp].x - M);
        const float inv = 1.f / L;
#pragma unroll
        for (int sp = 0; sp < 8; ++sp) s_w[threadIdx.x][sp] = sp < a.splits ? ex2_approx(ml[sp].x - M) * inv : 0.f;
      }
      __syncthreads();
      const int items = (t1 - t0) * (HD / 4);
      for (int it = threadIdx.x; it < items; it += kThreads) {
        const int tl = it / (HD / 4), d4 = (it - tl * (HD / 4)) * 4;
        const int t = t0 + tl;
        const uint32_t off = kv_s + (uint32_t)t * kStagePitch + (uint32_t)d4 * 4u;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int s0 = 0; s0 < 8; s0 += 4) {  // 4 splits' loads in flight at a time
          if (s0 >= a.splits) break;
          float4 o[4];
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (s0 + u < a.splits) o[u] = ld_dsmem_f4(mapa_shared(off, (uint32_t)(s0 + u)));
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (s0 + u < a.splits) {
              const float w = s_w[tl][s0 + u];
              acc[0] += o[u].x * w;
              acc[1] += o[u].y * w;
              acc[2] += o[u].z * w;
              acc[3] += o[u].w * w;
            }
        }
        const int q = qt * kQT + t;
        const size_t qidx = (size_t)(row0 + q / G) * a.H + (kvh * G + q % G);
        *reinterpret_cast<uint2 *>(a.out + qidx * HD + d4) =
            make_uint2(pack2_bf16(acc[0], acc[1]), pack2_bf16(acc[2], acc[3]));
      }
      cluster_sync();  // no CTA reuses or leaves its staged rows while a sibling reads them
    }
    cbase += (uint32_t)nch;
    __syncthreads();  // the next tile reuses Q, P, the TMEM buffers and the merge weights
  }
#undef K_FULL
#undef K_EMPTY
#undef V_FULL
#undef V_EMPTY
#undef S_FULL
#undef P_FULL
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace

size_t attn_tc_smem(int hd) { return hd == 128 ? TcAttnCfg<128>::kSmem : TcAttnCfg<64>::kSmem; }

int attn_tc_max_clusters(int hd, int splits) {
  if ((hd != 64 && hd != 128) || splits < 1 || splits > 8) return 0;
  static std::mutex mu;
  static std::vector<std::pair<std::pair<int, int>, std::pair<int, int>>> cache;  // ((dev, hd * 16 + splits), n)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  const int key = hd * 16 + splits;
  std::lock_guard<std::mutex> lock(mu);
  for (const auto &c : cache)
    if (c.first.first == dev && c.first.second == key) return c.second.first;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(splits * 64);
  cfg.blockDim = dim3(kThreads);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)splits;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  cudaError_t e;
  if (hd == 128) {
    static std::atomic<uint64_t> attr_set{0};
    cfg.dynamicSmemBytes = TcAttnCfg<128>::kSmem;
    e = ensure_smem_limit(k_attn_tc<128>, (int)cfg.dynamicSmemBytes, attr_set);
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveClusters(&n, k_attn_tc<128>, &cfg);
  } else {
    static std::atomic<uint64_t> attr_set{0};
    cfg.dynamicSmemBytes = TcAttnCfg<64>::kSmem;
    e = ensure_smem_limit(k_attn_tc<64>, (int)cfg.dynamicSmemBytes, attr_set);
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveClusters(&n, k_attn_tc<64>, &cfg);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  cache.push_back({{dev, key}, {n, 0}});
  return n;
}

cudaError_t launch_attention_tc(const void *Q, const int32_t *seq_off, int B, int N, int H, int Hkv, int hd,
                                const CUtensorMap *kmap, const CUtensorMap *vmap, void *out, int splits, int qt_grid,
                                int32_t *status, cudaStream_t s) {
  if ((hd != 64 && hd != 128) || splits < 1 || splits > 8 || !kmap || !vmap || qt_grid < 1 || N < 1)
    return cudaErrorInvalidValue;
  TcAttnArgs a;
  a.kmap = *kmap;
  a.vmap = *vmap;
  a.status = status;
  a.Q = (const bf16 *)Q;
  a.out = (bf16 *)out;
  a.seq_off = seq_off;
  a.B = B;
  a.N = N;
  a.H = H;
  a.Hkv = Hkv;
  a.splits = splits;
  a.kc = ((N + splits - 1) / splits + kKC - 1) / kKC * kKC;
  // every CTA of a cluster must reach its barriers: every split holds keys
  if ((long long)(splits - 1) * a.kc >= N) return cudaErrorInvalidValue;
  a.qt_grid = qt_grid;
  a.scale_log2 = 1.4426950408889634f / sqrtf((float)hd);
  const int grid = B * Hkv * splits * qt_grid;
  if (grid <= 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;  // the key splits of a tile form one cluster
  attr[1].val.clusterDim.x = (unsigned)splits;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (hd == 128) {
    static std::atomic<uint64_t> attr_set{0};
    cfg.dynamicSmemBytes = TcAttnCfg<128>::kSmem;
    if (cudaError_t e = ensure_smem_limit(k_attn_tc<128>, (int)cfg.dynamicSmemBytes, attr_set)) return e;
    prefer_max_smem(reinterpret_cast<const void *>(k_attn_tc<128>));
    if (cudaError_t e = cudaLaunchKernelEx(&cfg, k_attn_tc<128>, a)) return e;
  } else {
    static std::atomic<uint64_t> attr_set{0};
    cfg.dynamicSmemBytes = TcAttnCfg<64>::kSmem;
    if (cudaError_t e = ensure_smem_limit(k_attn_tc<64>, (int)cfg.dynamicSmemBytes, attr_set)) return e;
    prefer_max_smem(reinterpret_cast<const void *>(k_attn_tc<64>));
    if (cudaError_t e = cudaLaunchKernelEx(&cfg, k_attn_tc<64>, a)) return e;
  }
  return cudaGetLastError();
}

}  // namespace dcu
