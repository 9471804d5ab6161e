// Tensor-core attention of the recomputed queries over all N cached keys of
// their sequence (bidirectional, unmasked; [DLLM] "研究背景与动机").
//
// One CTA per (sequence b, kv head, key split, tile of 128 queries); a query is
// a (packed row, query head) pair of the kv head's GQA group, so the CTA reads
// its K/V chunk from HBM once for every query of the group.  8 warps x 16
// queries; K/V are staged in shared memory in 64-key sub-chunks with cp.async
// (a ring of 4, three sub-chunks in flight ahead of the one in use,
// zero-filled past N); S = Q K^T and O += P V run on
// mma.sync m16n8k16 bf16 (fp32 accumulate) with an online softmax in
// registers.  With several key splits, each CTA writes (O, max, sum) partials
// and k_attn_merge combines them in split order (one thread per query head and
// 4 output dims), so the result does not depend on CTA scheduling.
#include "common.cuh"
#include "kernels.h"

namespace dcu {
namespace {

constexpr int QT = 128;  // queries per CTA
constexpr int KS = 64;   // keys per sub-chunk
constexpr int NST = 4;   // K/V sub-chunk buffers: NST - 1 loads in flight ahead of the one in use

// Q tile bytes (padded rows), rounded to 1024 so the K / V ring that follows
// is aligned for the 128-byte swizzle.
__host__ __device__ constexpr uint32_t attn_q_bytes(int hd) {
  return ((uint32_t)QT * (uint32_t)(hd + 8) * 2u + 1023u) & ~1023u;
}

__device__ __forceinline__ uint32_t smem_u32a(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
  const int n = valid ? 16 : 0;  // zero-fill when invalid
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

struct AttnArgs {
  CUtensorMap kmap, vmap;   // the layer's K / V as [B*Hkv*N rows][hd], box 64 x 64, 128-byte swizzle
  const bf16 *Q;            // [cap][H][hd]
  const bf16 *Kc, *Vc;      // [B][Hkv][N][hd]
  bf16 *out;                // [cap][H][hd]
  const int32_t *seq_off;   // [B + 1] packed-row offsets of the sequences
  float *part_o;            // [splits][cap * H][hd] partial outputs
  float2 *part_ml;          // [splits][cap * H] (max, sum) in log2 units
  int32_t *status;          // device status word (DCU_ST_TIMEOUT)
  int B, N, H, Hkv, splits, kc, qt_grid;
  float scale_log2;         // log2(e) / sqrt(hd)
};

// Shared-memory address of the 16-byte chunk holding elements d .. d+7 of key
// row `key` in a K / V stage written by TMA with the 128-byte swizzle: hd is
// split in 64-wide boxes of 64 rows x 128 B, chunk c of row r sits at chunk
// c ^ (r & 7), so the 8 rows an ldmatrix reads hit 8 different bank groups.
__device__ __forceinline__ uint32_t kv_addr(uint32_t base, int key, int d) {
  return base + (uint32_t)(d >> 6) * 8192u + (uint32_t)key * 128u + ((uint32_t)(((d & 63) >> 3) ^ (key & 7)) << 4);
}

__device__ __forceinline__ void tma_load_2d_a(uint32_t dst, const CUtensorMap *map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// Bounded wait on a K / V stage (all threads): false after 1 s of wall-clock
// time (%globaltimer; try_wait may suspend, so an iteration count is no time
// bound), the caller abandons the tile and the host sees DCU_ST_TIMEOUT.
__device__ __forceinline__ bool kv_wait(uint32_t bar, uint32_t parity, int32_t *status) {
  uint64_t t0 = 0;
  for (uint32_t it = 0;; ++it) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    if (ok) return true;
    if ((it & 63u) == 0u) {
      uint64_t t;
      asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
      if (it == 0) t0 = t;
      else if (t - t0 > 1000000000ull) break;
    }
  }
  if (status) atomicOr(status, DCU_ST_TIMEOUT);
  return false;
}

// Stage layout: K boxes (HD / 64 of 8 KB) then V boxes; NST stages from `ring`.
// Returns false if a K / V stage never landed (the kernel then stops).
template <int HD>
__device__ __forceinline__ bool attn_tile(const AttnArgs &a, uint8_t *sm, uint32_t ring, uint32_t bar0,
                                          uint32_t &chunk_ctr, int b, int kvh, int ks, int qt, int row0, int nq) {
  constexpr int LD = HD + 8;  // padded Q row (elements): 16-byte shift per row, conflict-free ldmatrix
  constexpr int CPR = HD / 8;  // 16-byte chunks per row
  constexpr uint32_t KVB = (uint32_t)HD * 128u;  // bytes of one chunk's K (or V): HD/64 boxes of 8 KB
  constexpr uint32_t STAGE = 2u * KVB;
  bf16 *Qs = reinterpret_cast<bf16 *>(sm);  // [QT][LD]
  const int G = a.H / a.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int k_begin = ks * a.kc;
  const int k_end = min(a.N, k_begin + a.kc);
  const int rowbase = (b * a.Hkv + kvh) * a.N;  // first K / V row of this (sequence, kv head)

  // Q tile -> shared (query q -> packed row row0 + q / G, head kvh * G + q % G)
  for (int c = tid; c < QT * CPR; c += blockDim.x) {
    const int qi = c / CPR, ch = c - qi * CPR;
    const int q = qt * QT + qi;
    const bool ok = q < nq;
    const int r = row0 + (ok ? q / G : 0), h = kvh * G + (ok ? q % G : 0);
    cp_async16(smem_u32a(Qs + qi * LD + ch * 8), a.Q + ((size_t)r * a.H + h) * HD + ch * 8, ok);
  }
  cp_async_commit();
  // K / V sub-chunk j of this tile -> stage (chunk_ctr + j) % NST: one thread
  // issues 2 * HD / 64 TMA boxes (keys past this split are masked below; past
  // the tensor they are zero-filled)
  const uint32_t c0 = chunk_ctr;
  auto load_kv = [&](int j) {
    const uint32_t st = (c0 + (uint32_t)j) % NST;
    const uint32_t dst = ring + st * STAGE, bar = bar0 + 8u * st;
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(STAGE) : "memory");
    const int y = rowbase + k_begin + j * KS;
#pragma unroll
    for (int h = 0; h < HD / 64; ++h) {
      tma_load_2d_a(dst + (uint32_t)h * 8192u, &a.kmap, h * 64, y, bar);
      tma_load_2d_a(dst + KVB + (uint32_t)h * 8192u, &a.vmap, h * 64, y, bar);
    }
  };
  const int n_sub = (k_end - k_begin + KS - 1) / KS;
  chunk_ctr += (uint32_t)n_sub;
  if (tid == 0)
    for (int j = 0; j < NST - 1 && j < n_sub; ++j) load_kv(j);

  float o[HD / 8][4];
#pragma unroll
  for (int i = 0; i < HD / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  uint32_t qf[HD / 16][4];
  const bool warp_active = (qt * QT + warp * 16) < nq;

  for (int sc = 0; sc < n_sub; ++sc) {
    const uint32_t st = (c0 + (uint32_t)sc) % NST;
    const int nxt = sc + NST - 1;  // refills the stage consumed in iteration sc - 1
    if (tid == 0 && nxt < n_sub) load_kv(nxt);
    if (sc == 0) cp_async_wait<0>();
    const bool landed = kv_wait(bar0 + 8u * st, ((c0 + (uint32_t)sc) / NST) & 1u, a.status);
    if (__syncthreads_or(!landed)) {
      // timed out (status is set): wait, bounded, for this tile's copies still
      // in flight so none lands after the CTA has exited, then give up
      if (tid == 0) {
        const int issued = min(n_sub, sc + NST);
        for (int j = sc; j < issued; ++j) {
          const uint32_t cj = c0 + (uint32_t)j;
          kv_wait(bar0 + 8u * (cj % NST), (cj / NST) & 1u, nullptr);
        }
      }
      __syncthreads();
      return false;
    }
    const uint32_t Kt = ring + st * STAGE, Vt = Kt + KVB;
    if (sc == 0 && warp_active) {
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk) {
        const int rr = warp * 16 + (lane & 15), cc = kk * 16 + (lane >> 4) * 8;
        ldsm_x4(smem_u32a(Qs + rr * LD + cc), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
      }
    }
    if (warp_active) {
      float s[KS / 8][4];
#pragma unroll
      for (int j = 0; j < KS / 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk) {
#pragma unroll
        for (int j = 0; j < KS / 16; ++j) {
          // keys 16j .. 16j+15, d 16kk .. 16kk+15
          const int key = j * 16 + (lane & 7) + ((lane >> 4) << 3);
          const int d = kk * 16 + ((lane >> 3) & 1) * 8;
          uint32_t b0, b1, b2, b3;
          ldsm_x4(kv_addr(Kt, key, d), b0, b1, b2, b3);
          mma_bf16(s[2 * j], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b0, b1);
          mma_bf16(s[2 * j + 1], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b2, b3);
        }
      }
      // online softmax (log2 domain); keys past k_end are masked
      const int key_base = k_begin + sc * KS;
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int j = 0; j < KS / 8; ++j) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = key_base + j * 8 + t * 2 + (e & 1);
          const float v = key < k_end ? s[j][e] * a.scale_log2 : -INFINITY;
          s[j][e] = v;
          mx[e >> 1] = fmaxf(mx[e >> 1], v);
        }
      }
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        mx[h2] = fmaxf(mx[h2], __shfl_xor_sync(0xffffffffu, mx[h2], 1));
        mx[h2] = fmaxf(mx[h2], __shfl_xor_sync(0xffffffffu, mx[h2], 2));
      }
      float corr[2], mnew[2], psum[2] = {0.f, 0.f};
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        mnew[h2] = fmaxf(m_run[h2], mx[h2]);
        corr[h2] = (m_run[h2] == -INFINITY) ? 0.f : exp2f(m_run[h2] - mnew[h2]);
        m_run[h2] = mnew[h2];
      }
      uint32_t pf[KS / 16][4];
#pragma unroll
      for (int j = 0; j < KS / 8; ++j) {
        const float p0 = exp2f(s[j][0] - mnew[0]), p1 = exp2f(s[j][1] - mnew[0]);
        const float p2 = exp2f(s[j][2] - mnew[1]), p3 = exp2f(s[j][3] - mnew[1]);
        psum[0] += p0 + p1;
        psum[1] += p2 + p3;
        const int kk = j >> 1;
        if ((j & 1) == 0) {
          pf[kk][0] = pack_bf16(p0, p1);
          pf[kk][1] = pack_bf16(p2, p3);
        } else {
          pf[kk][2] = pack_bf16(p0, p1);
          pf[kk][3] = pack_bf16(p2, p3);
        }
      }
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        psum[h2] += __shfl_xor_sync(0xffffffffu, psum[h2], 1);
        psum[h2] += __shfl_xor_sync(0xffffffffu, psum[h2], 2);
        l_run[h2] = l_run[h2] * corr[h2] + psum[h2];
      }
#pragma unroll
      for (int i = 0; i < HD / 8; ++i) {
        o[i][0] *= corr[0];
        o[i][1] *= corr[0];
        o[i][2] *= corr[1];
        o[i][3] *= corr[1];
      }
      // O += P V: k = keys (KS / 16 steps), n = d (HD / 8 tiles)
#pragma unroll
      for (int kk = 0; kk < KS / 16; ++kk) {
#pragma unroll
        for (int i = 0; i < HD / 16; ++i) {
          const int key = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
          const int d = i * 16 + (lane >> 4) * 8;
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(kv_addr(Vt, key, d), b0, b1, b2, b3);
          mma_bf16(o[2 * i], pf[kk][0], pf[kk][1], pf[kk][2], pf[kk][3], b0, b1);
          mma_bf16(o[2 * i + 1], pf[kk][0], pf[kk][1], pf[kk][2], pf[kk][3], b2, b3);
        }
      }
    }
    __syncthreads();  // the buffer is refilled in the next iteration
  }

  if (a.splits == 1) {  // single split: normalise and store
    if (warp_active) {
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int q = qt * QT + warp * 16 + g + h2 * 8;
        if (q >= nq) continue;
        const int r = row0 + q / G, h = kvh * G + q % G;
        const float inv = 1.f / l_run[h2];
        bf16 *dst = a.out + ((size_t)r * a.H + h) * HD;
#pragma unroll
        for (int i = 0; i < HD / 8; ++i)
          *reinterpret_cast<__nv_bfloat162 *>(dst + i * 8 + t * 2) =
              __floats2bfloat162_rn(o[i][2 * h2] * inv, o[i][2 * h2 + 1] * inv);
      }
    }
    return true;
  }
  // partials of this split: plane = packed (row, head) pairs of all sequences
  const size_t plane = (size_t)a.seq_off[a.B] * a.H;
  if (warp_active) {
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const int q = qt * QT + warp * 16 + g + h2 * 8;
      if (q >= nq) continue;
      const int r = row0 + q / G, h = kvh * G + q % G;
      const size_t qidx = (size_t)r * a.H + h;
      float *dst = a.part_o + ((size_t)ks * plane + qidx) * HD;
#pragma unroll
      for (int i = 0; i < HD / 8; ++i)
        *reinterpret_cast<float2 *>(dst + i * 8 + t * 2) = make_float2(o[i][2 * h2], o[i][2 * h2 + 1]);
      if (t == 0) a.part_ml[(size_t)ks * plane + qidx] = make_float2(m_run[h2], l_run[h2]);
    }
  }
  return true;
}

// grid = B x Hkv x splits x qt_grid; the CTA walks query tiles qt, qt + qt_grid, ...
template <int HD>
__global__ void __launch_bounds__(256, 1) k_attn_mma(const __grid_constant__ AttnArgs a) {
  pdl_enter();
  extern __shared__ __align__(16) uint8_t sm_raw[];
  __shared__ __align__(8) uint64_t kv_full[NST];
  // Q tile (padded rows) at a 1024-byte aligned base, then the K / V ring
  uint8_t *sm = sm_raw + ((1024u - (smem_u32a(sm_raw) & 1023u)) & 1023u);
  const uint32_t ring = smem_u32a(sm) + attn_q_bytes(HD);
  const uint32_t bar0 = smem_u32a(kv_full);
  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar0 + 8u * i) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  uint32_t chunk_ctr = 0;
  int item = blockIdx.x;
  const int per_b = a.Hkv * a.splits * a.qt_grid;
  const int b = item / per_b;
  if (b >= a.B) return;
  item -= b * per_b;
  const int qt0 = item / (a.Hkv * a.splits);
  item -= qt0 * a.Hkv * a.splits;
  const int kvh = item / a.splits, ks = item - kvh * a.splits;
  const int row0 = a.seq_off[b], nq = (a.seq_off[b + 1] - row0) * (a.H / a.Hkv);
  if (ks * a.kc >= a.N) return;
  for (int qt = qt0; qt * QT < nq; qt += a.qt_grid) {
    if (!attn_tile<HD>(a, sm, ring, bar0, chunk_ctr, b, kvh, ks, qt, row0, nq)) return;
    __syncthreads();
  }
}

// out[q][d..d+3] = sum_s exp2(m_s - M) O_s / sum_s exp2(m_s - M) l_s over the
// key splits s, for every packed (row, head) pair q.
template <int HD>
__global__ void k_attn_merge(const float *__restrict__ part_o, const float2 *__restrict__ part_ml,
                             const int32_t *__restrict__ seq_off, int B, int H, int splits, bf16 *__restrict__ out) {
  pdl_enter();
  const size_t plane = (size_t)seq_off[B] * H;
  const long long items = (long long)plane * (HD / 4);
  for (long long it = blockIdx.x * (long long)blockDim.x + threadIdx.x; it < items;
       it += (long long)gridDim.x * blockDim.x) {
    const size_t q = (size_t)(it / (HD / 4));
    const int d4 = (int)(it - (long long)q * (HD / 4)) * 4;
    float2 ml[8];
    float4 ov[8];
#pragma unroll
    for (int sp = 0; sp < 8; ++sp) {
      if (sp < splits) {
        ml[sp] = __ldcg(part_ml + sp * plane + q);
        ov[sp] = __ldcg(reinterpret_cast<const float4 *>(part_o + (sp * plane + q) * HD + d4));
      }
    }
    float M = -INFINITY;
#pragma unroll
    for (int sp = 0; sp < 8; ++sp)
      if (sp < splits) M = fmaxf(M, ml[sp].x);
    float L = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int sp = 0; sp < 8; ++sp) {
      if (sp < splits && ml[sp].x != -INFINITY) {
        const float w = exp2f(ml[sp].x - M);
        L += ml[sp].y * w;
        acc[0] += ov[sp].x * w;
        acc[1] += ov[sp].y * w;
        acc[2] += ov[sp].z * w;
        acc[3] += ov[sp].w * w;
      }
    }
    const float inv = 1.f / L;
    bf16 *dst = out + q * HD + d4;
    *reinterpret_cast<__nv_bfloat162 *>(dst) = __floats2bfloat162_rn(acc[0] * inv, acc[1] * inv);
    *reinterpret_cast<__nv_bfloat162 *>(dst + 2) = __floats2bfloat162_rn(acc[2] * inv, acc[3] * inv);
  }
}

}  // namespace

// Q tile + NST stages of (K, V) x 64 keys + alignment slack.
size_t attn_mma_smem(int hd) { return (size_t)attn_q_bytes(hd) + (size_t)NST * 2u * (size_t)hd * 128u + 1024u; }

cudaError_t launch_attention_mma(const void *Q, const int32_t *seq_off, int B, int N, int H, int Hkv, int hd,
                                 const void *Kc, const void *Vc, const CUtensorMap *kmap, const CUtensorMap *vmap,
                                 void *out, float *part_o, float2 *part_ml, int splits, int qt_grid, int cap_rows,
                                 int32_t *status, cudaStream_t s) {
  if ((hd != 64 && hd != 128) || splits < 1 || splits > 8 || !kmap || !vmap) return cudaErrorInvalidValue;
  AttnArgs a;
  a.kmap = *kmap;
  a.vmap = *vmap;
  a.status = status;
  a.Q = (const bf16 *)Q;
  a.Kc = (const bf16 *)Kc;
  a.Vc = (const bf16 *)Vc;
  a.out = (bf16 *)out;
  a.seq_off = seq_off;
  a.part_o = part_o;
  a.part_ml = part_ml;
  a.B = B;
  a.N = N;
  a.H = H;
  a.Hkv = Hkv;
  a.splits = splits;
  a.kc = ((N + splits - 1) / splits + KS - 1) / KS * KS;
  a.qt_grid = qt_grid;
  a.scale_log2 = 1.4426950408889634f / sqrtf((float)hd);
  const size_t smem = attn_mma_smem(hd);
  const int grid = B * Hkv * splits * qt_grid;
  if (grid <= 0) return cudaSuccess;
  if (hd == 128) {
    static std::atomic<uint64_t> attr{0};
    if (cudaError_t e = ensure_smem_limit(k_attn_mma<128>, (int)smem, attr)) return e;
    launch_pdl(k_attn_mma<128>, grid, 256, smem, s, a);
  } else {
    static std::atomic<uint64_t> attr{0};
    if (cudaError_t e = ensure_smem_limit(k_attn_mma<64>, (int)smem, attr)) return e;
    launch_pdl(k_attn_mma<64>, grid, 256, smem, s, a);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || splits == 1) return e;
  return launch_attn_merge(part_o, part_ml, seq_off, B, H, hd, splits, cap_rows, out, s);
}

cudaError_t launch_attn_merge(const float *part_o, const float2 *part_ml, const int32_t *seq_off, int B, int H,
                              int hd, int splits, int cap_rows, void *out, cudaStream_t s) {
  if ((hd != 64 && hd != 128) || splits < 2 || splits > 8) return cudaErrorInvalidValue;
  const long long items = (long long)cap_rows * H * (hd / 4);
  long long mg = (items + 255) / 256;
  const int mgrid = (int)(mg < 148 * 8 ? mg : 148 * 8);
  if (hd == 128)
    launch_pdl(k_attn_merge<128>, mgrid, 256, 0, s, part_o, part_ml, seq_off, B, H, splits, (bf16 *)out);
  else
    launch_pdl(k_attn_merge<64>, mgrid, 256, 0, s, part_o, part_ml, seq_off, B, H, splits, (bf16 *)out);
  return cudaGetLastError();
}

}  // namespace dcu
