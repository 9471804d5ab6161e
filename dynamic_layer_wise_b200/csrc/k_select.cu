// Integer-deciding kernels of the DCU step and the commit:
//   * layer budget split (one thread per sequence, fp64),
//   * per-layer token selection: forced window + top-B radix select outside
//     it + index-ordered compaction, plus s = mean d (one CTA per sequence),
//   * row plans (which packed row is which sequence position),
//   * the commit rule: bitonic sort of confidences, fp64 prefix scan,
//     Fréchet / threshold / factor count, commit (one CTA per sequence).
#include "common.cuh"
#include "kernels.h"

namespace dcu {

static constexpr int kSelThreads = 1024;
static constexpr int kMaxSeq = 16384;
static constexpr int kSelRankMax = 256;  // candidates ranked directly (else radix select)

// ------------------------------------------------------------------ budget split
// [DLLM] "关键设计 1", the budget equation B^l = (B_layer * L) s^l / sum_k s^k,
// rounded by floor + largest remainder (ties -> lower layer) so that each row
// sums to B_layer * L; uniform when asked or when the row sums to 0.  If the
// floors overshoot (q rounded up to an integer), one is taken back from the
// layers with the smallest fractional parts (ties -> higher layer) above 0.
// One CTA per sequence, one thread per layer; the sum of s is taken in layer
// order by one thread so it matches a sequential fp64 sum bit for bit.
__global__ void k_budget_split(const float *__restrict__ s_prev, int L, int B_layer, int uniform_arg,
                               const int32_t *__restrict__ uniform_flag, int32_t *__restrict__ budgets) {
  pdl_enter();
  const int uniform = uniform_arg || (uniform_flag && *uniform_flag);
  extern __shared__ double sh[];  // [L] fractional parts, then [L] floors
  double *frac = sh, *flr = sh + L;
  __shared__ double s_total;
  __shared__ long long s_sumfl;
  const int b = blockIdx.x;
  const float *s = s_prev + (size_t)b * L;
  int32_t *out = budgets + (size_t)b * L;
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int l = 0; l < L; ++l) t = __dadd_rn(t, (double)s[l]);
    s_total = t;
  }
  __syncthreads();
  const double total = s_total;
  if (uniform || total == 0.0) {
    for (int l = threadIdx.x; l < L; l += blockDim.x) out[l] = B_layer;
    return;
  }
  const double T = (double)B_layer * (double)L;
  for (int l = threadIdx.x; l < L; l += blockDim.x) {
    const double q = __ddiv_rn(__dmul_rn(T, (double)s[l]), total);
    const double f = floor(q);
    flr[l] = f;
    frac[l] = q - f;  // exact (Sterbenz)
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    long long t = 0;
    for (int l = 0; l < L; ++l) t += (long long)flr[l];
    s_sumfl = t;
  }
  __syncthreads();
  const long long R = (long long)B_layer * L - s_sumfl;
  for (int l = threadIdx.x; l < L; l += blockDim.x) {
    const double frl = frac[l], fl = flr[l];
    int rank = 0;
    for (int k = 0; k < L; ++k) {
      const double frk = frac[k];
      if (R > 0) {
        if (frk > frl || (frk == frl && k < l)) ++rank;
      } else if (R < 0) {
        if (flr[k] > 0.0 && (frk < frl || (frk == frl && k > l))) ++rank;
      }
    }
    int v = (int)fl;
    if (R > 0 && rank < R) v += 1;
    if (R < 0 && fl > 0.0 && rank < -R) v -= 1;
    out[l] = v;
  }
}

cudaError_t launch_budget_split(const float *s_prev, int B, int L, int B_layer, int uniform,
                                const int32_t *uniform_flag, int32_t *budgets, cudaStream_t s) {
  if (B <= 0 || L <= 0) return cudaSuccess;
  const int threads = L < 256 ? ((L + 31) / 32) * 32 : 256;
  launch_pdl(k_budget_split, B, threads, (size_t)2 * L * sizeof(double), s, s_prev, L, B_layer, uniform, uniform_flag,
                                                                      budgets);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ selection
// One CTA per sequence.  s = mean(d) (fp64, fixed tree); W = union of the key
// windows ([DLLM] "关键设计 2"); k = min(budget, N - |W|); the k-th largest d
// outside W is found by a 4-pass MSB radix select on the float bits (d >= 0,
// so the bits order like the values); ties at the threshold go to the lower
// indices; U = W + selected, compacted in index order.
__global__ void __launch_bounds__(kSelThreads)
    k_select(const float *__restrict__ d, const int32_t *__restrict__ keys, const int32_t *__restrict__ nkeys,
             const int32_t *__restrict__ budgets, int budget_stride, int B, int N, int Bw, int mode, int force_lo,
             int force_hi, int32_t *__restrict__ idx, int32_t *__restrict__ count, float *__restrict__ s_out, int s_stride,
             float *__restrict__ d_next_zero, int32_t *__restrict__ rowmap, int32_t *__restrict__ m_total,
             int32_t *__restrict__ done, int32_t *__restrict__ seq_off, int32_t *__restrict__ status) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t *sd = reinterpret_cast<uint32_t *>(smem);     // [N] d bits
  uint8_t *flag = smem + (size_t)N * sizeof(uint32_t);   // [N] 0 none, 1 window, 2 top-B
  __shared__ int hist[256];
  __shared__ int red_i[32];
  __shared__ double red_d[32];
  __shared__ uint32_t cbits[kSelRankMax];
  __shared__ int cidx[kSelRankMax];
  __shared__ int s_bin, s_rem;
  __shared__ bool s_last;

  const int b = blockIdx.x;
  const int tid = threadIdx.x, nthr = blockDim.x;
  const float *db = d + (size_t)b * N;

  // Everything but d is written two or more launches earlier (key positions and
  // budgets before the step; the next layer's d is read only by later
  // launches), so the window is marked and d_next cleared before the wait for
  // the previous launch (the scatter that wrote this layer's d).
  const int nk_in = nkeys[b];
  const int k_in = budgets[(size_t)b * budget_stride];
  for (int i = tid; i < N; i += nthr) flag[i] = 0;
  if (d_next_zero)
    for (int i = tid; i < N; i += nthr) d_next_zero[(size_t)b * N + i] = 0.f;
  __syncthreads();
  // forced window
  int nk = nk_in;
  if (nk < 0 || nk > N) {
    if (tid == 0 && status) atomicOr(status, DCU_ST_BAD_KEY);
    nk = nk < 0 ? 0 : N;
  }
  if (Bw > 0 && nk > 0) {
    const int h = Bw / 2;
    const int width = (mode == 0) ? (2 * h + 1) : Bw;
    const long long total = (long long)nk * width;
    for (long long t = tid; t < total; t += nthr) {
      const int k = (int)(t / width), off = (int)(t - (long long)k * width);
      const int p = keys[(size_t)b * N + k];
      if (p < 0 || p >= N) {
        if (off == 0 && status) atomicOr(status, DCU_ST_BAD_KEY);
        continue;
      }
      const int i = p - h + off;
      if (i >= 0 && i < N) flag[i] = 1;
    }
  }
  // periodic refresh: the forced range joins the window (recomputed whatever the budget)
  for (int i = max(force_lo, 0) + tid; i < min(force_hi, N); i += nthr) flag[i] = 1;
  __syncthreads();
  int inW = 0;
  for (int i = tid; i < N; i += nthr) inW += (flag[i] == 1);
  inW = block_sum(inW, red_i);

  pdl_enter();  // this layer's d is final from here on
  for (int i = tid; i < N; i += nthr) sd[i] = __float_as_uint(db[i]);
  __syncthreads();
  int nz = 0;
  {
    double acc = 0.0;
    for (int i = tid; i < N; i += nthr) acc += (double)__uint_as_float(sd[i]);
    acc = block_sum(acc, red_d);
    if (tid == 0) s_out[(size_t)b * s_stride] = (float)(acc / (double)N);
    for (int i = tid; i < N; i += nthr) nz += (flag[i] == 0 && sd[i] != 0u);
    nz = block_sum(nz, red_i);
  }
  const int avail = N - inW;
  int k = k_in;
  k = k < 0 ? 0 : (k > avail ? avail : k);

  uint32_t thr = 0xffffffffu;  // select d > thr, plus `need` ties at thr
  int need = 0;
  bool take_all = (k == avail);
  if (k > 0 && !take_all && nz <= k) {  // every positive d fits: the threshold is 0
    thr = 0u;
    need = k - nz;
  } else if (k > 0 && !take_all && nz <= kSelRankMax) {
    // few candidates (typically the rows the previous layer recomputed): exact
    // ranks by (d desc, index asc) over the compacted candidate list
    const int chunk = (N + nthr - 1) / nthr;
    const int i0 = tid * chunk, i1 = min(N, i0 + chunk);
    int mine = 0;
    for (int i = i0; i < i1; ++i) mine += (flag[i] == 0 && sd[i] != 0u);
    int tot;
    int pos = block_exclusive_scan(mine, red_i, &tot);
    for (int i = i0; i < i1; ++i)
      if (flag[i] == 0 && sd[i] != 0u) {
        cidx[pos] = i;
        cbits[pos] = sd[i];
        ++pos;
      }
    __syncthreads();
    for (int c = tid; c < nz; c += nthr) {
      const uint32_t v = cbits[c];
      int rank = 0;
      for (int j = 0; j < nz; ++j) {
        const uint32_t w = cbits[j];
        rank += (w > v) || (w == v && j < c);
      }
      if (rank < k) flag[cidx[c]] = 2;
    }
    __syncthreads();  // thr / need keep their defaults: the marking below adds nothing
  } else if (k > 0 && !take_all) {
    uint32_t prefix = 0, mask = 0;
    int rem = k;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int t = tid; t < 256; t += nthr) hist[t] = 0;
      __syncthreads();
      // warp-aggregated: one shared atomic per distinct bin per warp (most d
      // share a few bins, e.g. the stuck-in-mud zeros)
      for (int base = 0; base < N; base += nthr) {
        const int i = base + tid;
        int bin = -1;
        if (i < N) {
          const uint32_t u = sd[i];
          if (flag[i] == 0 && (u & mask) == prefix) bin = (int)((u >> shift) & 255u);
        }
        const unsigned same = __match_any_sync(0xffffffffu, bin);
        if (bin >= 0 && (tid & 31) == __ffs(same) - 1) atomicAdd(&hist[bin], __popc(same));
      }
      __syncthreads();
      if (tid < 32) {
        // warp 0: lane j owns bins 255-8j .. 248-8j (descending); find the bin where
        // the count of candidates from the top reaches rem
        int cnt[8], tot = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          cnt[e] = hist[255 - 8 * tid - e];
          tot += cnt[e];
        }
        int incl = tot;  // inclusive prefix over lanes (higher bins first)
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (tid >= o) incl += y;
        }
        const int excl = incl - tot;
        const unsigned hit = __ballot_sync(0xffffffffu, excl < rem && incl >= rem);
        if (hit && tid == __ffs(hit) - 1) {
          int cum = excl, e = 0;
          for (; e < 8; ++e) {
            if (cum + cnt[e] >= rem) break;
            cum += cnt[e];
          }
          s_bin = 255 - 8 * tid - e;
          s_rem = rem - cum;
        }
      }
      __syncthreads();
      prefix |= (uint32_t)s_bin << shift;
      mask |= 255u << shift;
      rem = s_rem;
      __syncthreads();
    }
    thr = prefix;
    need = rem;
  }

  // mark the top-B: strictly above thr, then the first `need` ties in index order
  const int chunk = (N + nthr - 1) / nthr;
  const int i0 = tid * chunk, i1 = min(N, i0 + chunk);
  int nt = 0;
  if (k > 0) {
    for (int i = i0; i < i1; ++i) {
      if (flag[i] != 0) continue;
      if (take_all || sd[i] > thr) flag[i] = 2;
      else if (sd[i] == thr) ++nt;
    }
  }
  int tot;
  int before = block_exclusive_scan(nt, red_i, &tot);
  if (k > 0 && !take_all && need > 0) {
    for (int i = i0; i < i1; ++i) {
      if (flag[i] == 0 && sd[i] == thr) {
        if (before < need) flag[i] = 2;
        ++before;
      }
    }
  }
  __syncthreads();
  // compaction in index order
  int ns = 0;
  for (int i = i0; i < i1; ++i) ns += (flag[i] != 0);
  int pos = block_exclusive_scan(ns, red_i, &tot);
  int32_t *ib = idx + (size_t)b * N;
  if (rowmap != nullptr && B == 1) {
    // one sequence: its selection is the packed row plan (offset 0), no
    // cross-CTA step needed
    for (int i = i0; i < i1; ++i)
      if (flag[i] != 0) {
        ib[pos] = i;
        rowmap[pos] = i;
        ++pos;
      }
    if (tid == 0) {
      count[0] = tot;
      if (seq_off) {
        seq_off[0] = 0;
        seq_off[1] = tot;
      }
      *m_total = tot;
    }
    return;
  }
  for (int i = i0; i < i1; ++i)
    if (flag[i] != 0) ib[pos++] = i;
  if (tid == 0) count[b] = tot;

  // the last CTA to finish builds the packed row plan of all sequences
  if (rowmap == nullptr) return;
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(done, 1) == B - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  int off = 0;
  for (int bb = 0; bb < B; ++bb) {
    const int c = *((volatile int32_t *)count + bb);
    const volatile int32_t *src = idx + (size_t)bb * N;
    for (int j = tid; j < c; j += nthr) rowmap[off + j] = bb * N + src[j];
    if (tid == 0 && seq_off) seq_off[bb] = off;
    off += c;
  }
  if (tid == 0) {
    if (seq_off) seq_off[B] = off;
    *m_total = off;
    *done = 0;
  }
}

cudaError_t launch_select(const float *d, const int32_t *keys, const int32_t *nkeys, const int32_t *budgets,
                          int budget_stride, int B, int N, int Bw, int mode, int force_lo, int force_hi,
                          int32_t *idx, int32_t *count, float *s_out, int s_stride, float *d_next_zero,
                          int32_t *rowmap, int32_t *m_total, int32_t *done, int32_t *seq_off, int32_t *status,
                          cudaStream_t s) {
  if (N > kMaxSeq || B <= 0) return cudaErrorInvalidValue;
  size_t smem = (size_t)N * 5;
  static std::atomic<uint64_t> attr{0};
  if (cudaError_t e = ensure_smem_limit(k_select, kMaxSeq * 5, attr)) return e;
  // short sequences: fewer threads make the ~25 block barriers cheaper
  const int threads = N <= 2048 ? 256 : kSelThreads;
  launch_pdl(k_select, B, threads, smem, s, d, keys, nkeys, budgets, budget_stride, B, N, Bw, mode, force_lo, force_hi,
             idx, count, s_out, s_stride, d_next_zero, rowmap, m_total, done, seq_off, status);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ row plans
__global__ void k_plan_all(int B, int N, int32_t *rowmap, int32_t *m_total, int32_t *seq_off) {
  const int BN = B * N;
  for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < BN; r += gridDim.x * blockDim.x) rowmap[r] = r;
  if (blockIdx.x == 0 && threadIdx.x <= B) seq_off[threadIdx.x] = threadIdx.x * N;
  if (blockIdx.x == 0 && threadIdx.x == 0) *m_total = BN;
}

cudaError_t launch_plan_all(int B, int N, int32_t *rowmap, int32_t *m_total, int32_t *seq_off, cudaStream_t s) {
  const int BN = B * N;
  int grid = (BN + 255) / 256;
  if (grid > 1024) grid = 1024;
  k_plan_all<<<grid, 256, 0, s>>>(B, N, rowmap, m_total, seq_off);
  return cudaGetLastError();
}

// Masked positions of all sequences, in (b, i) order, as packed rows.
// Open block of the block-wise schedule ([README] "Quick Start": generate_mode
// "default"): generation positions from gen_start are cut into blocks of
// block_len and only the leftmost block that still holds a masked position is
// open.  first = that masked position (N when none is left); [b0, b1) out.
__device__ __forceinline__ void open_block(int first, int N, int gen_start, int block_len, int &b0, int &b1) {
  if (first >= N) {
    b0 = b1 = N;
    return;
  }
  b0 = gen_start + (first - gen_start) / block_len * block_len;
  b1 = min(N, b0 + block_len);
}

// Packed rows of the commit's candidates: every masked position, or with
// block_len > 0 the masked positions of each sequence's open block.
__global__ void __launch_bounds__(1024) k_plan_masked(const uint8_t *__restrict__ masked, int B, int N, int gen_start,
                                                      int block_len, int32_t *__restrict__ rowmap,
                                                      int32_t *__restrict__ m_total) {
  pdl_enter();
  __shared__ int red[32];
  __shared__ int first[256];  // B <= 255
  const int BN = B * N, nthr = blockDim.x, tid = threadIdx.x;
  if (block_len > 0) {
    for (int b = tid; b < B; b += nthr) first[b] = N;
    __syncthreads();
    for (int i = tid; i < BN; i += nthr) {
      const int b = i / N, j = i - b * N;
      if (j >= gen_start && masked[i]) atomicMin(&first[b], j);
    }
    __syncthreads();
  }
  auto open = [&](int i) -> bool {
    if (!masked[i]) return false;
    if (block_len <= 0) return true;
    const int b = i / N, j = i - b * N;
    int b0, b1;
    open_block(first[b], N, gen_start, block_len, b0, b1);
    return j >= b0 && j < b1;
  };
  const int chunk = (BN + nthr - 1) / nthr;
  const int i0 = tid * chunk, i1 = min(BN, i0 + chunk);
  int c = 0;
  for (int i = i0; i < i1; ++i) c += open(i);
  int tot;
  int pos = block_exclusive_scan(c, red, &tot);
  for (int i = i0; i < i1; ++i)
    if (open(i)) rowmap[pos++] = i;
  if (tid == 0) *m_total = tot;
}

cudaError_t launch_plan_masked(const uint8_t *masked, int B, int N, int gen_start, int block_len, int32_t *rowmap,
                               int32_t *m_total, cudaStream_t s) {
  if (B > 255) return cudaErrorInvalidValue;
  launch_pdl(k_plan_masked, 1, 1024, 0, s, masked, B, N, gen_start, block_len, rowmap, m_total);
  return cudaGetLastError();
}

// Stale rows of one layer (stale[r] != 0), in index order, as packed rows.
__global__ void __launch_bounds__(1024) k_plan_stale(const uint8_t *__restrict__ stale, int BN,
                                                     int32_t *__restrict__ rowmap, int32_t *__restrict__ m_total) {
  pdl_enter();
  __shared__ int red[32];
  const int nthr = blockDim.x, tid = threadIdx.x;
  const int chunk = (BN + nthr - 1) / nthr;
  const int i0 = tid * chunk, i1 = min(BN, i0 + chunk);
  int c = 0;
  for (int i = i0; i < i1; ++i) c += stale[i] != 0;
  int tot;
  int pos = block_exclusive_scan(c, red, &tot);
  for (int i = i0; i < i1; ++i)
    if (stale[i]) rowmap[pos++] = i;
  if (tid == 0) *m_total = tot;
}

cudaError_t launch_plan_stale(const uint8_t *stale, int BN, int32_t *rowmap, int32_t *m_total, cudaStream_t s) {
  launch_pdl(k_plan_stale, 1, 1024, 0, s, stale, BN, rowmap, m_total);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ commit rule
// [FRECHET] "整体框架": sort the masked positions by confidence (descending;
// ties -> lower position: key = c bits << 32 | ~position), then
//   Fréchet ("关键设计 1/2"): S_n = sum_{j<=n} c_(j) (fp64), L_n = max(0, S_n - (n-1)),
//     U_n = 1 - c_(n), n* = max{n : L_n - U_n > delta}, else 1;
//   threshold ("研究背景与动机"): n* = #{c >= tau}, else 1;
//   factor (same): n* = max{n : (n+1)(1 - c_(n)) < f}, else 1;
// commit the first n*: ids <- argmax, masked <- 0, out_positions, out_count.
__global__ void __launch_bounds__(1024)
    k_commit_rule(int rule, float param, const float *__restrict__ conf, const int32_t *__restrict__ amax,
                  uint8_t *__restrict__ masked, int32_t *__restrict__ ids, int N, int gen_start, int block_len,
                  int32_t *__restrict__ out_pos, int32_t *__restrict__ out_count, const float *__restrict__ tau) {
  pdl_enter();
  extern __shared__ uint64_t keys[];  // [P]
  __shared__ int red[32];
  __shared__ double redd[32];
  __shared__ int s_best, s_first;
  const int b = blockIdx.x, tid = threadIdx.x, nthr = blockDim.x;
  const uint8_t *mb = masked + (size_t)b * N;
  const float *cb = conf + (size_t)b * N;
  const int chunk = (N + nthr - 1) / nthr;
  const int i0 = tid * chunk, i1 = min(N, i0 + chunk);

  // candidates: the masked positions, or those of the open block
  int b0 = 0, b1 = N;
  if (block_len > 0) {
    if (tid == 0) s_first = N;
    __syncthreads();
    for (int i = max(i0, gen_start); i < i1; ++i)
      if (mb[i]) {
        atomicMin(&s_first, i);
        break;
      }
    __syncthreads();
    open_block(s_first, N, gen_start, block_len, b0, b1);
  }
  // compact the candidates (index order) into keys
  int c = 0;
  for (int i = i0; i < i1; ++i) c += (mb[i] != 0 && i >= b0 && i < b1);
  int m;
  int pos = block_exclusive_scan(c, red, &m);
  for (int i = i0; i < i1; ++i)
    if (mb[i] && i >= b0 && i < b1) keys[pos++] = ((uint64_t)__float_as_uint(cb[i]) << 32) | (uint64_t)(~(uint32_t)i);
  int P = 1;
  while (P < m) P <<= 1;
  for (int t = m + tid; t < P; t += nthr) keys[t] = 0ull;
  __syncthreads();
  // bitonic sort, descending
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = tid; t < P; t += nthr) {
        const int partner = t ^ stride;
        if (partner > t) {
          const bool desc = ((t & size) == 0);
          const uint64_t a = keys[t], bk = keys[partner];
          if (desc ? (a < bk) : (a > bk)) { keys[t] = bk; keys[partner] = a; }
        }
      }
      __syncthreads();
    }
  }
  // n*: each thread takes a contiguous run of sorted entries; fp64 prefix sums
  const int run = (m + nthr - 1) / nthr;
  const int j0 = tid * run, j1 = min(m, j0 + run);
  if (rule == DCU_APD) {
    // [DLLM] "关键设计 3": every candidate whose confidence reaches its own
    // threshold, in descending confidence; none -> the most confident one
    int cnt = 0;
    for (int j = j0; j < j1; ++j) {
      const int p = (int)(~(uint32_t)(keys[j] & 0xffffffffull));
      cnt += __uint_as_float((uint32_t)(keys[j] >> 32)) >= tau[(size_t)b * N + p];
    }
    int total;
    int k = block_exclusive_scan(cnt, red, &total);
    if (total > 0) {
      for (int j = j0; j < j1; ++j) {
        const int p = (int)(~(uint32_t)(keys[j] & 0xffffffffull));
        if (__uint_as_float((uint32_t)(keys[j] >> 32)) >= tau[(size_t)b * N + p]) {
          out_pos[(size_t)b * N + k++] = p;
          ids[(size_t)b * N + p] = amax[(size_t)b * N + p];
          masked[(size_t)b * N + p] = 0;
        }
      }
    } else if (tid == 0 && m > 0) {
      const int p = (int)(~(uint32_t)(keys[0] & 0xffffffffull));
      out_pos[(size_t)b * N] = p;
      ids[(size_t)b * N + p] = amax[(size_t)b * N + p];
      masked[(size_t)b * N + p] = 0;
    }
    if (tid == 0) out_count[b] = total > 0 ? total : (m > 0 ? 1 : 0);
    return;
  }
  double local = 0.0;
  for (int j = j0; j < j1; ++j) local += (double)__uint_as_float((uint32_t)(keys[j] >> 32));
  // exclusive scan of the per-thread fp64 sums (thread order)
  {
    const int lane = tid & 31, w = tid >> 5, nw = nthr >> 5;
    double x = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      double y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) redd[w] = x;
    __syncthreads();
    if (w == 0) {
      double t = (lane < nw) ? redd[lane] : 0.0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        double y = __shfl_up_sync(0xffffffffu, t, o);
        if (lane >= o) t += y;
      }
      redd[lane] = t;
    }
    __syncthreads();
    local = ((w > 0) ? redd[w - 1] : 0.0) + x - local;  // exclusive prefix of this thread's run
    __syncthreads();
  }
  if (tid == 0) s_best = 0;
  __syncthreads();
  int best = 0;
  const double prm = (double)param;
  double S = local;
  for (int j = j0; j < j1; ++j) {
    const int n = j + 1;
    const float cj = __uint_as_float((uint32_t)(keys[j] >> 32));
    const double c64 = (double)cj;
    S = __dadd_rn(S, c64);
    bool pass;
    if (rule == DCU_FRECHET) {
      double Ln = __dsub_rn(S, (double)(n - 1));
      Ln = Ln > 0.0 ? Ln : 0.0;
      const double Un = __dsub_rn(1.0, c64);
      pass = __dsub_rn(Ln, Un) > prm;
    } else if (rule == DCU_THRESHOLD) {
      pass = cj >= param;
    } else {
      pass = __dmul_rn((double)(n + 1), __dsub_rn(1.0, c64)) < prm;
    }
    if (pass && n > best) best = n;
  }
  if (rule == DCU_THRESHOLD) {
    int cnt = 0;
    for (int j = j0; j < j1; ++j) cnt += (__uint_as_float((uint32_t)(keys[j] >> 32)) >= param);
    cnt = block_sum(cnt, red);
    best = cnt;
    if (tid == 0) s_best = best;
  } else {
    atomicMax(&s_best, best);
  }
  __syncthreads();
  int nstar = s_best;
  if (m == 0) nstar = 0;
  else if (nstar == 0) nstar = 1;
  for (int j = tid; j < nstar; j += nthr) {
    const int p = (int)(~(uint32_t)(keys[j] & 0xffffffffull));
    out_pos[(size_t)b * N + j] = p;
    ids[(size_t)b * N + p] = amax[(size_t)b * N + p];
    masked[(size_t)b * N + p] = 0;
  }
  if (tid == 0) out_count[b] = nstar;
}

cudaError_t launch_commit_rule(int rule, float param, const float *conf, const int32_t *amax, uint8_t *masked,
                               int32_t *ids, int B, int N, int gen_start, int block_len, int32_t *out_pos,
                               int32_t *out_count, const float *tau, cudaStream_t s) {
  if (N > kMaxSeq || B <= 0) return cudaErrorInvalidValue;
  int P = 1;
  while (P < N) P <<= 1;
  static std::atomic<uint64_t> attr{0};
  if (cudaError_t e = ensure_smem_limit(k_commit_rule, kMaxSeq * (int)sizeof(uint64_t), attr)) return e;
  if (rule == DCU_APD && !tau) return cudaErrorInvalidValue;
  launch_pdl(k_commit_rule, B, 1024, (size_t)P * sizeof(uint64_t), s, rule, param, conf, amax, masked, ids, N,
             gen_start, block_len, out_pos, out_count, tau);
  return cudaGetLastError();
}

}  // namespace dcu
