// Host-side launchers of the libdcu kernels (internal).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "gemm_tc.h"

namespace dcu {

// Sets the text dcu_last_error(NULL) returns (calls that have no context).
void set_global_error(const char *msg);

// One weight matrix of a concatenated GEMM output: rows [row0, row0 + rows) of
// the output come from W ([rows][K], row-major).
struct GemmSeg {
  const void *W;
  int rows;
};

// ---- row kernels (k_rows.cu)
cudaError_t launch_rope_table(float2 *tab, int max_seq, int head_dim, float theta, cudaStream_t s);
// stale0 (may be null): set to 1 at rows whose H_0 content changed
cudaError_t launch_embed_refresh(int dtype, const int32_t *ids, int32_t *prev_ids, const void *embed, void *H0,
                                 float *d0, const float *g0, int BN, int D, int V, int full, int32_t *status,
                                 uint8_t *stale0, cudaStream_t s);
cudaError_t launch_cosine_distance(int dtype, const void *x, const void *y, const float *g, int64_t rows, int D,
                                   float *d, cudaStream_t s);
cudaError_t launch_gather_norm(int dtype, const int32_t *rowmap, const int32_t *m_total, int cap, const void *H,
                               const float *g, float eps, int D, void *xs, cudaStream_t s);
// C: GEMM output as slots [slot][cap][ldc] under the slot geometry `geo` (geo.grid == 0: one slot).
cudaError_t launch_epi_qkv(int dtype, const float *C, int ldc, const SlotGeo geo, const int32_t *rowmap,
                           const int32_t *m_total, int cap, int N, int H, int Hkv, int hd, const float2 *rope_tab,
                           int use_rope, void *Q, void *Kc, void *Vc, uint8_t *stale, cudaStream_t s);
cudaError_t launch_epi_o(int dtype, const float *C, int ldc, const SlotGeo geo, const int32_t *rowmap,
                         const int32_t *m_total, int cap, const void *Hl, const float *g2, float eps, int D,
                         float *hmid, void *xs, cudaStream_t s);
cudaError_t launch_epi_swiglu(int dtype, const float *C, int ldc, const SlotGeo geo, const int32_t *m_total,
                              int cap, int F, void *act, cudaStream_t s);
cudaError_t launch_epi_down_scatter(int dtype, const float *C, int ldc, const SlotGeo geo,
                                    const int32_t *rowmap, const int32_t *m_total, int cap, const float *hmid,
                                    void *Hnext, const float *g_next, float *d_next, uint8_t *stale_next, int D,
                                    cudaStream_t s);
// select_from = "v": Value distance of the packed stale rows against the layer's V cache
cudaError_t launch_value_dist(int dtype, const float *C, int ldc, const SlotGeo geo, const int32_t *rowmap,
                              const int32_t *m_total, int cap, int N, int Hkv, int hd, const void *Vc, float *d,
                              cudaStream_t s);
cudaError_t launch_softmax_max(const float *C, int ldc, const int32_t *rowmap, const int32_t *m_total, int cap,
                               int V, float *conf, int32_t *amax, cudaStream_t s);

// ---- selection, budgets and commit (k_select.cu)
// uniform split when `uniform` != 0 or *uniform_flag != 0 (uniform_flag may be null)
cudaError_t launch_budget_split(const float *s_prev, int B, int L, int B_layer, int uniform,
                                const int32_t *uniform_flag, int32_t *budgets, cudaStream_t s);
// budgets: pointer to element [0] of the layer's column; budget_stride = L.
// s_out: pointer to the layer's column of s [B][L]; s_stride = L.
// rowmap / m_total / done may be null (stateless use).  Positions [force_lo,
// force_hi) join the window (periodic refresh; an empty range forces nothing).
cudaError_t launch_select(const float *d, const int32_t *keys, const int32_t *nkeys, const int32_t *budgets,
                          int budget_stride, int B, int N, int Bw, int mode, int force_lo, int force_hi,
                          int32_t *idx, int32_t *count, float *s_out, int s_stride, float *d_next_zero,
                          int32_t *rowmap, int32_t *m_total, int32_t *done, int32_t *seq_off, int32_t *status,
                          cudaStream_t s);
// stale rows (stale[r] != 0 over B * N rows) as packed rows, one CTA
cudaError_t launch_plan_stale(const uint8_t *stale, int BN, int32_t *rowmap, int32_t *m_total, cudaStream_t s);
// rowmap = identity over B * N rows; seq_off[b] = b * N (B <= 255)
cudaError_t launch_plan_all(int B, int N, int32_t *rowmap, int32_t *m_total, int32_t *seq_off, cudaStream_t s);
cudaError_t launch_plan_masked(const uint8_t *masked, int B, int N, int gen_start, int block_len, int32_t *rowmap,
                               int32_t *m_total, cudaStream_t s);
// rule DCU_APD: commit every candidate with conf >= tau[b * N + i] (tau required), else the top one
cudaError_t launch_commit_rule(int rule, float param, const float *conf, const int32_t *amax, uint8_t *masked,
                               int32_t *ids, int B, int N, int gen_start, int block_len, int32_t *out_pos,
                               int32_t *out_count, const float *tau, cudaStream_t s);

// ---- GEMM (k_gemm_simt.cu): C[m][n] = sum_k X[m][k] * W[n][k], m < *m_total (m < m_cap when m_total is null)
cudaError_t launch_gemm_simt(int dtype, const void *X, int ldx, const int32_t *m_total, int m_cap,
                             const GemmSeg *segs, int nseg, int K, float *C, int ldc, cudaStream_t s);

// ---- tensor-core attention (k_attn_mma.cu), bf16, head_dim 64 or 128.  Rows of
// sequence b are packed rows [seq_off[b], seq_off[b + 1]).  With splits > 1 (<= 8)
// part_o / part_ml hold the key splits' partial results ([splits][rows * H][hd] /
// [splits][rows * H]) and a merge kernel follows (two launches); cap_rows bounds
// the packed rows.
size_t attn_mma_smem(int hd);
cudaError_t launch_attention_mma(const void *Q, const int32_t *seq_off, int B, int N, int H, int Hkv, int hd,
                                 const void *Kc, const void *Vc, const CUtensorMap *kmap, const CUtensorMap *vmap,
                                 void *out, float *part_o, float2 *part_ml, int splits, int qt_grid, int cap_rows,
                                 int32_t *status, cudaStream_t s);

// the split merge of both tensor-core attentions: out = sum_s w_s O_s / sum_s w_s l_s (2 <= splits <= 8)
cudaError_t launch_attn_merge(const float *part_o, const float2 *part_ml, const int32_t *seq_off, int B, int H,
                              int hd, int splits, int cap_rows, void *out, cudaStream_t s);

// ---- tcgen05 attention (k_attn_tc.cu), bf16, head_dim 64 or 128: same packing
// as above; K / V maps with a box of 64 x 128 keys; key splits (<= 8) of whole
// 128-key chunks, each split holding keys, merged inside the launch (the
// splits of a query tile form one cluster) -- one launch
size_t attn_tc_smem(int hd);
// clusters of `splits` CTAs of the kernel that can be resident at once (0: unknown)
int attn_tc_max_clusters(int hd, int splits);
cudaError_t launch_attention_tc(const void *Q, const int32_t *seq_off, int B, int N, int H, int Hkv, int hd,
                                const CUtensorMap *kmap, const CUtensorMap *vmap, void *out, int splits, int qt_grid,
                                int32_t *status, cudaStream_t s);

// ---- attention (k_attn.cu): out[r][h] = softmax(q K^T / sqrt(hd)) V over all N keys of row r's sequence
cudaError_t launch_attention(int dtype, const void *Q, const int32_t *rowmap, const int32_t *m_total, int cap,
                             int N, int H, int Hkv, int hd, const void *Kc, const void *Vc, void *out,
                             cudaStream_t s);

// ---- adaptive parallel decoding (k_apd.cu)
cudaError_t launch_apd_reset(float *tau, uint8_t *has_prev, int64_t n, float tau0, cudaStream_t s);
// signals and threshold update of the packed candidate rows (see k_apd.cu)
cudaError_t launch_apd_signals(const float *z_cur, int64_t ld_cur, int by_pos, float *z_copy, const float *z_prev,
                               const int32_t *rowmap, const int32_t *m_total, int cap, int V, uint8_t *has_prev,
                               float *tau, float alpha, float beta, float *out_c, float *out_h, cudaStream_t s);

// ---- self-test (k_selftest.cu): one bounded mbarrier wait that must expire
cudaError_t launch_wait_timeout_probe(int32_t *status, cudaStream_t s);

}  // namespace dcu
