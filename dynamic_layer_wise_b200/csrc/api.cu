// C ABI of libdcu: context (caches + scratch arena), host orchestration of
// the dense forward, the DCU step and the commit, stateless kernel entry
// points, introspection and per-kernel event timing.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "../../include/dcu.h"
#include "gemm_tc.h"
#include "kernels.h"

using namespace dcu;

namespace {

thread_local std::string g_last_error;

struct EventPair {
  cudaEvent_t a = nullptr, b = nullptr;
};

struct ProfClass {
  std::vector<EventPair> ev;
  int64_t used = 0;
  int64_t dropped = 0;
};

// A captured dcu_step or commit_select: instantiated graph, the kernels it
// launches and (when captured with profiling on) its event-record nodes.
struct GraphEntry {
  uint64_t key[12] = {};
  cudaGraphExec_t exec = nullptr;
  int64_t kernels = 0;
  std::vector<std::pair<int, EventPair>> ev;
  int64_t replays = 0;  // since the last profile reset
  uint64_t last_use = 0;
};
constexpr size_t kMaxGraphs = 16;

size_t esize(int dtype) { return dtype == DCU_BF16 ? 2 : 4; }

constexpr int kAttnMaxSplits = 8;
constexpr int kChainBars = 8;  // per layer: QKV launch 2, O + gate|up + down launch 6

}  // namespace

struct LayerMaps {
  CUtensorMap wq, wk, wv, wo, wg, wu, wd;
};

struct dcu_ctx {
  dcu_cfg cfg{};
  int device = 0;
  size_t esz = 2;
  // weights (caller-owned)
  const void *embed = nullptr, *lm_head = nullptr;
  const float *final_norm = nullptr;
  std::vector<const void *> wq, wk, wv, wo, wg, wu, wd;
  std::vector<const float *> g1, g2;
  // active shape
  int B = 0, N = 0;
  // periodic full refresh: schedule, DCU steps since the dense forward, and the
  // positions forced into every layer's recompute set by the step being enqueued
  int refresh_gen_start = 0, refresh_prompt = 0, refresh_gen = 0;
  int64_t step_count = 0;
  int force_lo = 0, force_hi = 0;
  // select_from: DCU_SELECT_INPUT (layer-input distance) or DCU_SELECT_VALUE;
  // stale[l][r] = H_l row r was rewritten since layer l last recomputed it
  int select_from = DCU_SELECT_INPUT;
  // adaptive parallel decoding: parameters, per-position thresholds, the
  // logits of the current and previous commit ([2][cap][vocab] fp32, flipped
  // every APD commit) and the last signals
  bool apd = false;
  float apd_alpha = 0.f, apd_beta = 0.f, apd_tau0 = 0.9f;
  float *apd_z = nullptr, *apd_tau = nullptr, *apd_c = nullptr, *apd_h = nullptr;
  uint8_t *apd_prev = nullptr;
  int apd_flip = 0;
  uint8_t *stale = nullptr;
  int32_t *vrowmap = nullptr;
  bool have_cache = false, first_step = true;
  int64_t cap = 0;  // max_batch * max_seq rows
  // caches
  char *H = nullptr, *K = nullptr, *V = nullptr;
  int32_t *prev_ids = nullptr;
  float *d = nullptr, *s_cur = nullptr, *s_prev = nullptr;
  int32_t *budgets = nullptr, *sel_idx = nullptr, *sel_cnt = nullptr;
  int32_t *rowmap = nullptr, *ints = nullptr;  // ints: m_total, done, status, m_masked
  float2 *rope_tab = nullptr;
  // scratch
  char *xs = nullptr, *Q = nullptr, *attn = nullptr, *act = nullptr;
  float *hmid = nullptr, *C = nullptr, *conf = nullptr;
  int32_t *seq_off = nullptr;
  float *attn_po = nullptr;
  float2 *attn_ml = nullptr;
  int attn_qt_cap = 1;
  int32_t *amax = nullptr, *mrow = nullptr;
  std::vector<void *> allocs;
  std::string err;
  // tcgen05 GEMM state (bf16 models)
  int num_sms = 148;
  int gemm_bn = 128;          // token tile of the current call
  int gemm_rows_hint = 128;   // expected rows per layer of the current call
  size_t ws_elems = 0;        // capacity of C in floats
  float2 *smx = nullptr;      // LM-head softmax statistics per (vocab tile, row)
  int32_t *smx_arg = nullptr;
  // chained GEMM launches with their epilogues (bf16, head_dim 64 / 128)
  int fused = 0;             // chained launches in use (DCU_OPT_FUSED_EPILOGUE and supported): 1 or 2
  bool fused_ok = false;     // the model supports them (bf16, head_dim 64 or 128)
  int nx_count = 16;         // units per CTA of the next GEMM's weights prefetched into L2 (0: off)
  size_t gemm_smem = kTcSmem;  // dynamic shared memory of a layer GEMM CTA (DCU_OPT_GEMM_SMEM_KB)
  int pass_sweep = 1;          // DCU_OPT_GEMM_PASS_SWEEP
  int32_t *chain_bar = nullptr;  // grid-barrier counters of the chained launches, kChainBars per layer
  std::vector<LayerMaps> lmaps;
  CUtensorMap lm_map;
  CUtensorMap xs_map[2], attn_map[2], act_map[2];  // boxes of min(128, cap) and min(256, cap) rows
  uint32_t act_box[2] = {128, 256};
  // per layer: K and V of the active shape as [B*Hkv*N rows][hd], box 64 x 64
  // (mma.sync attention) and box 64 x 128 (tcgen05 attention)
  std::vector<CUtensorMap> kv_maps, kv_maps_tc;
  int attn_impl = DCU_ATTN_TCGEN05;  // DCU_OPT_ATTENTION
  // per-tile piece counts of each stream-K geometry used so far (device tables)
  struct SlotTable {
    int n_tiles, kblocks, grid, tile_aligned;
    int32_t *dev;
  };
  std::vector<SlotTable> slot_tables;
  const int32_t *slot_table(const SlotGeo &g) {
    for (auto &t : slot_tables)
      if (t.n_tiles == g.n_tiles && t.kblocks == g.kblocks && t.grid == g.grid && t.tile_aligned == g.tile_aligned)
        return t.dev;
    if (capturing) return nullptr;  // no allocation inside a stream capture: geometries are registered at create
    std::vector<int32_t> h(g.n_tiles);
    for (int i = 0; i < g.n_tiles; ++i) h[i] = sk_nslots(g, i);
    int32_t *d = nullptr;
    if (cudaMalloc(&d, h.size() * 4) != cudaSuccess) return nullptr;
    if (cudaMemcpy(d, h.data(), h.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess) {
      cudaFree(d);
      return nullptr;
    }
    allocs.push_back(d);
    slot_tables.push_back({g.n_tiles, g.kblocks, g.grid, g.tile_aligned, d});
    return d;
  }
  // CUDA graphs of dcu_step / commit_select
  bool use_graphs = true;
  bool capturing = false;
  cudaStream_t cap_stream = nullptr;
  std::vector<GraphEntry> graphs;
  GraphEntry *cur_graph = nullptr;
  uint64_t use_clock = 0;
  // profiling
  int32_t prof_max = 0;
  int64_t launches = 0;
  ProfClass prof[DCU_K_COUNT];

  int32_t *m_total() { return ints + 0; }
  int32_t *done() { return ints + 1; }
  int32_t *status() { return ints + 2; }
  int32_t *m_masked() { return ints + 3; }
  int32_t *uniform_flag() { return ints + 4; }  // 1: the next step splits its budget uniformly
  int32_t *vm_total() { return ints + 5; }      // stale rows of the current layer (select_from = "v")
  uint8_t *stale_l(int l) { return stale + (size_t)l * cap; }
  size_t hslab() const { return (size_t)cap * cfg.d_model * esz; }
  size_t kvslab() const { return (size_t)cap * cfg.n_kv_heads * cfg.head_dim * esz; }
  void *Hl(int l) { return H + (size_t)l * hslab(); }
  void *Kl(int l) { return K + (size_t)l * kvslab(); }
  void *Vl(int l) { return V + (size_t)l * kvslab(); }
  float *dl(int l) { return d + (size_t)l * cap; }
};

namespace {

int fail(dcu_ctx *ctx, int code, const std::string &msg) {
  if (ctx) ctx->err = msg;
  g_last_error = msg;
  return code;
}

#define CK(ctx, expr)                                                                       \
  do {                                                                                      \
    cudaError_t e_ = (expr);                                                                \
    if (e_ != cudaSuccess)                                                                  \
      return fail((ctx), DCU_ECUDA, std::string(#expr) + ": " + cudaGetErrorString(e_)); \
  } while (0)

// A launch_* call enqueues exactly one kernel.
#define LAUNCH(ctx, expr)            \
  do {                               \
    CK(ctx, expr);                   \
    if (ctx) ++(ctx)->launches;      \
  } while (0)

struct Prof {
  dcu_ctx *c;
  int k;
  cudaStream_t s;
  EventPair *p = nullptr;
  bool ext = false;
  Prof(dcu_ctx *c_, int k_, cudaStream_t s_) : c(c_), k(k_), s(s_) {
    if (!c || c->prof_max <= 0) return;
    if (c->capturing && c->cur_graph) {  // event-record nodes inside the graph
      EventPair e;
      if (cudaEventCreate(&e.a) != cudaSuccess || cudaEventCreate(&e.b) != cudaSuccess) return;
      c->cur_graph->ev.push_back({k, e});
      p = &c->cur_graph->ev.back().second;
      ext = true;
      cudaEventRecordWithFlags(p->a, s, cudaEventRecordExternal);
      return;
    }
    ProfClass &pc = c->prof[k];
    if (pc.used >= (int64_t)pc.ev.size()) {
      ++pc.dropped;
      return;
    }
    p = &pc.ev[pc.used++];
    cudaEventRecord(p->a, s);
  }
  ~Prof() {
    if (p) {
      if (ext)
        cudaEventRecordWithFlags(p->b, s, cudaEventRecordExternal);
      else
        cudaEventRecord(p->b, s);
    }
  }
};

template <class T>
cudaError_t dalloc(dcu_ctx *c, T **p, size_t bytes) {
  void *q = nullptr;
  cudaError_t e = cudaMalloc(&q, bytes < 256 ? 256 : bytes);
  if (e != cudaSuccess) return e;
  c->allocs.push_back(q);
  *p = reinterpret_cast<T *>(q);
  return cudaSuccess;
}

void free_graph(GraphEntry &g) {
  if (g.exec) cudaGraphExecDestroy(g.exec);
  g.exec = nullptr;
  for (auto &e : g.ev) {
    if (e.second.a) cudaEventDestroy(e.second.a);
    if (e.second.b) cudaEventDestroy(e.second.b);
  }
  g.ev.clear();
}

void free_all(dcu_ctx *c) {
  for (auto &g : c->graphs) free_graph(g);
  c->graphs.clear();
  if (c->cap_stream) cudaStreamDestroy(c->cap_stream);
  c->cap_stream = nullptr;
  for (void *p : c->allocs) cudaFree(p);
  c->allocs.clear();
  for (auto &pc : c->prof)
    for (auto &e : pc.ev) {
      if (e.a) cudaEventDestroy(e.a);
      if (e.b) cudaEventDestroy(e.b);
    }
}

std::string check_cfg(const dcu_cfg *c) {
  if (c->n_layers <= 0 || c->d_model <= 0 || c->n_heads <= 0 || c->n_kv_heads <= 0 || c->head_dim <= 0 ||
      c->d_ffn <= 0 || c->vocab <= 0 || c->max_batch <= 0 || c->max_seq <= 0)
    return "every size must be > 0";
  if (c->dtype != DCU_F32 && c->dtype != DCU_BF16) return "dtype must be DCU_F32 or DCU_BF16";
  if (c->d_model % 64) return "d_model must be a multiple of 64";
  if (c->head_dim % 16 || c->head_dim > 256) return "head_dim must be a multiple of 16 and <= 256";
  if (c->n_heads % c->n_kv_heads) return "n_heads must be a multiple of n_kv_heads";
  if ((c->n_heads * c->head_dim) % 64 || (c->n_kv_heads * c->head_dim) % 64)
    return "n_heads*head_dim and n_kv_heads*head_dim must be multiples of 64";
  if (c->d_ffn % 64) return "d_ffn must be a multiple of 64";
  if (c->dtype == DCU_BF16 && (c->d_model % 128 || c->d_ffn % 128 || (c->n_heads * c->head_dim) % 128 ||
                               (c->n_kv_heads * c->head_dim) % 128))
    return "bf16 models need d_model, d_ffn, n_heads*head_dim and n_kv_heads*head_dim to be multiples of 128";
  if (c->max_seq > 16384) return "max_seq must be <= 16384";
  if (c->n_layers > 1024) return "n_layers must be <= 1024";
  if (c->max_batch > 255) return "max_batch must be <= 255";
  if (c->mask_id < 0 || c->mask_id >= c->vocab) return "mask_id must be in [0, vocab)";
  if (!(c->rms_eps > 0.0f)) return "rms_eps must be > 0";
  if (c->rope_theta < 0.0f) return "rope_theta must be >= 0";
  if (c->window_mode != DCU_WINDOW_INCLUSIVE && c->window_mode != DCU_WINDOW_HALFOPEN)
    return "window_mode must be DCU_WINDOW_INCLUSIVE or DCU_WINDOW_HALFOPEN";
  if ((long long)c->max_batch * c->max_seq > (1ll << 30)) return "max_batch * max_seq too large";
  return "";
}

// Activation operand of a GEMM: the packed rows X [cap][K] (row pitch ldx)
// and, for the tcgen05 path, its tensor map (16-row boxes).
struct ActOperand {
  const void *X;
  int ldx, K;
  const CUtensorMap *map128, *map256;  // activation boxes for 128- and 256-token passes
};

// One tcgen05 GEMM phase: C[m][n] = sum_k X[m][k] W[n][k] over the
// concatenated weight segments (stream-K over all SMs unless tile_aligned).
int gemm_phase(dcu_ctx *c, const ActOperand &x, const GemmSeg *segs, const CUtensorMap *const *amaps, int nseg,
               int ldc, bool tile_aligned, TcPhase *ph) {
  const int cap = (int)c->cap;
  memset(ph, 0, sizeof(*ph));
  int tile = 0, col = 0;
  for (int i = 0; i < nseg; ++i) {
    ph->a[i] = *amaps[i];
    ph->seg_tile0[i] = tile;
    ph->seg_col0[i] = col;
    ph->seg_rows[i] = segs[i].rows;
    tile += (segs[i].rows + 127) / 128;
    col += segs[i].rows;
  }
  ph->seg_tile0[nseg] = tile;
  ph->nseg = nseg;
  ph->b = c->gemm_bn == 128 ? *x.map128 : *x.map256;
  ph->ldc = ldc;
  SlotGeo g;
  g.n_tiles = tile;
  g.kblocks = x.K / 64;
  g.tile_aligned = tile_aligned ? 1 : 0;
  const long long T = (long long)tile * g.kblocks;
  g.grid = tile_aligned ? (tile < c->num_sms ? tile : c->num_sms) : (int)(T < c->num_sms ? T : c->num_sms);
  g.slot_stride = (long long)cap * ldc;
  if ((size_t)tc_max_slots(tile, g.grid) * cap * ldc > c->ws_elems)
    return fail(c, DCU_ECUDA, "GEMM workspace too small for the stream-K slots");
  g.nslots = c->slot_table(g);
  if (!g.nslots) return fail(c, DCU_ECUDA, "stream-K piece table unavailable for this GEMM geometry");
  ph->geo = g;
  return DCU_OK;
}

// Launch-wide fields of the tcgen05 GEMM (one phase until more are added).
void gemm_common(dcu_ctx *c, const int32_t *m_total, TcParams *tp) {
  memset(tp, 0, sizeof(*tp));
  tp->nphase = 1;
  tp->b_rows = (int)c->act_box[c->gemm_bn == 128 ? 0 : 1];
  tp->m_total = m_total;
  tp->out = c->C;
  tp->status = c->status();
  tp->smem_bytes = (uint32_t)c->gemm_smem;  // layer GEMMs (the LM head keeps the default)
  // pass sweep with the 256-row pass (recompute sets expected past 192 rows):
  // its activation stages take shared memory from the weight ring, which the
  // 128-row pass of the small sets keeps whole
  tp->sweep = (c->pass_sweep && c->gemm_bn == 256) ? 2 : 0;
}

// C[m][n] = sum_k X[m][k] W[n][k] over the concatenated segments: ctx->C as
// stream-K slots described by *geo (geo->grid == 0: a single slot).
// L2 prefetch target of a GEMM launch: the first units of the next weight
// stream, GEMM `which` (0 QKV, 1 O, 2 gate|up, 3 down) of layer l, or the LM
// head when l == n_layers (bf16 models; nothing otherwise).
void set_prefetch(dcu_ctx *c, int l, int which, TcParams *tp) {
  const dcu_cfg &g = c->cfg;
  if (c->lmaps.empty() || c->nx_count <= 0 || l > g.n_layers) return;
  const int D = g.d_model, F = g.d_ffn, Hhd = g.n_heads * g.head_dim, KVd = g.n_kv_heads * g.head_dim;
  SlotGeo &q = tp->nx_geo;
  memset(&q, 0, sizeof(q));
  if (l == g.n_layers) {  // LM head: tile-aligned ranges over the vocabulary
    tp->nx_a[0] = c->lm_map;
    q.n_tiles = (g.vocab + 127) / 128;
    q.kblocks = D / 64;
    q.tile_aligned = 1;
    q.grid = q.n_tiles < c->num_sms ? q.n_tiles : c->num_sms;
    tp->nx_seg_tile0[0] = 0;
    tp->nx_seg_tile0[1] = q.n_tiles;
    tp->nx_nseg = 1;
  } else {
    const LayerMaps &m = c->lmaps[l];
    int rows[3] = {0, 0, 0}, n = 0, K = D;
    if (which == 0) {
      tp->nx_a[0] = m.wq, tp->nx_a[1] = m.wk, tp->nx_a[2] = m.wv;
      rows[0] = Hhd, rows[1] = KVd, rows[2] = KVd, n = 3;
    } else if (which == 1) {
      tp->nx_a[0] = m.wo, rows[0] = D, n = 1, K = Hhd;
    } else if (which == 2) {
      tp->nx_a[0] = m.wg, tp->nx_a[1] = m.wu, rows[0] = rows[1] = F, n = 2;
    } else {
      tp->nx_a[0] = m.wd, rows[0] = D, n = 1, K = F;
    }
    int tile = 0;
    for (int i = 0; i < n; ++i) {
      tp->nx_seg_tile0[i] = tile;
      tile += (rows[i] + 127) / 128;
    }
    tp->nx_seg_tile0[n] = tile;
    tp->nx_nseg = n;
    q.n_tiles = tile;
    q.kblocks = K / 64;
    const long long T = (long long)tile * q.kblocks;
    q.grid = (int)(T < c->num_sms ? T : c->num_sms);
  }
  tp->nx_count = c->nx_count;
}

int run_gemm(dcu_ctx *c, const ActOperand &x, const int32_t *m_total, const GemmSeg *segs,
             const CUtensorMap *const *amaps, int nseg, int ldc, cudaStream_t s, SlotGeo *geo,
             bool tile_aligned = false, int prof_class = DCU_K_GEMM, int next_l = -1, int next_which = 0) {
  Prof p(c, prof_class, s);
  const int cap = (int)c->cap;
  memset(geo, 0, sizeof(*geo));
  if (c->cfg.dtype != DCU_BF16) {
    LAUNCH(c, launch_gemm_simt(c->cfg.dtype, x.X, x.ldx, m_total, cap, segs, nseg, x.K, c->C, ldc, s));
    return DCU_OK;
  }
  TcParams tp;
  gemm_common(c, m_total, &tp);
  if (int rc = gemm_phase(c, x, segs, amaps, nseg, ldc, tile_aligned, &tp.ph[0])) return rc;
  if (next_l >= 0) set_prefetch(c, next_l, next_which, &tp);
  *geo = tp.ph[0].geo;
  LAUNCH(c, launch_gemm_tc(tp, c->gemm_bn, s));
  return DCU_OK;
}


// One layer of recompute over the packed rows in ctx->rowmap / m_total.
// dense: the rows are every position (full forward): no selection, no d.
int run_layer(dcu_ctx *c, int l, bool dense, const int32_t *keys, const int32_t *nkeys, int Bw, cudaStream_t s) {
  const dcu_cfg &g = c->cfg;
  const int L = g.n_layers, D = g.d_model, H = g.n_heads, Hkv = g.n_kv_heads, hd = g.head_dim, F = g.d_ffn;
  const int dt = g.dtype, cap = (int)c->cap;
  const bool last = (l + 1 == L);
  // grid size of the row kernels: the expected recompute-set size (their loops
  // stride over the device row count, so any count is covered)
  const int gcap = dense ? cap : std::min(cap, std::max(1, c->gemm_rows_hint));
  if (!dense && c->select_from == DCU_SELECT_VALUE) {
    // select_from = "v": d of the stale rows from their recomputed Value
    // against the cached Value (every other row keeps d = 0)
    Prof p(c, DCU_K_SELECT, s);
    const int Wv = Hkv * hd;
    LAUNCH(c, launch_plan_stale(c->stale_l(l), c->B * c->N, c->vrowmap, c->vm_total(), s));
    LAUNCH(c, launch_gather_norm(dt, c->vrowmap, c->vm_total(), gcap, c->Hl(l), c->g1[l], g.rms_eps, D, c->xs, s));
    const LayerMaps *lmv = c->lmaps.empty() ? nullptr : &c->lmaps[l];
    const ActOperand xv{c->xs, D, D, &c->xs_map[0], &c->xs_map[1]};
    GemmSeg seg[1] = {{c->wv[l], Wv}};
    const CUtensorMap *am[1] = {lmv ? &lmv->wv : nullptr};
    SlotGeo vgeo;
    if (int rc = run_gemm(c, xv, c->vm_total(), seg, am, 1, Wv, s, &vgeo, false, DCU_K_SELECT)) return rc;
    LAUNCH(c, launch_value_dist(dt, c->C, Wv, vgeo, c->vrowmap, c->vm_total(), gcap, c->N, Hkv, hd, c->Vl(l),
                                c->dl(l), s));
  }
  if (!dense) {
    Prof p(c, DCU_K_SELECT, s);
    LAUNCH(c, launch_select(c->dl(l), keys, nkeys, c->budgets + l, L, c->B, c->N, Bw, g.window_mode,
                            c->force_lo, c->force_hi, c->sel_idx + (size_t)l * cap, c->sel_cnt + (size_t)l * g.max_batch, c->s_cur + l, L,
                            last ? nullptr : c->dl(l + 1), c->rowmap, c->m_total(), c->done(), c->seq_off,
                            c->status(), s));
  }
  {
    Prof p(c, DCU_K_GATHER, s);
    LAUNCH(c, launch_gather_norm(dt, c->rowmap, c->m_total(), gcap, c->Hl(l), c->g1[l], g.rms_eps, D, c->xs, s));
  }
  const LayerMaps *lm = c->lmaps.empty() ? nullptr : &c->lmaps[l];
  const ActOperand xs{c->xs, D, D, &c->xs_map[0], &c->xs_map[1]};
  const ActOperand at{c->attn, H * hd, H * hd, &c->attn_map[0], &c->attn_map[1]};
  const ActOperand ac{c->act, F, F, &c->act_map[0], &c->act_map[1]};
  SlotGeo geo;
  const int nqkv = (H + 2 * Hkv) * hd;
  // chained launches (DCU_OPT_FUSED_EPILOGUE): QKV with its epilogue, then O,
  // gate|up and down with theirs, each a persistent cooperative launch
  const bool chained = c->fused;
  EpiArgs ea;
  memset(&ea, 0, sizeof(ea));
  if (chained) {
    ea.rowmap = c->rowmap;
    ea.N = c->N;
    ea.H = H;
    ea.Hkv = Hkv;
    ea.hd = hd;
    ea.use_rope = g.rope_theta > 0.0f;
    ea.rope_tab = c->rope_tab;
    ea.Q = c->Q;
    ea.Kc = c->Kl(l);
    ea.Vc = c->Vl(l);
    ea.stale_l = c->stale_l(l);
    ea.D = D;
    ea.F = F;
    ea.eps = g.rms_eps;
    ea.Hl = c->Hl(l);
    ea.g2 = c->g2[l];
    ea.hmid = c->hmid;
    ea.xs = c->xs;
    ea.act = c->act;
    ea.Hn = c->Hl(l + 1);
    const bool want_d = !dense && !last;
    ea.g_next = want_d ? c->g1[l + 1] : nullptr;
    ea.d_next = want_d ? c->dl(l + 1) : nullptr;
    ea.stale_next = want_d ? c->stale_l(l + 1) : nullptr;
  }
  {
    GemmSeg seg[3] = {{c->wq[l], H * hd}, {c->wk[l], Hkv * hd}, {c->wv[l], Hkv * hd}};
    const CUtensorMap *am[3] = {lm ? &lm->wq : nullptr, lm ? &lm->wk : nullptr, lm ? &lm->wv : nullptr};
    if (chained) {
      Prof p(c, DCU_K_GEMM, s);
      TcParams tp;
      gemm_common(c, c->m_total(), &tp);
      if (int rc = gemm_phase(c, xs, seg, am, 3, nqkv, false, &tp.ph[0])) return rc;
      tp.ph[0].epi = EPI_QKV;
      tp.chain = c->fused;
      tp.bar = c->chain_bar + (size_t)l * kChainBars;
      tp.e = ea;
      set_prefetch(c, l, 1, &tp);
      LAUNCH(c, launch_gemm_tc(tp, c->gemm_bn, s));
    } else {
      if (int rc = run_gemm(c, xs, c->m_total(), seg, am, 3, nqkv, s, &geo, false, DCU_K_GEMM, l, 1)) return rc;
      Prof p(c, DCU_K_EPILOGUE, s);
      LAUNCH(c, launch_epi_qkv(dt, c->C, nqkv, geo, c->rowmap, c->m_total(), gcap, c->N, H, Hkv, hd, c->rope_tab,
                               g.rope_theta > 0.0f, c->Q, c->Kl(l), c->Vl(l), c->stale_l(l), s));
    }
  }
  {
    Prof p(c, DCU_K_ATTN, s);
    if (c->attn_po) {
      const int G = H / Hkv;
      // query tiles per (sequence, kv head) sized for the typical recompute set
      // (half the GEMM's rows hint: B_layer + B_window + 1 per sequence); a
      // larger set makes each CTA walk more than one query tile
      const int rows_seq = dense ? c->N : (c->gemm_rows_hint / 2 + c->B - 1) / c->B;
      int qt_grid = (rows_seq * G + 127) / 128;
      qt_grid = qt_grid < 1 ? 1 : (qt_grid > c->attn_qt_cap ? c->attn_qt_cap : qt_grid);
      // one wave: (sequence, kv head, query tile) items x key splits <= SM count (one CTA per SM)
      const long long items = (long long)c->B * Hkv * qt_grid;
      int splits = (int)(c->num_sms / items);
      if (c->attn_impl == DCU_ATTN_TCGEN05) {
        // tensor cores to spare: one wave of CTAs, each streaming whole 128-key
        // chunks; the splits of a query tile form a cluster, so the split count
        // is also capped by how many such clusters can be resident at once
        const int max_tc = (c->N + 127) / 128;
        splits = splits < 1 ? 1 : (splits > kAttnMaxSplits ? kAttnMaxSplits : splits);
        if (splits > max_tc) splits = max_tc;
        while (splits > 1 && (long long)attn_tc_max_clusters(hd, splits) < items) --splits;
        const int kc = ((c->N + splits - 1) / splits + 127) / 128 * 128;
        splits = (c->N + kc - 1) / kc;
        LAUNCH(c, launch_attention_tc(c->Q, c->seq_off, c->B, c->N, H, Hkv, hd, &c->kv_maps_tc[2 * l],
                                      &c->kv_maps_tc[2 * l + 1], c->attn, splits, qt_grid, c->status(), s));
      } else {
        const int max_sp = (c->N + 63) / 64;
        splits = splits < 1 ? 1 : splits;
        // long sequences: the legacy-MMA attention is compute-bound, so when one
        // wave leaves more than 2048 keys per CTA, cut them to <= 1024 even past
        // one wave (the heavy query tiles then spread over all SMs instead of the
        // few that hold them; measured +12 % attention at N = 8192, while at
        // N = 2048 x 4 sequences the extra wave and merge cost 10 %)
        if ((c->N + splits - 1) / splits > 2048)
          while (splits < kAttnMaxSplits && (c->N + splits - 1) / splits > 1024) splits *= 2;
        splits = splits > kAttnMaxSplits ? kAttnMaxSplits : splits;
        if (splits > max_sp) splits = max_sp;
        const int kc = ((c->N + splits - 1) / splits + 63) / 64 * 64;
        splits = (c->N + kc - 1) / kc;
        LAUNCH(c, launch_attention_mma(c->Q, c->seq_off, c->B, c->N, H, Hkv, hd, c->Kl(l), c->Vl(l),
                                       &c->kv_maps[2 * l], &c->kv_maps[2 * l + 1], c->attn, c->attn_po, c->attn_ml,
                                       splits, qt_grid, gcap, c->status(), s));
        if (splits > 1) ++c->launches;  // the merge kernel
      }
    } else {
      LAUNCH(c, launch_attention(dt, c->Q, c->rowmap, c->m_total(), gcap, c->N, H, Hkv, hd, c->Kl(l), c->Vl(l),
                                 c->attn, s));
    }
  }
  GemmSeg seg_o[1] = {{c->wo[l], D}}, seg_gu[2] = {{c->wg[l], F}, {c->wu[l], F}}, seg_d[1] = {{c->wd[l], D}};
  const CUtensorMap *am_o[1] = {lm ? &lm->wo : nullptr}, *am_gu[2] = {lm ? &lm->wg : nullptr, lm ? &lm->wu : nullptr},
                    *am_d[1] = {lm ? &lm->wd : nullptr};
  if (chained) {
    Prof p(c, DCU_K_GEMM, s);
    TcParams tp;
    gemm_common(c, c->m_total(), &tp);
    if (int rc = gemm_phase(c, at, seg_o, am_o, 1, D, false, &tp.ph[0])) return rc;
    if (int rc = gemm_phase(c, xs, seg_gu, am_gu, 2, 2 * F, false, &tp.ph[1])) return rc;
    if (int rc = gemm_phase(c, ac, seg_d, am_d, 1, D, false, &tp.ph[2])) return rc;
    tp.ph[0].epi = EPI_O;
    tp.ph[1].epi = EPI_GU;
    tp.ph[2].epi = EPI_DOWN;
    tp.nphase = 3;
    tp.chain = c->fused;
    tp.bar = c->chain_bar + (size_t)l * kChainBars + 2;
    tp.e = ea;
    set_prefetch(c, l + 1, 0, &tp);
    LAUNCH(c, launch_gemm_tc(tp, c->gemm_bn, s));
    return DCU_OK;
  }
  if (int rc = run_gemm(c, at, c->m_total(), seg_o, am_o, 1, D, s, &geo, false, DCU_K_GEMM, l, 2)) return rc;
  {
    Prof p(c, DCU_K_EPILOGUE, s);
    LAUNCH(c, launch_epi_o(dt, c->C, D, geo, c->rowmap, c->m_total(), gcap, c->Hl(l), c->g2[l],
                           g.rms_eps, D, c->hmid, c->xs, s));
  }
  if (int rc = run_gemm(c, xs, c->m_total(), seg_gu, am_gu, 2, 2 * F, s, &geo, false, DCU_K_GEMM, l, 3)) return rc;
  {
    Prof p(c, DCU_K_EPILOGUE, s);
    LAUNCH(c, launch_epi_swiglu(dt, c->C, 2 * F, geo, c->m_total(), gcap, F, c->act, s));
  }
  if (int rc = run_gemm(c, ac, c->m_total(), seg_d, am_d, 1, D, s, &geo, false, DCU_K_GEMM, l + 1, 0)) return rc;
  {
    Prof p(c, DCU_K_SCATTER, s);
    const bool want_d = !dense && !last;
    LAUNCH(c, launch_epi_down_scatter(dt, c->C, D, geo, c->rowmap, c->m_total(), gcap, c->hmid,
                                      c->Hl(l + 1), want_d ? c->g1[l + 1] : nullptr,
                                      want_d ? c->dl(l + 1) : nullptr, want_d ? c->stale_l(l + 1) : nullptr, D,
                                      s));
  }
  return DCU_OK;
}

}  // namespace

namespace dcu {
void set_global_error(const char *msg) { g_last_error = msg; }
}  // namespace dcu

extern "C" {

const char *dcu_last_error(const dcu_ctx *ctx) { return ctx ? ctx->err.c_str() : g_last_error.c_str(); }

int dcu_create(const dcu_weights *w, const dcu_cfg *cfg, dcu_ctx **out) {
  if (!out) return fail(nullptr, DCU_EINVAL, "out is NULL");
  *out = nullptr;
  if (!w || !cfg) return fail(nullptr, DCU_EINVAL, "weights or cfg is NULL");
  std::string why = check_cfg(cfg);
  if (!why.empty()) return fail(nullptr, DCU_EINVAL, "bad cfg: " + why);
  if (!w->embed || !w->final_norm || !w->lm_head || !w->attn_norm || !w->wq || !w->wk || !w->wv || !w->wo ||
      !w->ffn_norm || !w->w_gate || !w->w_up || !w->w_down)
    return fail(nullptr, DCU_EINVAL, "a weight pointer is NULL");
  for (int l = 0; l < cfg->n_layers; ++l)
    if (!w->attn_norm[l] || !w->wq[l] || !w->wk[l] || !w->wv[l] || !w->wo[l] || !w->ffn_norm[l] ||
        !w->w_gate[l] || !w->w_up[l] || !w->w_down[l])
      return fail(nullptr, DCU_EINVAL, "layer " + std::to_string(l) + ": a weight pointer is NULL");

  {
    auto mis = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; };
    bool bad = mis(w->embed) || mis(w->lm_head) || mis(w->final_norm);
    for (int l = 0; l < cfg->n_layers && !bad; ++l)
      bad = mis(w->wq[l]) || mis(w->wk[l]) || mis(w->wv[l]) || mis(w->wo[l]) || mis(w->w_gate[l]) ||
            mis(w->w_up[l]) || mis(w->w_down[l]) || mis(w->attn_norm[l]) || mis(w->ffn_norm[l]);
    if (bad) return fail(nullptr, DCU_EINVAL, "weight pointers must be 16-byte aligned");
  }
  dcu_ctx *c = new (std::nothrow) dcu_ctx();
  if (!c) return fail(nullptr, DCU_ENOMEM, "host allocation failed");
  c->cfg = *cfg;
  c->esz = esize(cfg->dtype);
  cudaGetDevice(&c->device);
  c->embed = w->embed;
  c->lm_head = w->lm_head;
  c->final_norm = (const float *)w->final_norm;
  const int L = cfg->n_layers;
  for (int l = 0; l < L; ++l) {
    c->wq.push_back(w->wq[l]);
    c->wk.push_back(w->wk[l]);
    c->wv.push_back(w->wv[l]);
    c->wo.push_back(w->wo[l]);
    c->wg.push_back(w->w_gate[l]);
    c->wu.push_back(w->w_up[l]);
    c->wd.push_back(w->w_down[l]);
    c->g1.push_back((const float *)w->attn_norm[l]);
    c->g2.push_back((const float *)w->ffn_norm[l]);
  }
  c->cap = (int64_t)cfg->max_batch * cfg->max_seq;
  const size_t cap = (size_t)c->cap, D = cfg->d_model, F = cfg->d_ffn, Hhd = (size_t)cfg->n_heads * cfg->head_dim;
  const size_t nqkv = (size_t)(cfg->n_heads + 2 * cfg->n_kv_heads) * cfg->head_dim;
  {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, c->device) == cudaSuccess && sms > 0)
      c->num_sms = sms;
  }
  // C holds a GEMM output as its stream-K slots (bf16) or one result (float32)
  size_t cw = cfg->dtype == DCU_BF16 ? 0 : (size_t)cfg->vocab;  // bf16: the LM head stores no logits
  if (nqkv > cw) cw = nqkv;
  if (2 * F > cw) cw = 2 * F;
  if (D > cw) cw = D;
  if (cfg->dtype == DCU_BF16) {
    const size_t widths[5] = {nqkv, D, 2 * F, D, (size_t)cfg->n_kv_heads * cfg->head_dim};
    const size_t ks[5] = {D, Hhd, D, F, D};
    for (int i = 0; i < 5; ++i) {
      const size_t tiles = (widths[i] + 127) / 128;
      const long long T = (long long)tiles * (long long)(ks[i] / 64);
      const int grid = (int)(T < c->num_sms ? T : c->num_sms);
      const size_t w = (size_t)tc_max_slots((int)tiles, grid) * widths[i];
      if (w > cw) cw = w;
    }
  }
  c->ws_elems = cap * cw;
  size_t xw = D > F ? D : F;
  cudaError_t e = cudaSuccess;
#define AL(ptr, bytes)                                                                  \
  if (e == cudaSuccess) {                                                               \
    e = dalloc(c, &(ptr), (bytes));                                                     \
  }
  AL(c->H, (size_t)(L + 1) * c->hslab());
  AL(c->K, (size_t)L * c->kvslab());
  AL(c->V, (size_t)L * c->kvslab());
  AL(c->prev_ids, cap * 4);
  AL(c->d, (size_t)L * cap * 4);
  AL(c->s_cur, (size_t)cfg->max_batch * L * 4);
  AL(c->s_prev, (size_t)cfg->max_batch * L * 4);
  AL(c->budgets, (size_t)cfg->max_batch * L * 4);
  AL(c->sel_idx, (size_t)L * cap * 4);
  AL(c->sel_cnt, (size_t)L * cfg->max_batch * 4);
  AL(c->rowmap, cap * 4);
  AL(c->vrowmap, cap * 4);
  AL(c->stale, (size_t)L * cap);
  AL(c->mrow, cap * 4);
  AL(c->ints, 64);
  AL(c->rope_tab, (size_t)cfg->max_seq * (cfg->head_dim / 2) * sizeof(float2));
  AL(c->xs, cap * xw * c->esz);
  AL(c->Q, cap * Hhd * c->esz);
  AL(c->attn, cap * Hhd * c->esz);
  AL(c->act, cap * F * c->esz);
  AL(c->hmid, cap * D * 4);
  AL(c->C, cap * cw * 4);
  if (cfg->dtype == DCU_BF16) {
    const size_t vt = ((size_t)cfg->vocab + 127) / 128;
    AL(c->smx, vt * cap * sizeof(float2));
    AL(c->smx_arg, vt * cap * 4);
  }
  AL(c->conf, cap * 4);
  AL(c->amax, cap * 4);
  AL(c->seq_off, ((size_t)cfg->max_batch + 1) * 4);
  if (cfg->dtype == DCU_BF16 && (cfg->head_dim == 64 || cfg->head_dim == 128)) {
    const int G = cfg->n_heads / cfg->n_kv_heads;
    c->attn_qt_cap = (int)(((size_t)cfg->max_seq * G + 127) / 128);
    AL(c->attn_po, (size_t)kAttnMaxSplits * cap * Hhd * 4);
    AL(c->attn_ml, (size_t)kAttnMaxSplits * cap * cfg->n_heads * sizeof(float2));
    // chained launches: grid-barrier counters
    c->fused_ok = true;
    AL(c->chain_bar, (size_t)L * kChainBars * 4);
  }
#undef AL
  if (e != cudaSuccess) {
    std::string m = std::string("device allocation failed: ") + cudaGetErrorString(e);
    cudaGetLastError();
    free_all(c);
    delete c;
    return fail(nullptr, DCU_ENOMEM, m);
  }
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&c->cap_stream, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaMemset(c->ints, 0, 64);
  if (e == cudaSuccess && c->chain_bar) e = cudaMemset(c->chain_bar, 0, (size_t)L * kChainBars * 4);
  if (e == cudaSuccess && c->attn_po)  // cluster residency of the tcgen05 attention, queried outside any capture
    for (int sp = 1; sp <= kAttnMaxSplits; ++sp) attn_tc_max_clusters(cfg->head_dim, sp);
  if (e == cudaSuccess) e = cudaMemset(c->stale, 0, (size_t)L * cap);
  if (e == cudaSuccess) e = cudaMemset(c->d, 0, (size_t)L * cap * 4);
  if (e == cudaSuccess) e = cudaMemset(c->s_prev, 0, (size_t)cfg->max_batch * L * 4);
  if (e == cudaSuccess && cfg->rope_theta > 0.0f)
    e = launch_rope_table(c->rope_tab, cfg->max_seq, cfg->head_dim, cfg->rope_theta, 0);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e == cudaSuccess && cfg->dtype == DCU_BF16) {
    // tensor maps of every weight matrix (box 64 x 128) and of the packed activation buffers (box 64 x 128|256)
    bool ok = true;
    auto wmap = [&](CUtensorMap *m, const void *w, size_t rows, size_t k) {
      ok = ok && encode_tmap_bf16(m, w, k, rows, k * 2, 64, 128);
    };
    c->lmaps.resize(L);
    for (int l = 0; l < L; ++l) {
      LayerMaps &m = c->lmaps[l];
      wmap(&m.wq, c->wq[l], Hhd, D);
      wmap(&m.wk, c->wk[l], (size_t)cfg->n_kv_heads * cfg->head_dim, D);
      wmap(&m.wv, c->wv[l], (size_t)cfg->n_kv_heads * cfg->head_dim, D);
      wmap(&m.wo, c->wo[l], D, Hhd);
      wmap(&m.wg, c->wg[l], F, D);
      wmap(&m.wu, c->wu[l], F, D);
      wmap(&m.wd, c->wd[l], D, F);
    }
    wmap(&c->lm_map, c->lm_head, (size_t)cfg->vocab, D);
    // box rows: the token pass, or the buffer rounded up to 16 when it is shorter
    // (rows past the buffer are zero-filled; a box height that is not a multiple
    // of 16 is never used)
    const uint32_t cap16 = (uint32_t)((cap + 15) / 16 * 16);
    c->act_box[0] = cap16 < 128u ? cap16 : 128u;
    c->act_box[1] = cap16 < 256u ? cap16 : 256u;
    const uint32_t boxes[2] = {c->act_box[0], c->act_box[1]};
    for (int i = 0; i < 2; ++i) {
      ok = ok && encode_tmap_bf16(&c->xs_map[i], c->xs, D, cap, D * 2, 64, boxes[i]);
      ok = ok && encode_tmap_bf16(&c->attn_map[i], c->attn, Hhd, cap, Hhd * 2, 64, boxes[i]);
      ok = ok && encode_tmap_bf16(&c->act_map[i], c->act, F, cap, F * 2, 64, boxes[i]);
    }
    if (!ok) {
      free_all(c);
      delete c;
      return fail(nullptr, DCU_ECUDA, "cuTensorMapEncodeTiled failed (driver entry point missing or bad layout)");
    }
    // piece-count tables of the four layer GEMMs' stream-K geometries (built
    // here so that no allocation happens while a step is captured)
    // (the fifth: the W_v GEMM of select_from = "v")
    const size_t widths[5] = {nqkv, D, 2 * F, D, (size_t)cfg->n_kv_heads * cfg->head_dim};
    const size_t ks[5] = {D, Hhd, D, F, D};
    for (int i = 0; i < 5; ++i) {
      SlotGeo g;
      g.n_tiles = (int)((widths[i] + 127) / 128);
      g.kblocks = (int)(ks[i] / 64);
      g.tile_aligned = 0;
      const long long T = (long long)g.n_tiles * g.kblocks;
      g.grid = (int)(T < c->num_sms ? T : c->num_sms);
      g.slot_stride = 0;
      if (!c->slot_table(g)) {
        free_all(c);
        delete c;
        return fail(nullptr, DCU_ENOMEM, "slot table allocation failed");
      }
    }
  }
  if (e != cudaSuccess) {
    std::string m = std::string("context setup failed: ") + cudaGetErrorString(e);
    free_all(c);
    delete c;
    return fail(nullptr, DCU_ECUDA, m);
  }
  *out = c;
  return DCU_OK;
}

void dcu_destroy(dcu_ctx *ctx) {
  if (!ctx) return;
  cudaDeviceSynchronize();
  free_all(ctx);
  delete ctx;
}

int dcu_full_forward(dcu_ctx *c, const int32_t *ids, int32_t B, int32_t N, dcu_stream_t stream) {
  if (!c) return fail(nullptr, DCU_EINVAL, "ctx is NULL");
  if (!ids) return fail(c, DCU_EINVAL, "token_ids is NULL");
  if (B <= 0 || N <= 0) return fail(c, DCU_EINVAL, "B and N must be > 0");
  if (B > c->cfg.max_batch || N > c->cfg.max_seq)
    return fail(c, DCU_ECAPACITY, "B or N above the context's max_batch / max_seq");
  cudaStream_t s = (cudaStream_t)stream;
  c->B = B;
  c->N = N;
  const int BN = B * N;
  if (c->attn_po) {  // K / V tensor maps of the tensor-core attention for this shape
    const dcu_cfg &g = c->cfg;
    c->kv_maps.resize(2 * (size_t)g.n_layers);
    c->kv_maps_tc.resize(2 * (size_t)g.n_layers);
    const uint64_t rows = (uint64_t)B * g.n_kv_heads * N, hd = (uint64_t)g.head_dim;
    for (int l = 0; l < g.n_layers; ++l)
      if (!encode_tmap_bf16(&c->kv_maps[2 * l], c->Kl(l), hd, rows, hd * 2, 64, 64) ||
          !encode_tmap_bf16(&c->kv_maps[2 * l + 1], c->Vl(l), hd, rows, hd * 2, 64, 64) ||
          !encode_tmap_bf16(&c->kv_maps_tc[2 * l], c->Kl(l), hd, rows, hd * 2, 64, 128) ||
          !encode_tmap_bf16(&c->kv_maps_tc[2 * l + 1], c->Vl(l), hd, rows, hd * 2, 64, 128))
        return fail(c, DCU_ECUDA, "cuTensorMapEncodeTiled failed for the K / V cache");
  }
  {
    Prof p(c, DCU_K_REFRESH, s);
    LAUNCH(c, launch_embed_refresh(c->cfg.dtype, ids, c->prev_ids, c->embed, c->Hl(0), c->dl(0), c->g1[0], BN,
                                   c->cfg.d_model, c->cfg.vocab, 1, c->status(), nullptr, s));
  }
  LAUNCH(c, launch_plan_all(B, N, c->rowmap, c->m_total(), c->seq_off, s));
  if (c->chain_bar) CK(c, cudaMemsetAsync(c->chain_bar, 0, (size_t)c->cfg.n_layers * kChainBars * 4, s));
  c->gemm_bn = 256;
  c->gemm_rows_hint = BN;
  for (int l = 0; l < c->cfg.n_layers; ++l)
    if (int rc = run_layer(c, l, true, nullptr, nullptr, 0, s)) return rc;
  CK(c, cudaMemsetAsync(c->s_prev, 0, (size_t)c->cfg.max_batch * c->cfg.n_layers * 4, s));
  CK(c, cudaMemsetAsync(c->stale, 0, (size_t)c->cfg.n_layers * c->cap, s));  // every row was just recomputed
  {
    static const int32_t one = 1;
    CK(c, cudaMemcpyAsync(c->uniform_flag(), &one, 4, cudaMemcpyHostToDevice, s));
  }
  if (c->apd) LAUNCH(c, launch_apd_reset(c->apd_tau, c->apd_prev, c->cap, c->apd_tau0, s));  // a new generation
  c->first_step = true;
  c->have_cache = true;
  c->step_count = 0;
  return DCU_OK;
}

}  // extern "C"

namespace {

// Every launch of one DCU step on stream s (uses only state that is fixed for
// a given (pointers, B_layer, B_window, B, N), so it can be captured once).
int enqueue_step(dcu_ctx *c, const int32_t *ids, const int32_t *keys, const int32_t *nkeys, int B_layer,
                 int B_window, cudaStream_t s) {
  const int L = c->cfg.n_layers, BN = c->B * c->N;
  {
    // expected rows per layer: twice the mean budget plus a few windows per sequence
    // (and the refreshed positions on a refresh step)
    const long long est =
        (long long)c->B * (2LL * B_layer + 2LL * (B_window + 1) + 2LL * (c->force_hi - c->force_lo));
    c->gemm_rows_hint = (int)(est < BN ? est : BN);
    // token pass of the GEMMs: 128 rows when the typical recompute set (half the
    // hint) leaves headroom, since the smaller activation box leaves more shared
    // memory to weight tiles in flight (measured +0.5 % per step at N = 1024);
    // a larger set is still correct (a second pass re-streams the weights)
    c->gemm_bn = (c->gemm_rows_hint / 2) <= 96 ? 128 : 256;
  }
  // grid-barrier counters of the chained launches count up from zero once per step
  if (c->chain_bar) CK(c, cudaMemsetAsync(c->chain_bar, 0, (size_t)L * kChainBars * 4, s));
  {
    Prof p(c, DCU_K_BUDGET, s);
    LAUNCH(c, launch_budget_split(c->s_prev, c->B, L, B_layer, 0, c->uniform_flag(), c->budgets, s));
  }
  {
    Prof p(c, DCU_K_REFRESH, s);
    LAUNCH(c, launch_embed_refresh(c->cfg.dtype, ids, c->prev_ids, c->embed, c->Hl(0), c->dl(0), c->g1[0], BN,
                                   c->cfg.d_model, c->cfg.vocab, 0, c->status(), c->stale_l(0), s));
  }
  for (int l = 0; l < L; ++l)
    if (int rc = run_layer(c, l, false, keys, nkeys, B_window, s)) return rc;
  CK(c, cudaMemcpyAsync(c->s_prev, c->s_cur, (size_t)c->B * L * 4, cudaMemcpyDeviceToDevice, s));
  CK(c, cudaMemsetAsync(c->uniform_flag(), 0, 4, s));
  return DCU_OK;
}

int enqueue_commit(dcu_ctx *c, int rule, float param, int gen_start, int block_len, uint8_t *masked, int32_t *ids,
                   int32_t *out_pos, int32_t *out_count, cudaStream_t s) {
  const dcu_cfg &g = c->cfg;
  const int cap = (int)c->cap;
  {
    {
      Prof p(c, DCU_K_LMHEAD, s);
      LAUNCH(c, launch_plan_masked(masked, c->B, c->N, gen_start, block_len, c->mrow, c->m_masked(), s));
    }
    {
      Prof p(c, DCU_K_LMHEAD, s);
      LAUNCH(c, launch_gather_norm(g.dtype, c->mrow, c->m_masked(), cap, c->Hl(g.n_layers), c->final_norm,
                                   g.rms_eps, g.d_model, c->xs, s));
    }
    GemmSeg lm[1] = {{c->lm_head, g.vocab}};
    const int lm_tiles = (g.vocab + 127) / 128;
    const int lm_grid = lm_tiles < c->num_sms ? lm_tiles : c->num_sms;  // one statistics row per CTA
    c->gemm_bn = 256;
    c->gemm_rows_hint = 256;
    if (g.dtype == DCU_BF16) {
      // tcgen05 LM head with the softmax statistics fused into its epilogue
      Prof p(c, DCU_K_LMHEAD, s);
      TcParams tp;
      memset(&tp, 0, sizeof(tp));
      tp.nphase = 1;
      TcPhase &q = tp.ph[0];
      q.a[0] = c->lm_map;
      q.b = c->xs_map[1];
      tp.b_rows = (int)c->act_box[1];
      const int tiles = (g.vocab + 127) / 128;
      q.seg_tile0[0] = 0;
      q.seg_tile0[1] = tiles;
      q.seg_rows[0] = g.vocab;
      q.nseg = 1;
      q.geo.n_tiles = tiles;
      q.geo.kblocks = g.d_model / 64;
      q.geo.grid = tiles < c->num_sms ? tiles : c->num_sms;
      q.geo.tile_aligned = 1;
      q.ldc = g.vocab;
      tp.m_total = c->m_masked();
      tp.status = c->status();
      tp.epi_mode = EPI_LMHEAD;
      tp.smx = c->smx;
      tp.smx_arg = c->smx_arg;
      tp.ldm = cap;
      tp.sweep = c->pass_sweep ? 2 : 0;  // more than 256 masked rows: two passes per weight tile
      if (rule == DCU_APD) {  // this commit's logits, by position, for the APD signals
        tp.zout = c->apd_z + (size_t)c->apd_flip * cap * g.vocab;
        tp.zrow = c->mrow;
        tp.ldz = g.vocab;
      }
      LAUNCH(c, launch_gemm_tc(tp, 256, s));
    } else {
      SlotGeo geo;
      const ActOperand xs{c->xs, g.d_model, g.d_model, nullptr, nullptr};
      if (int rc = run_gemm(c, xs, c->m_masked(), lm, nullptr, 1, g.vocab, s, &geo, true, DCU_K_LMHEAD)) return rc;
    }
    Prof p(c, DCU_K_LMHEAD, s);
    if (g.dtype == DCU_BF16)
      LAUNCH(c, launch_lm_combine(c->smx, c->smx_arg, lm_grid, cap, c->mrow, c->m_masked(), cap,
                                  c->conf, c->amax, s));
    else
      LAUNCH(c, launch_softmax_max(c->C, g.vocab, c->mrow, c->m_masked(), cap, g.vocab, c->conf, c->amax, s));
    if (rule == DCU_APD) {
      // [DLLM] "关键设计 3": concentration, instability and the threshold update
      float *zcur = c->apd_z + (size_t)c->apd_flip * cap * g.vocab;
      const float *zprev = c->apd_z + (size_t)(1 - c->apd_flip) * cap * g.vocab;
      if (g.dtype == DCU_BF16)
        LAUNCH(c, launch_apd_signals(zcur, g.vocab, 1, nullptr, zprev, c->mrow, c->m_masked(), cap, g.vocab,
                                     c->apd_prev, c->apd_tau, c->apd_alpha, c->apd_beta, c->apd_c, c->apd_h, s));
      else  // the float32 LM head left the logits of packed row r in C
        LAUNCH(c, launch_apd_signals(c->C, g.vocab, 0, zcur, zprev, c->mrow, c->m_masked(), cap, g.vocab,
                                     c->apd_prev, c->apd_tau, c->apd_alpha, c->apd_beta, c->apd_c, c->apd_h, s));
    }
  }
  {
    Prof p(c, DCU_K_COMMIT, s);
    LAUNCH(c, launch_commit_rule(rule, param, c->conf, c->amax, masked, ids, c->B, c->N, gen_start, block_len,
                                 out_pos, out_count, rule == DCU_APD ? c->apd_tau : nullptr, s));
  }
  return DCU_OK;
}

// Runs `body` directly, or through a cached CUDA graph keyed by `key` (captured
// on the context's private stream, launched on s).
template <class F>
int run_graphed(dcu_ctx *c, const uint64_t (&key)[12], cudaStream_t s, F &&body) {
  if (!c->use_graphs) return body(s);
  GraphEntry *g = nullptr;
  for (auto &e : c->graphs)
    if (memcmp(e.key, key, sizeof(key)) == 0) g = &e;
  if (!g) {
    if (c->graphs.size() >= kMaxGraphs) {  // evict the least recently used
      size_t victim = 0;
      for (size_t i = 1; i < c->graphs.size(); ++i)
        if (c->graphs[i].last_use < c->graphs[victim].last_use) victim = i;
      CK(c, cudaStreamSynchronize(c->cap_stream));
      CK(c, cudaDeviceSynchronize());
      free_graph(c->graphs[victim]);
      c->graphs.erase(c->graphs.begin() + (long)victim);
    }
    c->graphs.emplace_back();
    g = &c->graphs.back();
    memcpy(g->key, key, sizeof(key));
    CK(c, cudaStreamBeginCapture(c->cap_stream, cudaStreamCaptureModeThreadLocal));
    const int64_t l0 = c->launches;
    c->capturing = true;
    c->cur_graph = g;
    const int rc = body(c->cap_stream);
    c->capturing = false;
    c->cur_graph = nullptr;
    cudaGraph_t graph = nullptr;
    const cudaError_t e = cudaStreamEndCapture(c->cap_stream, &graph);
    g->kernels = c->launches - l0;
    c->launches = l0;
    cudaError_t ei = cudaSuccess;
    if (rc == DCU_OK && e == cudaSuccess) ei = cudaGraphInstantiate(&g->exec, graph, 0);
    if (graph) cudaGraphDestroy(graph);
    if (rc != DCU_OK || e != cudaSuccess || ei != cudaSuccess) {
      free_graph(*g);
      c->graphs.pop_back();
      cudaGetLastError();
      if (rc != DCU_OK) return rc;
      return fail(c, DCU_ECUDA, std::string("graph capture failed: ") +
                                    cudaGetErrorString(e != cudaSuccess ? e : ei));
    }
  }
  g->last_use = ++c->use_clock;
  CK(c, cudaGraphLaunch(g->exec, s));
  ++g->replays;
  c->launches += g->kernels;
  return DCU_OK;
}

}  // namespace

extern "C" {

int dcu_step(dcu_ctx *c, const int32_t *ids, const int32_t *keys, const int32_t *nkeys, int32_t B_layer,
             int32_t B_window, dcu_stream_t stream) {
  if (!c) return fail(nullptr, DCU_EINVAL, "ctx is NULL");
  if (!c->have_cache) return fail(c, DCU_ESTATE, "dcu_step before dcu_full_forward");
  if (!ids || !keys || !nkeys) return fail(c, DCU_EINVAL, "token_ids, key_positions or n_keys is NULL");
  if (B_layer < 0 || B_window < 0) return fail(c, DCU_EINVAL, "B_layer and B_window must be >= 0");
  // periodic full refresh due at this step (1, 2, ... after the dense forward)
  const int64_t step = c->step_count + 1;
  {
    const int g0 = c->refresh_gen_start < c->N ? c->refresh_gen_start : c->N;
    const bool pr = c->refresh_prompt > 0 && step % c->refresh_prompt == 0;
    const bool gr = c->refresh_gen > 0 && step % c->refresh_gen == 0;
    c->force_lo = pr ? 0 : (gr ? g0 : 0);
    c->force_hi = gr ? c->N : (pr ? g0 : 0);
  }
  const uint64_t key[12] = {1,
                            (uint64_t)(uintptr_t)ids,
                            (uint64_t)(uintptr_t)keys,
                            (uint64_t)(uintptr_t)nkeys,
                            (uint64_t)B_layer,
                            (uint64_t)B_window,
                            ((uint64_t)c->B << 32) | (uint64_t)c->N,
                            (uint64_t)(c->prof_max > 0),
                            ((uint64_t)(uint32_t)c->force_lo << 32) | (uint64_t)(uint32_t)c->force_hi,
                            (uint64_t)c->select_from | ((uint64_t)c->fused << 8) | ((uint64_t)c->nx_count << 16) |
                                ((uint64_t)c->attn_impl << 32) | ((uint64_t)(c->gemm_smem >> 10) << 36) |
                                ((uint64_t)c->pass_sweep << 48),
                            0,
                            0};
  int rc = run_graphed(c, key, (cudaStream_t)stream,
                       [&](cudaStream_t s) { return enqueue_step(c, ids, keys, nkeys, B_layer, B_window, s); });
  if (rc == DCU_OK) {
    c->first_step = false;
    c->step_count = step;
  }
  return rc;
}

int dcu_set_option(dcu_ctx *c, int32_t option, int32_t value) {
  if (!c) return fail(nullptr, DCU_EINVAL, "ctx is NULL");
  switch (option) {
    case DCU_OPT_FUSED_EPILOGUE:
      if (value && !c->fused_ok)
        return fail(c, DCU_EINVAL, "fused epilogues need a bf16 model with head_dim 64 or 128");
      if (value < 0 || value > 2) return fail(c, DCU_EINVAL, "DCU_OPT_FUSED_EPILOGUE takes 0, 1 or 2");
      c->fused = value;
      return DCU_OK;
    case DCU_OPT_L2_PREFETCH:
      if (value < 0 || value > 4096) return fail(c, DCU_EINVAL, "L2 prefetch units must lie in [0, 4096]");
      c->nx_count = value;
      return DCU_OK;
    case DCU_OPT_GEMM_SMEM_KB:
      if (value < 136 || (size_t)value * 1024u > kTcSmem)
        return fail(c, DCU_EINVAL, "DCU_OPT_GEMM_SMEM_KB must lie in [136, 220]");
      c->gemm_smem = (size_t)value * 1024u;
      return DCU_OK;
    case DCU_OPT_ATTENTION:
      if (value != DCU_ATTN_TCGEN05 && value != DCU_ATTN_MMA_SYNC)
        return fail(c, DCU_EINVAL, "DCU_OPT_ATTENTION takes DCU_ATTN_TCGEN05 or DCU_ATTN_MMA_SYNC");
      c->attn_impl = value;
      return DCU_OK;
    case DCU_OPT_GEMM_PASS_SWEEP:
      if (value != 0 && value != 1) return fail(c, DCU_EINVAL, "DCU_OPT_GEMM_PASS_SWEEP takes 0 or 1");
      c->pass_sweep = value;
      return DCU_OK;
    default:
      return fail(c, DCU_EINVAL, "unknown option");
  }
}

int dcu_set_apd(dcu_ctx *c, float alpha, float beta, float tau0) {
  if (!c) return fail(nullptr, DCU_EINVAL, "ctx is NULL");
  if (!(alpha >= 0.0f) || !(beta >= 0.0f) || !std::isfinite(alpha) || !std::isfinite(beta) || !std::isfinite(tau0))
    return fail(c, DCU_EINVAL, "alpha and beta must be finite and >= 0, tau0 finite");
  if (c->capturing) return fail(c, DCU_ESTATE, "dcu_set_apd inside a stream capture");
  if (!c->apd_z) {
    const size_t cap = (size_t)c->cap, V = (size_t)c->cfg.vocab;
    cudaError_t e = dalloc(c, &c->apd_z, 2 * cap * V * sizeof(float));
    if (e == cudaSuccess) e = dalloc(c, &c->apd_tau, cap * sizeof(float));
    if (e == cudaSuccess) e = dalloc(c, &c->apd_c, cap * sizeof(float));
    if (e == cudaSuccess) e = dalloc(c, &c->apd_h, cap * sizeof(float));
    if (e == cudaSuccess) e = dalloc(c, &c->apd_prev, cap);
    if (e == cudaSuccess) e = cudaMemset(c->apd_c, 0, cap * sizeof(float));
    if (e == cudaSuccess) e = cudaMemset(c->apd_h, 0, cap * sizeof(float));
    if (e != cudaSuccess) {
      cudaGetLastError();
      return fail(c, DCU_ENOMEM, std::string("APD buffers: ") + cudaGetErrorString(e));
    }
  }
  c->apd = true;
  c->apd_alpha = alpha;
  c->apd_beta = beta;
  c->apd_tau0 = tau0;
  c->apd_flip = 0;
  CK(c, launch_apd_reset(c->apd_tau, c->apd_prev, c->cap, tau0, nullptr));
  CK(c, cudaDeviceSynchronize());
  return DCU_OK;
}

int dcu_set_select_from(dcu_ctx *c, int32_t source) {
  if (!c) return fail(nullptr, DCU_EINVAL, "ctx is NULL");
  if (source != DCU_SELECT_INPUT && source != DCU_SELECT_VALUE)
    return fail(c, DCU_EINVAL, "source must be DCU_SELECT_INPUT or DCU_SELECT_VALUE");
  c->select_from = source;
  return DCU_OK;
}

int dcu_set_refresh(dcu_ctx *c, int32_t gen_start, int32_t prompt_interval, int32_t gen_interval) {
  if (!c) return fail(nullptr, DCU_EINVAL, "ctx is NULL");
  if (gen_start < 0 || prompt_interval < 0 || gen_interval < 0)
    return fail(c, DCU_EINVAL, "gen_start and the intervals must be >= 0");
  c->refresh_gen_start = gen_start;
  c->refresh_prompt = prompt_interval;
  c->refresh_gen = gen_interval;
  return DCU_OK;
}

int commit_select_block(dcu_ctx *c, int32_t rule, float param, int32_t gen_start, int32_t block_len,
                        uint8_t *masked, int32_t *ids, int32_t *out_pos, int32_t *out_count, dcu_stream_t stream) {
  if (!c) return fail(nullptr, DCU_EINVAL, "ctx is NULL");
  if (!c->have_cache) return fail(c, DCU_ESTATE, "commit_select before dcu_full_forward");
  if (rule != DCU_FRECHET && rule != DCU_THRESHOLD && rule != DCU_FACTOR && rule != DCU_APD)
    return fail(c, DCU_EINVAL, "rule must be DCU_FRECHET, DCU_THRESHOLD, DCU_FACTOR or DCU_APD");
  if (rule == DCU_APD && !c->apd) return fail(c, DCU_ESTATE, "DCU_APD before dcu_set_apd");
  if (!masked || !ids || !out_pos || !out_count) return fail(c, DCU_EINVAL, "a buffer is NULL");
  if (block_len > 0 && (gen_start < 0 || gen_start >= c->N))
    return fail(c, DCU_EINVAL, "gen_start must lie in [0, N) when block_len > 0");
  if (block_len < 0) block_len = 0;
  uint32_t pbits;
  memcpy(&pbits, &param, 4);
  uint32_t abits = 0, bbits = 0;
  memcpy(&abits, &c->apd_alpha, 4);
  memcpy(&bbits, &c->apd_beta, 4);
  const bool apd = rule == DCU_APD;
  const uint64_t key[12] = {2,
                            (uint64_t)rule,
                            (uint64_t)pbits,
                            (uint64_t)(uintptr_t)masked,
                            (uint64_t)(uintptr_t)ids,
                            (uint64_t)(uintptr_t)out_pos,
                            (uint64_t)(uintptr_t)out_count,
                            ((uint64_t)c->B << 32) | (uint64_t)c->N,
                            (uint64_t)(c->prof_max > 0),
                            ((uint64_t)(uint32_t)gen_start << 32) | (uint64_t)(uint32_t)block_len,
                            apd ? (uint64_t)(1 + c->apd_flip) : 0,
                            apd ? (((uint64_t)abits << 32) | bbits) : 0};
  const int rc = run_graphed(c, key, (cudaStream_t)stream, [&](cudaStream_t s) {
    return enqueue_commit(c, rule, param, gen_start, block_len, masked, ids, out_pos, out_count, s);
  });
  if (rc == DCU_OK && apd) c->apd_flip ^= 1;  // this commit's logits are the next one's previous
  return rc;
}

int commit_select(dcu_ctx *c, int32_t rule, float param, uint8_t *masked, int32_t *ids, int32_t *out_pos,
                  int32_t *out_count, dcu_stream_t stream) {
  return commit_select_block(c, rule, param, 0, 0, masked, ids, out_pos, out_count, stream);
}

int dcu_set_graphs(dcu_ctx *c, int32_t on) {
  if (!c) return fail(nullptr, DCU_EINVAL, "ctx is NULL");
  c->use_graphs = on != 0;
  return DCU_OK;
}

int dcu_status(dcu_ctx *c, dcu_stream_t stream, int32_t *bits) {
  if (!c) return fail(nullptr, DCU_EINVAL, "ctx is NULL");
  CK(c, cudaStreamSynchronize((cudaStream_t)stream));
  int32_t v = 0;
  CK(c, cudaMemcpy(&v, c->status(), 4, cudaMemcpyDeviceToHost));
  if (bits) *bits = v;
  if (v != 0) {
    CK(c, cudaMemset(c->status(), 0, 4));
    return fail(c, DCU_EDEVICE, "device status word " + std::to_string(v));
  }
  return DCU_OK;
}

// ---------------------------------------------------------------- stateless kernels

int dcu_budget_split(const float *s_prev, int32_t B, int32_t L, int32_t B_layer, int32_t uniform, int32_t *budgets,
                     dcu_stream_t stream) {
  if (!s_prev || !budgets || B <= 0 || L <= 0 || L > 1024 || B_layer < 0)
    return fail(nullptr, DCU_EINVAL, "dcu_budget_split: bad argument");
  CK(nullptr, launch_budget_split(s_prev, B, L, B_layer, uniform, nullptr, budgets, (cudaStream_t)stream));
  return DCU_OK;
}

int dcu_select_tokens(const float *d, const int32_t *keys, const int32_t *nkeys, const int32_t *budgets, int32_t B,
                      int32_t N, int32_t B_window, int32_t window_mode, int32_t *idx, int32_t *count, float *s,
                      int32_t *status, dcu_stream_t stream) {
  if (!d || !keys || !nkeys || !budgets || !idx || !count || !s || B <= 0 || N <= 0 || N > 16384 ||
      B_window < 0 || (window_mode != 0 && window_mode != 1))
    return fail(nullptr, DCU_EINVAL, "dcu_select_tokens: bad argument");
  CK(nullptr, launch_select(d, keys, nkeys, budgets, 1, B, N, B_window, window_mode, 0, 0, idx, count, s, 1, nullptr,
                            nullptr, nullptr, nullptr, nullptr, status, (cudaStream_t)stream));
  return DCU_OK;
}

int dcu_cosine_distance(const void *x, const void *y, const float *gain, int64_t rows, int32_t D, int32_t dtype,
                        float *d, dcu_stream_t stream) {
  if (!x || !y || !gain || !d || rows < 0 || D <= 0 || D % 8 || (dtype != DCU_F32 && dtype != DCU_BF16))
    return fail(nullptr, DCU_EINVAL, "dcu_cosine_distance: bad argument");
  CK(nullptr, launch_cosine_distance(dtype, x, y, gain, rows, D, d, (cudaStream_t)stream));
  return DCU_OK;
}

int dcu_selftest_wait_timeout(int32_t *status, dcu_stream_t stream) {
  if (!status) return fail(nullptr, DCU_EINVAL, "dcu_selftest_wait_timeout: status is NULL");
  CK(nullptr, launch_wait_timeout_probe(status, (cudaStream_t)stream));
  return DCU_OK;
}

int dcu_commit_rule_block(int32_t rule, float param, int32_t gen_start, int32_t block_len, const float *conf,
                          const int32_t *argmax, uint8_t *masked, int32_t *ids, int32_t B, int32_t N,
                          int32_t *out_pos, int32_t *out_count, dcu_stream_t stream) {
  if ((rule != DCU_FRECHET && rule != DCU_THRESHOLD && rule != DCU_FACTOR) || !conf || !argmax || !masked || !ids ||
      !out_pos || !out_count || B <= 0 || N <= 0 || N > 16384 || (block_len > 0 && (gen_start < 0 || gen_start >= N)))
    return fail(nullptr, DCU_EINVAL, "dcu_commit_rule: bad argument");
  CK(nullptr, launch_commit_rule(rule, param, conf, argmax, masked, ids, B, N, gen_start, block_len > 0 ? block_len : 0,
                                 out_pos, out_count, nullptr, (cudaStream_t)stream));
  return DCU_OK;
}

int dcu_commit_rule(int32_t rule, float param, const float *conf, const int32_t *argmax, uint8_t *masked,
                    int32_t *ids, int32_t B, int32_t N, int32_t *out_pos, int32_t *out_count, dcu_stream_t stream) {
  return dcu_commit_rule_block(rule, param, 0, 0, conf, argmax, masked, ids, B, N, out_pos, out_count, stream);
}

int dcu_linear(const void *X, const void *W, int32_t M, int32_t K, int32_t Nout, int32_t dtype, float *Y,
               dcu_stream_t stream) {
  auto mis = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; };
  if (!X || !W || !Y || M < 0 || K <= 0 || Nout <= 0 || (dtype != DCU_F32 && dtype != DCU_BF16) || mis(X) ||
      mis(W) || mis(Y) || (dtype == DCU_BF16 ? (K % 64) : (K % 16)))
    return fail(nullptr, DCU_EINVAL, "dcu_linear: bad argument");
  if (M == 0) return DCU_OK;
  cudaStream_t s = (cudaStream_t)stream;
  if (dtype == DCU_F32) {
    GemmSeg seg{W, Nout};
    CK(nullptr, launch_gemm_simt(dtype, X, K, nullptr, M, &seg, 1, K, Y, Nout, s));
    return DCU_OK;
  }
  TcParams tp;
  memset(&tp, 0, sizeof(tp));
  tp.nphase = 1;
  TcPhase &q = tp.ph[0];
  const int bn = M <= 128 ? 128 : 256;
  const int m16 = (M + 15) / 16 * 16, b_rows = m16 < bn ? m16 : bn;  // activation box rows (multiple of 16)
  if (!encode_tmap_bf16(&q.a[0], W, (uint64_t)K, (uint64_t)Nout, (uint64_t)K * 2, 64, 128) ||
      !encode_tmap_bf16(&q.b, X, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, 64, (uint32_t)b_rows))
    return fail(nullptr, DCU_ECUDA, "dcu_linear: cuTensorMapEncodeTiled failed");
  tp.b_rows = b_rows;
  tp.sweep = 512 / bn;  // several token passes share each weight tile
  const int tiles = (Nout + 127) / 128;
  q.seg_tile0[0] = 0;
  q.seg_tile0[1] = tiles;
  q.seg_col0[0] = 0;
  q.seg_rows[0] = Nout;
  q.nseg = 1;
  q.ldc = Nout;
  tp.m_total = nullptr;
  tp.m_host = M;
  tp.out = Y;
  tp.status = nullptr;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  q.geo.n_tiles = tiles;
  q.geo.kblocks = K / 64;
  q.geo.tile_aligned = 1;
  q.geo.grid = tiles < sms ? tiles : sms;
  CK(nullptr, launch_gemm_tc(tp, bn, s));
  return DCU_OK;
}

// ---------------------------------------------------------------- introspection

static int tensor_ptr(dcu_ctx *c, int kind, int layer, char **p, int64_t *bytes) {
  if (!c->have_cache) return fail(c, DCU_ESTATE, "no active shape (run dcu_full_forward first)");
  const dcu_cfg &g = c->cfg;
  const int L = g.n_layers;
  const int64_t BN = (int64_t)c->B * c->N;
  auto need = [&](int lo, int hi) { return layer >= lo && layer <= hi; };
  switch (kind) {
    case DCU_T_H:
      if (!need(0, L)) break;
      *p = (char *)c->Hl(layer);
      *bytes = BN * g.d_model * (int64_t)c->esz;
      return DCU_OK;
    case DCU_T_K:
    case DCU_T_V:
      if (!need(0, L - 1)) break;
      *p = (char *)(kind == DCU_T_K ? c->Kl(layer) : c->Vl(layer));
      *bytes = BN * g.n_kv_heads * g.head_dim * (int64_t)c->esz;
      return DCU_OK;
    case DCU_T_D:
      if (!need(0, L - 1)) break;
      *p = (char *)c->dl(layer);
      *bytes = BN * 4;
      return DCU_OK;
    case DCU_T_S:
      *p = (char *)c->s_cur;
      *bytes = (int64_t)c->B * L * 4;
      return DCU_OK;
    case DCU_T_S_PREV:
      *p = (char *)c->s_prev;
      *bytes = (int64_t)c->B * L * 4;
      return DCU_OK;
    case DCU_T_BUDGET:
      *p = (char *)c->budgets;
      *bytes = (int64_t)c->B * L * 4;
      return DCU_OK;
    case DCU_T_SEL:
      if (!need(0, L - 1)) break;
      *p = (char *)(c->sel_idx + (size_t)layer * c->cap);
      *bytes = BN * 4;
      return DCU_OK;
    case DCU_T_SEL_COUNT:
      if (!need(0, L - 1)) break;
      *p = (char *)(c->sel_cnt + (size_t)layer * g.max_batch);
      *bytes = (int64_t)c->B * 4;
      return DCU_OK;
    case DCU_T_CONF:
      *p = (char *)c->conf;
      *bytes = BN * 4;
      return DCU_OK;
    case DCU_T_ARGMAX:
      *p = (char *)c->amax;
      *bytes = BN * 4;
      return DCU_OK;
    case DCU_T_APD_TAU:
    case DCU_T_APD_C:
    case DCU_T_APD_H:
      if (!c->apd) return fail(c, DCU_ESTATE, "APD is not enabled (dcu_set_apd)");
      *p = (char *)(kind == DCU_T_APD_TAU ? c->apd_tau : (kind == DCU_T_APD_C ? c->apd_c : c->apd_h));
      *bytes = BN * 4;
      return DCU_OK;
    case DCU_T_STALE:
      if (!need(0, L - 1)) break;
      *p = (char *)c->stale_l(layer);
      *bytes = BN;
      return DCU_OK;
    case DCU_T_ATTN:
      *p = c->attn;
      *bytes = BN * g.n_heads * g.head_dim * (int64_t)c->esz;
      return DCU_OK;
    default:
      return fail(c, DCU_EINVAL, "unknown tensor kind");
  }
  return fail(c, DCU_EINVAL, "layer out of range for this tensor kind");
}

int dcu_tensor_bytes(const dcu_ctx *cc, int32_t kind, int64_t *bytes) {
  dcu_ctx *c = const_cast<dcu_ctx *>(cc);
  if (!c || !bytes) return fail(nullptr, DCU_EINVAL, "ctx or bytes is NULL");
  char *p;
  return tensor_ptr(c, kind, 0, &p, bytes);  // every kind's size is the same at every layer
}

int dcu_get_tensor(dcu_ctx *c, int32_t kind, int32_t layer, void *dst, int64_t bytes, dcu_stream_t stream) {
  if (!c || !dst) return fail(c, DCU_EINVAL, "ctx or dst is NULL");
  char *p;
  int64_t n;
  if (int rc = tensor_ptr(c, kind, layer, &p, &n)) return rc;
  if (bytes != n) return fail(c, DCU_EINVAL, "size mismatch: expected " + std::to_string(n) + " bytes");
  CK(c, cudaMemcpyAsync(dst, p, n, cudaMemcpyDeviceToDevice, (cudaStream_t)stream));
  return DCU_OK;
}

int dcu_set_tensor(dcu_ctx *c, int32_t kind, int32_t layer, const void *src, int64_t bytes, dcu_stream_t stream) {
  if (!c || !src) return fail(c, DCU_EINVAL, "ctx or src is NULL");
  if (kind != DCU_T_H && kind != DCU_T_K && kind != DCU_T_V && kind != DCU_T_S_PREV && kind != DCU_T_STALE)
    return fail(c, DCU_EINVAL, "only H, K, V, S_PREV and STALE can be set");
  char *p;
  int64_t n;
  if (int rc = tensor_ptr(c, kind, layer, &p, &n)) return rc;
  if (bytes != n) return fail(c, DCU_EINVAL, "size mismatch: expected " + std::to_string(n) + " bytes");
  CK(c, cudaMemcpyAsync(p, src, n, cudaMemcpyDeviceToDevice, (cudaStream_t)stream));
  if (kind == DCU_T_S_PREV) {
    c->first_step = false;
    CK(c, cudaMemsetAsync(c->uniform_flag(), 0, 4, (cudaStream_t)stream));
  }
  return DCU_OK;
}

// ---------------------------------------------------------------- profiling

int dcu_profile_enable(dcu_ctx *c, int32_t max_launches) {
  if (!c || max_launches < 0) return fail(c, DCU_EINVAL, "bad argument");
  for (auto &pc : c->prof) {
    for (auto &e : pc.ev) {
      cudaEventDestroy(e.a);
      cudaEventDestroy(e.b);
    }
    pc.ev.clear();
    pc.used = pc.dropped = 0;
    for (int i = 0; i < max_launches; ++i) {
      EventPair e;
      CK(c, cudaEventCreate(&e.a));
      CK(c, cudaEventCreate(&e.b));
      pc.ev.push_back(e);
    }
  }
  c->prof_max = max_launches;
  return DCU_OK;
}

int dcu_profile_read(dcu_ctx *c, int32_t k, double *total_ms, int64_t *launches, int32_t reset) {
  if (!c || k < 0 || k >= DCU_K_COUNT || !total_ms || !launches) return fail(c, DCU_EINVAL, "bad argument");
  ProfClass &pc = c->prof[k];
  double t = 0.0;
  for (int64_t i = 0; i < pc.used; ++i) {
    CK(c, cudaEventSynchronize(pc.ev[i].b));
    float ms = 0.f;
    CK(c, cudaEventElapsedTime(&ms, pc.ev[i].a, pc.ev[i].b));
    t += ms;
  }
  int64_t n = pc.used;
  // graphs: event-record nodes hold the times of the graph's most recent
  // replay; they stand for each of its replays since the last reset
  for (auto &g : c->graphs) {
    if (g.replays == 0) continue;
    double tg = 0.0;
    int64_t ng = 0;
    for (auto &e : g.ev) {
      if (e.first != k) continue;
      CK(c, cudaEventSynchronize(e.second.b));
      float ms = 0.f;
      CK(c, cudaEventElapsedTime(&ms, e.second.a, e.second.b));
      tg += ms;
      ++ng;
    }
    t += tg * (double)g.replays;
    n += ng * g.replays;
  }
  *total_ms = t;
  *launches = n;
  if (pc.dropped) return fail(c, DCU_ECAPACITY, "more launches than profile slots");
  if (reset) {
    pc.used = pc.dropped = 0;
    bool all_read = true;
    for (int kk = 0; kk < DCU_K_COUNT; ++kk) all_read = all_read && (kk <= k);
    if (all_read)
      for (auto &g : c->graphs) g.replays = 0;
  }
  return DCU_OK;
}

int64_t dcu_launch_count(const dcu_ctx *c) { return c ? c->launches : 0; }

const char *dcu_kernel_class_name(int32_t k) {
  static const char *names[DCU_K_COUNT] = {"refresh", "budget",   "select", "gather", "gemm",
                                           "epilogue", "attention", "scatter", "lmhead", "commit"};
  return (k >= 0 && k < DCU_K_COUNT) ? names[k] : "?";
}

}  // extern "C"
