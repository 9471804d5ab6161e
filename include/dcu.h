/*
 * dcu.h -- C ABI of the B200 (sm_100a) Dynamic Cache Updating library, libdcu.so.
 *
 * The library runs the data-parallel hot path of one denoising step of a
 * masked-diffusion LLM with bidirectional attention under Dynamic Cache
 * Updating (DCU), and the per-step commit that follows it.  Sources:
 *
 *   [DLLM]    "Dynamic-dLLM: Dynamic Cache-Budget and Adaptive Parallel
 *             Decoding for Training-Free Acceleration of Diffusion LLM"
 *             (papernotes.org ICLR 2026 note), section "关键设计 1" (token
 *             dynamics d, layer dynamics s, proportional layer budget) and
 *             section "关键设计 2" (forced update window around key tokens).
 *   [FRECHET] "Fast-dLLM++: Fréchet Profile Decoding for Faster Diffusion LLM
 *             Inference" (papernotes.org ICML 2026 workshop note), sections
 *             "整体框架", "关键设计 1", "关键设计 2" (Fréchet profile rule) and
 *             "研究背景与动机" (Fast-dLLM threshold and factor rules).
 *
 * Conventions
 *   - Every call returns int: DCU_OK (0) or a negative DCU_E* code; the text
 *     of the last error is dcu_last_error(ctx) (ctx may be NULL for errors of
 *     calls that have no context).  No C++ exception crosses the ABI.
 *   - Pointers marked "dev" are CUDA device pointers; "host" are host
 *     pointers.  The caller owns every pointer it passes; the library never
 *     frees them.  A context owns its caches and scratch and frees them in
 *     dcu_destroy.
 *   - Work is enqueued asynchronously on the given stream (a cudaStream_t;
 *     NULL is the legacy default stream).  Arguments are checked on the host
 *     at call time (DCU_EINVAL).  Conditions only the device can see (a key
 *     position outside [0, N), a token id outside [0, vocab)) set bits of a
 *     device status word, which dcu_status() reads; kernels never trap.
 *   - Row-major layouts throughout.  bf16 is IEEE bfloat16 (uint16 storage).
 *   - Norm gains are always float32.
 */
#ifndef DCU_H
#define DCU_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- error codes ---- */
#define DCU_OK          0
#define DCU_EINVAL     -1   /* bad argument or shape, checked on the host          */
#define DCU_ENOMEM     -2   /* a device allocation failed                          */
#define DCU_ECUDA      -3   /* a CUDA runtime call or kernel launch failed         */
#define DCU_ECAPACITY  -4   /* B or N above the context's max_batch / max_seq      */
#define DCU_ESTATE     -5   /* call out of order (e.g. dcu_step before a full forward) */
#define DCU_EDEVICE    -6   /* dcu_status: the device status word was non-zero     */

/* ---- device status word bits (dcu_status) ---- */
#define DCU_ST_BAD_KEY   1  /* a key position outside [0, N) was ignored */
#define DCU_ST_BAD_TOKEN 2  /* a token id outside [0, vocab) was clamped   */
#define DCU_ST_TIMEOUT   4  /* a bounded device wait gave up                */

/* ---- dtypes, rules, window modes ---- */
#define DCU_F32   0
#define DCU_BF16  1

#define DCU_FRECHET   0     /* n* = max{n : G_n > delta}, else 1  ([FRECHET] "关键设计 2") */
#define DCU_THRESHOLD 1     /* commit every c_i >= tau, else the top one ([FRECHET] "研究背景与动机") */
#define DCU_FACTOR    2     /* largest n with (n+1)(1 - c_(n)) < f, else 1 (same section)      */
#define DCU_APD       3     /* c_i >= tau_i with per-position adaptive tau, else the top one
                               ([DLLM] "关键设计 3"; commit_select after dcu_set_apd only)      */

#define DCU_SELECT_INPUT 0   /* d from the normalised layer inputs ([DLLM] "关键设计 1")          */
#define DCU_SELECT_VALUE 1   /* d from recomputed vs cached Value rows ([README] select_from="v") */

#define DCU_WINDOW_INCLUSIVE 0  /* [p - Bw/2, p + Bw/2], Bw+1 positions ([DLLM] "关键设计 2") */
#define DCU_WINDOW_HALFOPEN  1  /* [p - Bw/2, p - Bw/2 + Bw), Bw positions                   */

typedef struct dcu_ctx dcu_ctx;
typedef void *dcu_stream_t;   /* cudaStream_t */

/* Model and capacity.  Invariants checked by dcu_create: every size > 0;
 * d_model % 64 == 0; head_dim % 16 == 0 and head_dim <= 256 and even;
 * n_heads % n_kv_heads == 0; d_ffn % 64 == 0; max_seq <= 16384;
 * mask_id in [0, vocab); dtype DCU_F32 or DCU_BF16. */
typedef struct {
  int32_t n_layers, d_model, n_heads, n_kv_heads, head_dim, d_ffn, vocab, mask_id;
  int32_t max_batch, max_seq;
  int32_t dtype;          /* DCU_F32 | DCU_BF16: weights, caches and GEMM operands */
  float   rms_eps;        /* RMSNorm epsilon                                       */
  float   rope_theta;     /* rotate-half RoPE base; 0 disables RoPE                */
  int32_t window_mode;    /* DCU_WINDOW_INCLUSIVE | DCU_WINDOW_HALFOPEN            */
} dcu_cfg;

/* Weights: device pointers in cfg.dtype (norm gains float32), row-major
 * [out][in].  embed, lm_head: [vocab][d_model]; final_norm: [d_model].
 * Per layer (host arrays of n_layers device pointers): attn_norm, ffn_norm
 * [d_model]; wq [n_heads*head_dim][d_model]; wk, wv [n_kv_heads*head_dim][d_model];
 * wo [d_model][n_heads*head_dim]; w_gate, w_up [d_ffn][d_model];
 * w_down [d_model][d_ffn].  Device pointers must be 16-byte aligned and stay
 * valid for the life of the context; the host arrays are copied. */
typedef struct {
  const void *embed, *final_norm, *lm_head;
  const void *const *attn_norm, *const *wq, *const *wk, *const *wv, *const *wo;
  const void *const *ffn_norm, *const *w_gate, *const *w_up, *const *w_down;
} dcu_weights;

/* Creates a context on the current CUDA device: validates cfg, allocates the
 * per-layer caches (H_0..H_L [max_batch][max_seq][d_model], K/V
 * [max_batch][n_kv_heads][max_seq][head_dim] per layer) and scratch.
 * Returns DCU_EINVAL (bad cfg/weights), DCU_ENOMEM or DCU_ECUDA. */
int dcu_create(const dcu_weights *weights, const dcu_cfg *cfg, dcu_ctx **out);

/* Frees everything the context owns (after synchronising its device). */
void dcu_destroy(dcu_ctx *ctx);

/* Text of the last error of ctx (or of a context-less call when ctx is NULL). */
const char *dcu_last_error(const dcu_ctx *ctx);

/* Dense forward of B sequences of N tokens (the full recompute that
 * DCU avoids, [DLLM] "研究背景与动机"): fills H_0..H_L and every layer's K/V
 * for all positions and makes (B, N) the active shape.  The next dcu_step
 * splits its budget uniformly.  token_ids: dev int32 [B][N]. */
int dcu_full_forward(dcu_ctx *ctx, const int32_t *token_ids, int32_t B, int32_t N, dcu_stream_t stream);

/* One DCU step on the active (B, N) ([DLLM] "关键设计 1" and "关键设计 2"):
 *   1. layer budgets B^l = floor + largest remainder of (B_layer * L) s^{prev,l} / sum_k s^{prev,k}
 *      (uniform B_layer on the first step after a full forward or when sum s = 0);
 *   2. layer-0 inputs of positions whose id changed since the last call are
 *      replaced by their embeddings;
 *   3. per layer: d_i = 1 - cos(g*x_new, g*x_cached), s^l = mean_i d_i,
 *      U^l = window(keys, B_window) union top-B^l of d outside it, recompute of
 *      U^l's rows (QKV + RoPE, K/V write, attention over all N cached keys,
 *      O + residual, SwiGLU FFN + residual) and scatter into H_{l+1}.
 * token_ids: dev int32 [B][N] (current ids); key_positions: dev int32 [B][N]
 * (row b holds n_keys[b] positions unmasked at the previous step, e.g. the
 * out_positions of commit_select); n_keys: dev int32 [B].
 * Returns DCU_ESTATE before the first dcu_full_forward. */
int dcu_step(dcu_ctx *ctx, const int32_t *token_ids, const int32_t *key_positions, const int32_t *n_keys,
             int32_t B_layer, int32_t B_window, dcu_stream_t stream);

/* Performance options of a context (results agree within the parity
 * tolerances either way; every path is tested).
 *   DCU_OPT_FUSED_EPILOGUE (bf16 models with head_dim 64 or 128; default 0):
 *     0 = each layer GEMM stores its split-K pieces and separate kernels apply
 *     the epilogues (RoPE and the K/V write, residual + RMSNorm, SwiGLU,
 *     residual + scatter + next-layer d);
 *     1 = chained launches: the QKV GEMM with its epilogue, and the O, gate|up
 *     and down GEMMs with theirs, each run as one persistent cooperative
 *     launch (one CTA per SM) whose phases are separated by grid barriers and
 *     whose epilogues are spread over all CTAs;
 *     2 = as 1 without the cooperative launch attribute (every CTA still fits
 *     one per SM; every barrier wait is time-bounded and reports
 *     DCU_ST_TIMEOUT if a CTA never arrives).
 * DCU_EINVAL for an unknown option or an unsupported value. */
#define DCU_OPT_FUSED_EPILOGUE 1
/*   DCU_OPT_L2_PREFETCH (default 16): when a layer GEMM has issued its own
 *     weight loads, each CTA prefetches this many (tile, k block) units of the
 *     next GEMM's weights (the next layer's QKV, or the LM head after the last
 *     layer) into L2, so HBM keeps streaming through the dependent kernels in
 *     between; 0 turns it off, at most 4096. */
#define DCU_OPT_L2_PREFETCH 2
/*   DCU_OPT_ATTENTION (bf16 models with head_dim 64 or 128): the attention of
 *     the recomputed rows over all N keys.  DCU_ATTN_TCGEN05 (default): 5th-gen
 *     tensor cores, S and O accumulated in tensor memory, 128-key chunks;
 *     DCU_ATTN_MMA_SYNC: warp-level mma.sync with the online softmax in
 *     registers, 64-key chunks.  Both split the keys over at most 8 CTAs per
 *     (sequence, kv head, query tile) and merge the splits in split order. */
#define DCU_OPT_ATTENTION 3
/*   DCU_OPT_GEMM_SMEM_KB (136 .. 220, default 220): dynamic shared memory of a
 *     layer GEMM CTA (its weight ring).  A smaller ring leaves room on each SM
 *     for the CTAs of the small kernels before it, so the GEMM's CTAs become
 *     resident, and start streaming weights, while those still run. */
#define DCU_OPT_GEMM_SMEM_KB 4
/*   DCU_OPT_GEMM_PASS_SWEEP (0 or 1, default 1): a layer GEMM multiplies its
 *     rows in token passes of 128 rows (small expected recompute sets) or 256
 *     (larger ones, and the dense forward); the LM head of a commit takes the
 *     masked rows 256 at a time.  With 256-row passes and more than one pass,
 *     1 multiplies each weight tile held in shared memory by two passes of
 *     activations, each into its own tensor-memory accumulator, so the
 *     weights stream from HBM once per two passes; 0 streams them once per
 *     pass.  Results are bit-identical either way. */
#define DCU_OPT_GEMM_PASS_SWEEP 5
#define DCU_ATTN_TCGEN05 0
#define DCU_ATTN_MMA_SYNC 1
int dcu_set_option(dcu_ctx *ctx, int32_t option, int32_t value);

/* Adaptive parallel decoding, APD ([DLLM] "关键设计 3").  Enables rule DCU_APD of
 * commit_select / commit_select_block: at every such commit, for each
 * candidate position i (masked, in the open block),
 *   c_i = 1 - (second-highest probability of its LM-head distribution),
 *   H_i = 1 - cos(p_i, p_i^prev), p^prev its distribution at the previous APD
 *         commit (H_i = 0 the first time a position is a candidate),
 *   tau_i <- tau_i - alpha c_i + beta H_i     (fp64, stored float32),
 * then every candidate with confidence >= tau_i is committed (descending
 * confidence), or the most confident one when none is.  The pages leave
 * alpha, beta >= 0 open and start tau near 0.9, so all three are parameters.
 * tau resets to tau0 and the history is cleared here and at every
 * dcu_full_forward.  Allocates the logits of two commits, 2 x max_batch x
 * max_seq x vocab floats, the first time (DCU_ENOMEM); synchronises the
 * device; not inside a stream capture (DCU_ESTATE).  DCU_EINVAL for negative
 * or non-finite alpha / beta or non-finite tau0.  Thresholds and signals:
 * DCU_T_APD_TAU, DCU_T_APD_C, DCU_T_APD_H. */
int dcu_set_apd(dcu_ctx *ctx, float alpha, float beta, float tau0);

/* Feature source of the token dynamics d ([README] "Quick Start":
 * select_from; [DLLM] "关键设计 1" contrasts the layer-input proxy with
 * recomputing and comparing the Value vectors).  DCU_SELECT_INPUT (default):
 * d compares the normalised layer inputs.  DCU_SELECT_VALUE: per layer, for
 * every row whose layer input was rewritten with a different value since the
 * layer last recomputed that row ("stale"; DCU_T_STALE), the Value
 * W_v RMSNorm(x) is recomputed, rounded to the cache dtype and compared with
 * the cached Value row over all kv heads, d = 1 - cos; every other row has
 * d = 0 (its input, hence its Value, is unchanged).  This costs a compaction,
 * a gather + RMSNorm, a W_v GEMM over the stale rows and a distance kernel per
 * layer.  Stale flags are kept in both modes.  Takes effect from the next
 * dcu_step; DCU_EINVAL for another value. */
int dcu_set_select_from(dcu_ctx *ctx, int32_t source);

/* Periodic full refresh ([README] "Quick Start": prompt_interval_steps,
 * gen_interval_steps; the pages name the parameters, not their semantics, so
 * this is the reading taken): counting the DCU steps after the last
 * dcu_full_forward as 1, 2, ..., a step whose number is a multiple of
 * prompt_interval forces every prompt position [0, gen_start) into the
 * recompute set U of every layer, and a multiple of gen_interval every
 * generated position [gen_start, N) (both: a dense recompute).  Forced
 * positions join the window: the top-B budget is spent outside them, and d, s
 * and the next step's budgets are computed as on any step.  0 disables an
 * interval (the default: no refresh).  gen_start is clamped to N.  Takes
 * effect from the next dcu_step; DCU_EINVAL for negative arguments. */
int dcu_set_refresh(dcu_ctx *ctx, int32_t gen_start, int32_t prompt_interval, int32_t gen_interval);

/* Per-step commit ([FRECHET] "整体框架"): final RMSNorm + LM head on the
 * masked positions of H_L only, fused softmax giving the max-probability
 * confidence c and the argmax (lowest id on ties), then dcu_commit_rule.
 * masked: dev uint8 [B][N] (1 = masked), cleared at committed positions;
 * token_ids: dev int32 [B][N], committed positions set to their argmax;
 * out_positions: dev int32 [B][N], row b starts with the out_count[b]
 * committed positions in descending confidence; out_count: dev int32 [B]. */
int commit_select(dcu_ctx *ctx, int32_t rule, float param, uint8_t *masked, int32_t *token_ids,
                  int32_t *out_positions, int32_t *out_count, dcu_stream_t stream);

/* commit_select under the block-wise schedule ([README] "Quick Start":
 * generate_mode "default", fixed-schedule block-wise decoding; [FRECHET]
 * "实验关键数据": block size 32): per sequence, the positions from gen_start on
 * are cut into consecutive blocks of block_len and only the masked positions
 * of the leftmost block that still holds one are candidates (LM head and
 * rule both); a sequence with no masked position at or after gen_start
 * commits nothing.  block_len <= 0 is commit_select.  gen_start must lie in
 * [0, N) when block_len > 0 (DCU_EINVAL otherwise). */
int commit_select_block(dcu_ctx *ctx, int32_t rule, float param, int32_t gen_start, int32_t block_len,
                        uint8_t *masked, int32_t *token_ids, int32_t *out_positions, int32_t *out_count,
                        dcu_stream_t stream);

/* dcu_step and commit_select are captured into CUDA graphs (once per distinct
 * set of pointers, budgets and active shape; at most 16 kept, least recently
 * used evicted) and replayed on the caller's stream.  on = 0 launches every
 * kernel directly instead.  Default: on. */
int dcu_set_graphs(dcu_ctx *ctx, int32_t on);

/* Synchronises the stream, returns DCU_EDEVICE if the device status word is
 * non-zero (its bits in *bits when bits is not NULL) and clears it. */
int dcu_status(dcu_ctx *ctx, dcu_stream_t stream, int32_t *bits);

/* ---- stateless kernels (no context) ---- */

/* Layer budgets of [DLLM] "关键设计 1" for B sequences: s_prev dev float [B][L]
 * -> budgets dev int32 [B][L], each row summing to B_layer * L exactly
 * (fp64, floor + largest remainder, ties to the lower layer; uniform when
 * `uniform` != 0 or the row sums to 0). */
int dcu_budget_split(const float *s_prev, int32_t B, int32_t L, int32_t B_layer, int32_t uniform,
                     int32_t *budgets, dcu_stream_t stream);

/* Token selection of one layer ([DLLM] "关键设计 1" top-B by d, "关键设计 2"
 * forced window): for each sequence b, s[b] = mean of d[b][0..N) and
 * idx[b][0..count[b]) = sorted U = W union top-budgets[b] (by d descending,
 * then index ascending) outside W.  d: dev float [B][N] (>= 0);
 * key_positions: dev int32 [B][N]; n_keys, budgets: dev int32 [B];
 * outputs dev: idx int32 [B][N], count int32 [B], s float [B]; status: dev
 * int32 or NULL (DCU_ST_BAD_KEY).  N <= 16384. */
int dcu_select_tokens(const float *d, const int32_t *key_positions, const int32_t *n_keys, const int32_t *budgets,
                      int32_t B, int32_t N, int32_t B_window, int32_t window_mode, int32_t *idx, int32_t *count,
                      float *s, int32_t *status, dcu_stream_t stream);

/* Token dynamics of [DLLM] "关键设计 1" on `rows` row pairs:
 * d[r] = 1 - <g*x_r, g*y_r> / (|g*x_r| |g*y_r|) in fp64, 0 for bitwise-equal
 * rows, 1 if exactly one row is zero, clamped to [0, 2].  x, y: dev [rows][D]
 * in dtype; gain: dev float [D]; d: dev float [rows].  D % 8 == 0. */
int dcu_cosine_distance(const void *x, const void *y, const float *gain, int64_t rows, int32_t D, int32_t dtype,
                        float *d, dcu_stream_t stream);

/* Commit rule alone (the drop-in selector of [FRECHET] "整体框架"; rules
 * DCU_FRECHET, DCU_THRESHOLD, DCU_FACTOR -- DCU_APD needs a context): per
 * sequence, sorts the masked positions by conf (descending, ties to the lower
 * position) and commits n* of them by `rule` (param = delta | tau | f; fp64
 * prefix sums).  conf: dev float [B][N]; argmax: dev int32 [B][N];
 * masked, token_ids, out_positions, out_count as in commit_select.  N <= 16384. */
int dcu_commit_rule(int32_t rule, float param, const float *conf, const int32_t *argmax, uint8_t *masked,
                    int32_t *token_ids, int32_t B, int32_t N, int32_t *out_positions, int32_t *out_count,
                    dcu_stream_t stream);

/* Self-test of the device-side failure detection (the pages have no
 * counterpart): launches one CTA whose thread waits on an mbarrier that nothing
 * arrives on.  The bounded wait gives up after its wall-clock limit (about 1 s)
 * and ORs DCU_ST_TIMEOUT into *status (dev int32, caller-zeroed); bit 30 would
 * mean the wait wrongly succeeded, bit 29 that the expiry did not raise the
 * CTA's abort flag.  The kernel always finishes; the context stays usable. */
int dcu_selftest_wait_timeout(int32_t *status, dcu_stream_t stream);

/* dcu_commit_rule restricted to each sequence's open block (as in
 * commit_select_block; block_len <= 0: no restriction). */
int dcu_commit_rule_block(int32_t rule, float param, int32_t gen_start, int32_t block_len, const float *conf,
                          const int32_t *argmax, uint8_t *masked, int32_t *token_ids, int32_t B, int32_t N,
                          int32_t *out_positions, int32_t *out_count, dcu_stream_t stream);

/* Y[m][n] = sum_k X[m][k] W[n][k] in fp32: the recompute GEMM (tcgen05 with
 * TMA-staged operands for bf16, CUDA cores for float32) as a stateless call.
 * X: dev [M][K] dtype; W: dev [Nout][K] dtype; Y: dev float [M][Nout]; all
 * 16-byte aligned; K % 64 == 0 (bf16) or K % 16 == 0 (float32). */
int dcu_linear(const void *X, const void *W, int32_t M, int32_t K, int32_t Nout, int32_t dtype, float *Y,
               dcu_stream_t stream);

/* LM-head confidence and argmax of m final-layer rows without any device
 * allocation, for callers that cannot call cudaMalloc (a host framework that
 * owns every device allocation through its own pool, or a serving process
 * whose allocator is frozen).  The pages have no counterpart to this call: it
 * is the LM-head stage of commit_select (final RMSNorm, logits, max softmax
 * probability, lowest-id argmax) as a stateless function.
 * h_rows: dev [m][D] in dtype; final_norm: dev float [D]; lm_head: dev
 * [V][D] in dtype; conf: dev float [m]; argmax: dev int32 [m].
 * Scratch is one static device array of about 12 MB inside libdcu, held by
 * every GPU that loads the library until the process exits; the call
 * allocates nothing.  The first call on a device takes the array's address
 * (cudaGetSymbolAddress) with that device current, so make that first call
 * before any stream capture.  Calls share the array: calls that overlap on
 * the GPU (other streams, other host threads) race and must be serialised by
 * the caller.  Limits: m <= 256 and D <= 8192 (DCU_ECAPACITY beyond),
 * D % 64 == 0 (DCU_EINVAL). */
int dcu_lm_confidence_noalloc(const void *h_rows, const float *final_norm, const void *lm_head, int32_t m,
                              int32_t D, int32_t V, int32_t dtype, float rms_eps, float *conf, int32_t *argmax,
                              dcu_stream_t stream);

/* ---- introspection (tests, teacher forcing) ---- */

#define DCU_T_H         0  /* layer 0..L   : [B][N][d_model] dtype        */
#define DCU_T_K         1  /* layer 0..L-1 : [B][n_kv_heads][N][head_dim] dtype */
#define DCU_T_V         2  /* layer 0..L-1 : same as K                    */
#define DCU_T_D         3  /* layer 0..L-1 : [B][N] float, input dynamics d of the layer in the last step */
#define DCU_T_S         4  /* [B][L] float, s of the last step            */
#define DCU_T_S_PREV    5  /* [B][L] float, s the next step splits by     */
#define DCU_T_BUDGET    6  /* [B][L] int32, budgets of the last step      */
#define DCU_T_SEL       7  /* layer 0..L-1 : [B][N] int32, row b: the selected positions, sorted */
#define DCU_T_SEL_COUNT 8  /* layer 0..L-1 : [B] int32                    */
#define DCU_T_CONF      9  /* [B][N] float, confidence of the last commit (masked positions) */
#define DCU_T_ARGMAX   10  /* [B][N] int32, argmax of the last commit (masked positions)      */
#define DCU_T_STALE    12  /* layer 0..L-1 : [B][N] uint8, 1 = the H_l row was rewritten with a new
                              value since layer l last recomputed it (settable) */
#define DCU_T_APD_TAU  13  /* [B][N] float: APD thresholds tau (after dcu_set_apd)           */
#define DCU_T_APD_C    14  /* [B][N] float: APD concentration c of the last APD commit      */
#define DCU_T_APD_H    15  /* [B][N] float: APD instability H of the last APD commit        */
#define DCU_T_ATTN     11  /* [B*N][n_heads*head_dim] dtype: attention output of the rows the
                              most recent layer recomputed (layer L-1 after dcu_step or
                              dcu_full_forward), packed sequence by sequence in ascending
                              position; the first sum_b SEL_COUNT[b] rows (B*N after a dense
                              forward) are defined, the rest are scratch */

/* Size in bytes of a tensor kind for the active (B, N). */
int dcu_tensor_bytes(const dcu_ctx *ctx, int32_t kind, int64_t *bytes);
/* Device-to-device copy of a tensor kind into dst (dev, `bytes` long). */
int dcu_get_tensor(dcu_ctx *ctx, int32_t kind, int32_t layer, void *dst, int64_t bytes, dcu_stream_t stream);
/* Device-to-device copy from src into a tensor kind (H, K, V, S_PREV, STALE only). */
int dcu_set_tensor(dcu_ctx *ctx, int32_t kind, int32_t layer, const void *src, int64_t bytes, dcu_stream_t stream);

/* ---- per-kernel timing (CUDA events on the launch stream) ---- */

#define DCU_K_REFRESH   0  /* layer-0 input refresh + d^0            */
#define DCU_K_BUDGET    1  /* budget split                           */
#define DCU_K_SELECT    2  /* window + top-B + compaction + s         */
#define DCU_K_GATHER    3  /* row gather + RMSNorm                    */
#define DCU_K_GEMM      4  /* recompute GEMMs (QKV, O, gate/up, down) */
#define DCU_K_EPILOGUE  5  /* GEMM epilogues (RoPE/KV write, residual+norm, SwiGLU) */
#define DCU_K_ATTN      6  /* attention of the selected queries       */
#define DCU_K_SCATTER   7  /* scatter into H_{l+1} + next-layer d     */
#define DCU_K_LMHEAD    8  /* LM head + softmax-max                   */
#define DCU_K_COMMIT    9  /* sort + rule + commit                    */
#define DCU_K_COUNT    10

/* Turns event timing of every launch on (max_launches per kernel class
 * between resets) or off (0). */
int dcu_profile_enable(dcu_ctx *ctx, int32_t max_launches);
/* Synchronises and returns the summed event time (ms) and launch count of a
 * kernel class since the last reset; reset != 0 clears the class afterwards.
 * Launches inside a graph are timed by event-record nodes of the graph's most
 * recent replay, counted once per replay; the replay counts are cleared when
 * the last class (DCU_K_COUNT - 1) is read with reset. */
int dcu_profile_read(dcu_ctx *ctx, int32_t kernel_class, double *total_ms, int64_t *launches, int32_t reset);
const char *dcu_kernel_class_name(int32_t kernel_class);
/* Number of kernels the context has launched since it was created. */
int64_t dcu_launch_count(const dcu_ctx *ctx);

#ifdef __cplusplus
}
#endif
#endif /* DCU_H */
