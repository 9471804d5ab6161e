"""Plain fp64 CPU oracle of the Dynamic Cache Updating (DCU) step and its commit.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this
module: only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline leg use it.  It shares no code with the CUDA path.

Every function states the passage it follows.  Sources (web pages):

* [DLLM] "Dynamic-dLLM: Dynamic Cache-Budget and Adaptive Parallel Decoding for
  Training-Free Acceleration of Diffusion LLM" (papernotes.org, ICLR 2026 note).
  Section "关键设计 1" (dynamic cache updating: cosine distance d, layer
  dynamics s, proportional budget), section "关键设计 2" (forced update window),
  section "研究背景与动机" (bidirectional attention, full recompute per step).
* [FRECHET] "Fast-dLLM++: Fréchet Profile Decoding for Faster Diffusion LLM
  Inference" (papernotes.org, ICML 2026 workshop note).  Section "研究背景与动机"
  (Fast-dLLM threshold and factor rules), "整体框架" (argmax + confidence,
  descending sort, drop-in selector), "关键设计 1" (Theorem 4.1: L_n, U_n, G_n),
  "关键设计 2" (n* = max{n : G_n > delta}, else 1), "关键设计 3"
  (Proposition 4.3 / Corollary 4.4: G_n = F_n + B_n).

Readings where the pages are silent (each also listed in the design notes):

* The model is a pre-norm bidirectional transformer: RMSNorm (gain g, eps),
  Q/K/V projections, rotate-half RoPE (theta = 10000; 0 disables it),
  unmasked softmax attention with scale 1/sqrt(head_dim), GQA head j -> kv head
  floor(j * H_kv / H), O projection + residual, RMSNorm, SwiGLU FFN + residual,
  final RMSNorm, LM head.  No biases.
* The layer caches H_l (layer l input = layer l-1 output) and K/V are *stored*
  in the model dtype (bf16 rounds to nearest even); everything else is fp64.
* d is computed on the RMSNorm-normalised inputs, i.e. on g*x (the RMS scale
  cancels in a cosine).  Bitwise-identical rows give d = 0 exactly; both zero
  -> 0; one zero -> 1; the value is clamped to [0, 2].
* Decisions are taken in the precision the product stores them in: d and the
  confidence c are rounded to float32 before any ranking; s is the fp64 mean of
  the float32 d values, rounded to float32.
* Budget split: floor + largest remainder (ties -> lower layer) in fp64;
  uniform (B_layer each) on the first cached step or when sum(s) = 0.
* Window: inclusive [p - floor(Bw/2), p + floor(Bw/2)] (mode 0, Bw+1 positions)
  or [p - floor(Bw/2), p - floor(Bw/2) + Bw) (mode 1, Bw positions), clipped
  to [0, N); Bw = 0 means no window.  Top-B is taken outside the window, then
  unioned: |U| = min(N, |W| + B).  Ties in d go to the lower index.
* Inside a layer the new K/V rows of U are written before attention.
* Confidence is the max softmax probability over the full vocabulary; argmax
  ties go to the lowest id.  Sort ties go to the lower position.  Threshold
  rule with no c >= tau commits the top one; factor rule with no passing n
  commits one.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

# ----------------------------------------------------------------- configuration


@dataclass
class Config:
    n_layers: int
    d_model: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    d_ffn: int
    vocab: int
    dtype: str = "bf16"         # storage dtype of the H and K/V caches: 'bf16' | 'f32'
    rms_eps: float = 1e-5
    rope_theta: float = 10000.0
    window_mode: int = 0

    @property
    def mask_id(self) -> int:
        return self.vocab - 1


def store(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round fp64 values to the storage dtype and return them as fp64."""
    x = np.asarray(x, dtype=np.float64)
    if dtype == "f32":
        return x.astype(np.float32).astype(np.float64)
    if dtype == "bf16":
        bits = np.ascontiguousarray(x).view(np.uint64)
        keep = np.uint64(0xFFFFE00000000000)          # sign, exponent, 7 mantissa bits
        half = np.uint64(1 << 44)
        low = bits & np.uint64((1 << 45) - 1)
        lsb = (bits >> np.uint64(45)) & np.uint64(1)
        up = (low > half) | ((low == half) & (lsb == np.uint64(1)))
        with np.errstate(over="ignore"):
            out = (bits & keep) + np.where(up, np.uint64(1 << 45), np.uint64(0))
        return out.view(np.float64).copy()
    raise ValueError(dtype)


def to_f32(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float32)


# ----------------------------------------------------------------- model pieces

def rmsnorm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * g."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * g


def rope(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half rotary embedding.  x: [M, heads, hd]; pos: [M] integer positions.

    Pair (j, j + hd/2) is rotated by the angle pos * theta^(-2j/hd).
    """
    if theta == 0.0:
        return x
    hd = x.shape[-1]
    half = hd // 2
    inv = theta ** (-(2.0 * np.arange(half, dtype=np.float64)) / hd)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * inv[None, :]      # [M, half]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def softmax_rows(z: np.ndarray) -> np.ndarray:
    z = z - np.max(z, axis=-1, keepdims=True)
    e = np.exp(z)
    return e / np.sum(e, axis=-1, keepdims=True)


def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray) -> np.ndarray:
    """Bidirectional (unmasked) attention of queries over all cached keys.

    q: [M, H, hd]; K, V: [H_kv, N, hd] -> [M, H, hd].  Scale 1/sqrt(hd); query
    head h reads kv head floor(h * H_kv / H).  [DLLM] "研究背景与动机": the
    dLLM denoises with bidirectional attention over the whole sequence.
    """
    M, H, hd = q.shape
    Hkv = K.shape[0]
    out = np.empty_like(q)
    for h in range(H):
        kvh = (h * Hkv) // H
        p = softmax_rows(q[:, h, :] @ K[kvh].T / math.sqrt(hd))
        out[:, h, :] = p @ V[kvh]
    return out


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def ffn(m: np.ndarray, lw: dict) -> np.ndarray:
    """SwiGLU: W_down (silu(W_gate m) * (W_up m))."""
    return (silu(m @ lw["w_gate"].T) * (m @ lw["w_up"].T)) @ lw["w_down"].T


# ----------------------------------------------------------------- weights

@dataclass
class Weights:
    """fp64 weights.  ``embed``/``lm_head`` must support row indexing; ``layers[l]``
    is a dict with attn_norm, wq, wk, wv, wo, ffn_norm, w_gate, w_up, w_down
    (matrices row-major [out][in])."""
    embed: object
    lm_head: object
    final_norm: np.ndarray
    layers: object


# ----------------------------------------------------------------- dense full forward

@dataclass
class State:
    """Per-sequence caches.  H[l]: [B, N, D] for l = 0..L; K[l], V[l]: [B, Hkv, N, hd]."""
    H: list
    K: list
    V: list
    ids: np.ndarray                # [B, N] ids the caches were built for
    s_prev: np.ndarray             # [B, L] float32 values of the previous step's s
    first: bool = True             # no previous-step s yet -> uniform split
    stale: list = None             # stale[l]: [B, N] bool, H_l row rewritten since layer l last recomputed it

    def copy(self) -> "State":
        return State([h.copy() for h in self.H], [k.copy() for k in self.K], [v.copy() for v in self.V],
                     self.ids.copy(), self.s_prev.copy(), self.first,
                     None if self.stale is None else [x.copy() for x in self.stale])


def full_forward(w: Weights, cfg: Config, ids: np.ndarray) -> State:
    """Dense forward over every position: the cost DCU avoids ([DLLM]
    "研究背景与动机": every denoising step recomputes all tokens).  Fills H_0..H_L
    and the post-RoPE K/V caches of every layer."""
    ids = np.asarray(ids, dtype=np.int64)
    B, N = ids.shape
    L, D, H, Hkv, hd = cfg.n_layers, cfg.d_model, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    Hs = [np.zeros((B, N, D)) for _ in range(L + 1)]
    Ks = [np.zeros((B, Hkv, N, hd)) for _ in range(L)]
    Vs = [np.zeros((B, Hkv, N, hd)) for _ in range(L)]
    pos = np.arange(N)
    for b in range(B):
        Hs[0][b] = store(np.asarray(w.embed[ids[b]], dtype=np.float64), cfg.dtype)
    for l in range(L):
        lw = w.layers[l]
        for b in range(B):
            x = Hs[l][b]
            n = rmsnorm(x, lw["attn_norm"], cfg.rms_eps)
            q = rope((n @ lw["wq"].T).reshape(N, H, hd), pos, cfg.rope_theta)
            k = rope((n @ lw["wk"].T).reshape(N, Hkv, hd), pos, cfg.rope_theta)
            v = (n @ lw["wv"].T).reshape(N, Hkv, hd)
            Ks[l][b] = store(k.transpose(1, 0, 2), cfg.dtype)
            Vs[l][b] = store(v.transpose(1, 0, 2), cfg.dtype)
            a = attend(q, Ks[l][b], Vs[l][b]).reshape(N, H * hd)
            h = x + a @ lw["wo"].T
            y = h + ffn(rmsnorm(h, lw["ffn_norm"], cfg.rms_eps), lw)
            Hs[l + 1][b] = store(y, cfg.dtype)
    return State(Hs, Ks, Vs, ids.copy(), np.zeros((B, L), dtype=np.float32), True,
                 [np.zeros((B, N), dtype=bool) for _ in range(L)])


# ----------------------------------------------------------------- DCU pieces

def cosine_distance(x: np.ndarray, y: np.ndarray, g: np.ndarray) -> np.ndarray:
    """Token dynamics, [DLLM] "关键设计 1", the cosine-distance equation:
    d = 1 - <x', y'> / (|x'| |y'|) between the normalised layer inputs of the
    current step (x) and the cached previous step (y), here x' = g*x, y' = g*y.
    x, y: [n, D] -> d: [n] fp64."""
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    y = np.atleast_2d(np.asarray(y, dtype=np.float64))
    out = np.zeros(x.shape[0])
    for r in range(x.shape[0]):
        if np.array_equal(x[r], y[r]):
            out[r] = 0.0
            continue
        a, b = g * x[r], g * y[r]
        na, nb = math.sqrt(float(a @ a)), math.sqrt(float(b @ b))
        if na == 0.0 and nb == 0.0:
            out[r] = 0.0
        elif na == 0.0 or nb == 0.0:
            out[r] = 1.0
        else:
            out[r] = min(2.0, max(0.0, 1.0 - float(a @ b) / (na * nb)))
    return out


def value_dynamics(lw: dict, cfg: Config, x: np.ndarray, V: np.ndarray, stale: np.ndarray) -> np.ndarray:
    """Token dynamics with select_from = "v" ([README] "Quick Start": the
    feature source of the similarity is the Value; [DLLM] "关键设计 1" contrasts
    the input proxy with recomputing the Value vectors and comparing their
    cosine similarity).  Reading: for every row whose layer input changed since
    this layer last recomputed it (``stale``), the Value is recomputed from the
    current input x (W_v RMSNorm(x), rounded as the cache stores it) and
    compared with the cached Value row over all kv heads: d = 1 - cos(v_new,
    v_cached) with the zero / equal-row rules of cosine_distance.  Every other
    row has an unchanged input, hence an unchanged Value, and d = 0.
    x: [N, D] layer inputs; V: [Hkv, N, hd] cached values; -> float32 [N]."""
    N = x.shape[0]
    d = np.zeros(N)
    idx = np.flatnonzero(np.asarray(stale, dtype=bool))
    if len(idx):
        _, v = kv_rows(lw, cfg, x[idx], idx)
        vn = v.transpose(1, 0, 2).reshape(len(idx), -1)
        vc = V[:, idx, :].transpose(1, 0, 2).reshape(len(idx), -1)
        d[idx] = cosine_distance(vn, vc, np.ones(vn.shape[1]))
    return to_f32(d)


def layer_dynamics(d32: np.ndarray) -> np.float32:
    """Layer dynamics s = (1/N) sum_i d_i ([DLLM] "关键设计 1"), on the float32
    d values, summed in fp64 and rounded to float32."""
    d = np.asarray(d32, dtype=np.float32).astype(np.float64)
    total = 0.0
    for v in d:
        total += float(v)
    return np.float32(total / len(d)) if len(d) else np.float32(0.0)


def split_budget(s_prev: np.ndarray, B_layer: int, uniform: bool) -> np.ndarray:
    """Per-layer budget, [DLLM] "关键设计 1", the budget equation:
    B^l = (B_layer * LayerNum) * s^{prev,l} / sum_k s^{prev,k}.

    Rounded by floor + largest remainder so the shares sum to B_layer * L
    exactly (ties -> lower layer); computed in fp64 from the float32 s values,
    the sum taken in layer order.  Uniform (B_layer each) when there is no
    previous step or the dynamics sum to zero.  If rounding of q made the
    floors overshoot the total, one is taken back from the layers with the
    smallest fractional parts (ties -> higher layer) among those above zero.
    """
    s = np.asarray(s_prev, dtype=np.float32).astype(np.float64)
    L = len(s)
    T = int(B_layer) * L
    total = 0.0
    for v in s:
        total += float(v)
    if uniform or total == 0.0:
        return np.full(L, int(B_layer), dtype=np.int64)
    q = [float(T) * float(v) / total for v in s]
    fl = [int(math.floor(v)) for v in q]
    frac = [q[l] - fl[l] for l in range(L)]
    R = T - sum(fl)
    out = list(fl)
    if R > 0:
        for l in sorted(range(L), key=lambda l: (-frac[l], l))[:R]:
            out[l] += 1
    elif R < 0:
        cand = [l for l in range(L) if fl[l] > 0]
        for l in sorted(cand, key=lambda l: (frac[l], -l))[:(-R)]:
            out[l] -= 1
    return np.array(out, dtype=np.int64)


def window_mask(keys, B_window: int, N: int, mode: int = 0) -> np.ndarray:
    """Forced update window, [DLLM] "关键设计 2", the window-union equation:
    every position i with p - B_w/2 <= i <= p + B_w/2 around each key token p
    (a token unmasked at the previous step) is updated whatever the budget."""
    W = np.zeros(N, dtype=bool)
    if B_window <= 0:
        return W
    h = B_window // 2
    for p in keys:
        p = int(p)
        lo = p - h
        hi = p + h if mode == 0 else p - h + B_window - 1
        lo, hi = max(lo, 0), min(hi, N - 1)
        if lo <= hi:
            W[lo:hi + 1] = True
    return W


def top_outside(d32: np.ndarray, W: np.ndarray, k: int) -> np.ndarray:
    """The k indices outside the window with the largest d ([DLLM] "关键设计 1":
    each layer recomputes its top-B tokens by d; "关键设计 2": the remaining
    budget is spent outside the window).  Ties go to the lower index."""
    cand = np.flatnonzero(~W)
    d = np.asarray(d32, dtype=np.float32)[cand].astype(np.float64)
    order = np.lexsort((cand, -d))           # primary: d descending; secondary: index ascending
    return np.sort(cand[order[:k]])


def select_rows(d32: np.ndarray, keys, B_window: int, budget: int, mode: int = 0, force=None) -> np.ndarray:
    """U = W  union  top-B outside W, as sorted row indices.  ``force`` = (lo, hi)
    adds the positions [lo, hi) to W (a periodic refresh, see refresh_range):
    they are recomputed whatever the budget, which is then spent outside them."""
    N = len(d32)
    W = window_mask(keys, B_window, N, mode)
    if force is not None:
        W[max(0, int(force[0])):max(0, min(N, int(force[1])))] = True
    k = int(min(max(int(budget), 0), N - int(W.sum())))
    U = W.copy()
    U[top_outside(d32, W, k)] = True
    return np.flatnonzero(U)


def refresh_range(step: int, gen_start: int, N: int, prompt_interval: int, gen_interval: int):
    """Periodic full refresh ([README] "Quick Start": prompt_interval_steps and
    gen_interval_steps; the function name _compute_sim_for_budget_full_refresh
    in the code index).  Reading: DCU step ``step`` (1, 2, ... after the dense
    forward) recomputes every prompt position [0, gen_start) when
    prompt_interval > 0 divides it, and every generated position
    [gen_start, N) when gen_interval > 0 divides it; d and s are still computed,
    so the next step's budgets follow this step.  Returns the forced range
    (lo, hi), or None when no refresh is due."""
    p = prompt_interval > 0 and step % prompt_interval == 0
    g = gen_interval > 0 and step % gen_interval == 0
    if p and g:
        return 0, N
    if p:
        return 0, gen_start
    if g:
        return gen_start, N
    return None


def kv_rows(lw: dict, cfg: Config, x: np.ndarray, pos: np.ndarray):
    """Keys and values of the given layer-input rows, as the cache stores them:
    k = RoPE(W_k RMSNorm(x)) at the rows' positions, v = W_v RMSNorm(x).
    Returns (k, v), each [Hkv, M, hd], rounded to the storage dtype."""
    M = x.shape[0]
    Hkv, hd = cfg.n_kv_heads, cfg.head_dim
    n = rmsnorm(x, lw["attn_norm"], cfg.rms_eps)
    k = rope((n @ lw["wk"].T).reshape(M, Hkv, hd), pos, cfg.rope_theta)
    v = (n @ lw["wv"].T).reshape(M, Hkv, hd)
    return store(k.transpose(1, 0, 2), cfg.dtype), store(v.transpose(1, 0, 2), cfg.dtype)


def layer_rows(lw: dict, cfg: Config, x: np.ndarray, pos: np.ndarray, K: np.ndarray, V: np.ndarray,
               trace: dict | None = None) -> np.ndarray:
    """Recompute the selected rows through one layer, reusing every other row's
    cached K/V ([DLLM] "关键设计 1": only the top tokens are recomputed, the rest
    reuse their cache).  K, V ([Hkv, N, hd]) are updated in place with the new
    rows (written before attention).  Returns the new layer outputs, stored.
    When ``trace`` is a dict it receives the attention output ('attn',
    [M, H*hd], fp64) for checks of that stage alone."""
    M = x.shape[0]
    H, hd = cfg.n_heads, cfg.head_dim
    n = rmsnorm(x, lw["attn_norm"], cfg.rms_eps)
    q = rope((n @ lw["wq"].T).reshape(M, H, hd), pos, cfg.rope_theta)
    K[:, pos, :], V[:, pos, :] = kv_rows(lw, cfg, x, pos)
    a = attend(q, K, V).reshape(M, H * hd)
    if trace is not None:
        trace["attn"] = a
    h = x + a @ lw["wo"].T
    y = h + ffn(rmsnorm(h, lw["ffn_norm"], cfg.rms_eps), lw)
    return store(y, cfg.dtype)


@dataclass
class StepTrace:
    budgets: np.ndarray                      # [B, L]
    d: list = field(default_factory=list)    # d[l]: [B, N] float32 (layer l input dynamics)
    s: np.ndarray = None                     # [B, L] float32
    sel: list = field(default_factory=list)  # sel[l][b]: sorted int array


def dcu_step(w: Weights, cfg: Config, state: State, ids: np.ndarray, keys: list, B_layer: int,
             B_window: int, force=None, select_from: str = "input") -> tuple[State, StepTrace]:
    """One cached denoising step (the DCU procedure of [DLLM] "关键设计 1/2").

    1. Layer-0 inputs of positions whose id changed are replaced by their
       embeddings; d^0 compares them with the cached rows.
    2. For each layer l: s^l = mean d^l; U^l = window union top-B^l (B^l from
       the previous step's s); the rows of U^l are recomputed and scattered
       into H_{l+1}; d^{l+1} is their distance to the cached H_{l+1} rows and 0
       elsewhere ("关键设计 2": an unselected token feeds the next layer an
       unchanged input, so its next-layer d is 0).
    3. The step's s becomes the previous-step s of the next step.
    ``force`` = (lo, hi) forces the positions [lo, hi) into every layer's U
    (periodic refresh, see refresh_range).  ``select_from`` = "v" ranks the
    rows by value_dynamics instead of the input distance; the stale flags it
    needs are kept in either mode (set where a write changes an H_l row, cleared
    where layer l recomputes it).
    """
    st = state.copy()
    ids = np.asarray(ids, dtype=np.int64)
    B, N = ids.shape
    L = cfg.n_layers
    budgets = np.stack([split_budget(st.s_prev[b], B_layer, st.first) for b in range(B)])
    tr = StepTrace(budgets=budgets, s=np.zeros((B, L), dtype=np.float32))
    d_cur = np.zeros((B, N), dtype=np.float32)
    if select_from not in ("input", "v"):
        raise ValueError(select_from)
    if st.stale is None:
        st.stale = [np.zeros((B, N), dtype=bool) for _ in range(L)]
    for b in range(B):
        ch = np.flatnonzero(ids[b] != st.ids[b])
        if len(ch):
            xn = store(np.asarray(w.embed[ids[b][ch]], dtype=np.float64), cfg.dtype)
            d_cur[b, ch] = to_f32(cosine_distance(xn, st.H[0][b][ch], w.layers[0]["attn_norm"]))
            st.stale[0][b][ch[np.any(xn != st.H[0][b][ch], axis=1)]] = True
            st.H[0][b][ch] = xn
    for l in range(L):
        if select_from == "v":
            d_cur = np.stack([value_dynamics(w.layers[l], cfg, st.H[l][b], st.V[l][b], st.stale[l][b])
                              for b in range(B)])
        tr.d.append(d_cur.copy())
        d_next = np.zeros((B, N), dtype=np.float32)
        sel_l = []
        for b in range(B):
            tr.s[b, l] = layer_dynamics(d_cur[b])
            U = select_rows(d_cur[b], keys[b], B_window, int(budgets[b, l]), cfg.window_mode, force)
            sel_l.append(U)
            if len(U) == 0:
                continue
            y = layer_rows(w.layers[l], cfg, st.H[l][b][U], U, st.K[l][b], st.V[l][b])
            st.stale[l][b][U] = False
            if l + 1 < L:
                d_next[b, U] = to_f32(cosine_distance(y, st.H[l + 1][b][U], w.layers[l + 1]["attn_norm"]))
                st.stale[l + 1][b][U[np.any(y != st.H[l + 1][b][U], axis=1)]] = True
            st.H[l + 1][b][U] = y
        tr.sel.append(sel_l)
        d_cur = d_next
    st.s_prev = tr.s.copy()
    st.first = False
    st.ids = ids.copy()
    return st, tr


# ----------------------------------------------------------------- commit

def logits(h_rows: np.ndarray, final_norm: np.ndarray, lm_head, eps: float, chunk: int = 16384) -> np.ndarray:
    """z = W_lm RMSNorm(h) for the given final-layer rows, fp64 [m, V]."""
    h = rmsnorm(np.atleast_2d(np.asarray(h_rows, dtype=np.float64)), final_norm, eps)
    V = lm_head.shape[0]
    z = np.empty((h.shape[0], V))
    for v0 in range(0, V, chunk):
        z[:, v0:v0 + chunk] = h @ np.asarray(lm_head[v0:v0 + chunk], dtype=np.float64).T
    return z


def confidence(h_rows: np.ndarray, final_norm: np.ndarray, lm_head, eps: float, chunk: int = 16384):
    """LM head on the given final-layer rows, softmax, max probability and argmax
    ([FRECHET] "整体框架": the argmax of every masked position and its
    confidence c_i).  c = 1 / sum_v exp(z_v - z_max); argmax ties -> lowest id.
    Returns (c as float32, argmax as int64)."""
    z = logits(h_rows, final_norm, lm_head, eps, chunk)
    zmax = np.max(z, axis=1)
    amax = np.argmax(z, axis=1)              # first maximum -> lowest id
    c = 1.0 / np.sum(np.exp(z - zmax[:, None]), axis=1)
    return to_f32(c), amax.astype(np.int64)


def frechet_count(c_sorted, delta: float) -> int:
    """Fréchet profile rule, [FRECHET] "关键设计 1" (Theorem 4.1) and "关键设计 2":
    L_n = max(0, sum_{j<=n} c_(j) - (n-1)), U_n = 1 - c_(n), G_n = L_n - U_n,
    n* = max{n : G_n > delta}, else 1 (progress is guaranteed).  fp64 on the
    float32 confidences sorted in descending order."""
    c = [float(v) for v in np.asarray(c_sorted, dtype=np.float32)]
    m = len(c)
    if m == 0:
        return 0
    best, S = 0, 0.0
    for n in range(1, m + 1):
        S += c[n - 1]
        Ln = max(0.0, S - float(n - 1))
        Un = 1.0 - c[n - 1]
        if Ln - Un > float(delta):
            best = n
    return best if best > 0 else 1


def frechet_profile(c_sorted):
    """(L_n, U_n, G_n) for n = 1..m, [FRECHET] "关键设计 1"."""
    c = [float(v) for v in c_sorted]
    Ls, Us, Gs, S = [], [], [], 0.0
    for n in range(1, len(c) + 1):
        S += c[n - 1]
        Ln = max(0.0, S - (n - 1))
        Un = 1.0 - c[n - 1]
        Ls.append(Ln)
        Us.append(Un)
        Gs.append(Ln - Un)
    return np.array(Ls), np.array(Us), np.array(Gs)


def threshold_count(c_sorted, tau: float) -> int:
    """Fast-dLLM threshold rule c_i >= tau ([FRECHET] "研究背景与动机"); with no
    passing position the top one is committed."""
    c = np.asarray(c_sorted, dtype=np.float32)
    if len(c) == 0:
        return 0
    n = int(np.sum(c >= np.float32(tau)))
    return max(n, 1)


def factor_count(c_sorted, f: float) -> int:
    """Fast-dLLM factor rule ([FRECHET] "研究背景与动机"): the largest n with
    (n + 1)(1 - c_(n)) < f, else 1.  fp64 on the float32 confidences."""
    c = [float(v) for v in np.asarray(c_sorted, dtype=np.float32)]
    if not c:
        return 0
    best = 0
    for n in range(1, len(c) + 1):
        if float(n + 1) * (1.0 - c[n - 1]) < float(f):
            best = n
    return best if best > 0 else 1


RULE_FRECHET, RULE_THRESHOLD, RULE_FACTOR, RULE_APD = 0, 1, 2, 3


# ----------------------------------------------------------------- APD (adaptive parallel decoding)

def apd_signals(z: np.ndarray, z_prev) -> tuple:
    """The two per-token signals of [DLLM] "关键设计 3", from the logits z [m, V]
    of this step and z_prev (the same positions' logits at the previous step,
    or None where a position has none, given as a list of arrays / None):

    * confidence concentration c = 1 - max_{v != u} p_v, u = argmax (the second
      highest probability; with a tie at the top it is the top probability);
    * temporal instability H = 1 - cos(p, p_prev) of the full probability
      vectors of adjacent steps; 0 for a position seen for the first time
      (reading: the page defines H from step t+1, which a first visit lacks).

    Returns (c, H) as fp64 arrays [m]."""
    z = np.atleast_2d(np.asarray(z, dtype=np.float64))
    m = z.shape[0]
    c = np.zeros(m)
    H = np.zeros(m)
    for i in range(m):
        p = softmax_rows(z[i][None])[0]
        top2 = np.sort(p)[-2:] if len(p) > 1 else np.array([0.0, p[0]])
        c[i] = 1.0 - top2[0]
        zp = None if z_prev is None else z_prev[i]
        if zp is not None:
            q = softmax_rows(np.asarray(zp, dtype=np.float64)[None])[0]
            H[i] = 1.0 - float(p @ q) / (math.sqrt(float(p @ p)) * math.sqrt(float(q @ q)))
    return c, H


def apd_update(tau, c, H, alpha: float, beta: float) -> np.ndarray:
    """[DLLM] "关键设计 3": tau_i^t = tau_i^{t+1} - alpha c_i^t + beta H_i^t, in fp64
    from the stored float32 thresholds, stored again as float32."""
    tau = np.asarray(tau, dtype=np.float32).astype(np.float64)
    return to_f32(tau - float(alpha) * np.asarray(c, dtype=np.float64) + float(beta) * np.asarray(H, dtype=np.float64))


def apd_commit(c, amax, masked, ids, tau, gen_start: int = 0, block_len: int = 0):
    """APD commit ("τ 满足则 unmask": a token is unmasked once its confidence
    reaches its own threshold): every candidate with c_i >= tau_i (float32),
    in descending confidence (ties -> lower position); none -> the top one (as
    the threshold rule, so decoding progresses).  Candidates as in commit().
    Returns (positions, new ids, new masked)."""
    masked = np.asarray(masked, dtype=bool)
    blk = active_block(masked, gen_start, block_len)
    open_ = np.zeros_like(masked)
    if blk is not None:
        open_[blk[0]:blk[1]] = True
    pos = np.flatnonzero(masked & open_)
    c32 = np.asarray(c, dtype=np.float32)
    order = pos[np.lexsort((pos, -c32[pos].astype(np.float64)))]
    t32 = np.asarray(tau, dtype=np.float32)
    chosen = np.array([i for i in order if c32[i] >= t32[i]], dtype=np.int64)
    if len(chosen) == 0 and len(order):
        chosen = order[:1]
    new_ids = np.array(ids, dtype=np.int64, copy=True)
    new_masked = masked.copy()
    new_ids[chosen] = np.asarray(amax)[chosen]
    new_masked[chosen] = False
    return chosen, new_ids, new_masked


def rule_count(rule: int, c_sorted, param: float) -> int:
    if rule == RULE_FRECHET:
        return frechet_count(c_sorted, param)
    if rule == RULE_THRESHOLD:
        return threshold_count(c_sorted, param)
    if rule == RULE_FACTOR:
        return factor_count(c_sorted, param)
    raise ValueError(rule)


def active_block(masked: np.ndarray, gen_start: int, block_len: int):
    """Block-wise schedule ([README] "Quick Start": generate_mode "default",
    fixed-schedule block-wise decoding; [FRECHET] "实验关键数据": block size 32):
    the generation region from gen_start is cut into consecutive blocks of
    block_len positions and only the leftmost block that still holds a masked
    position is open for commits.  Returns its [b0, b1), or None when no masked
    position is left at or after gen_start.  block_len <= 0: no blocks (the
    whole sequence is open)."""
    masked = np.asarray(masked, dtype=bool)
    N = masked.shape[0]
    if block_len <= 0:
        return 0, N
    left = np.flatnonzero(masked[gen_start:])
    if len(left) == 0:
        return None
    first = gen_start + int(left[0])
    b0 = gen_start + (first - gen_start) // block_len * block_len
    return b0, min(N, b0 + block_len)


def commit(c: np.ndarray, amax: np.ndarray, masked: np.ndarray, ids: np.ndarray, rule: int, param: float,
           gen_start: int = 0, block_len: int = 0):
    """Per-sequence commit ([FRECHET] "整体框架"): sort the masked positions by
    confidence (descending; ties -> lower position), take n* by the rule, set
    their ids to the argmax and unmask them.  With block_len > 0 only the
    masked positions of the active block (see active_block) are candidates.

    c, amax: [N] values at every position (only masked ones are read).
    Returns (positions in descending-confidence order, new ids, new masked)."""
    masked = np.asarray(masked, dtype=bool)
    blk = active_block(masked, gen_start, block_len)
    open_ = np.zeros_like(masked)
    if blk is not None:
        open_[blk[0]:blk[1]] = True
    pos = np.flatnonzero(masked & open_)
    cm = np.asarray(c, dtype=np.float32)[pos].astype(np.float64)
    order = pos[np.lexsort((pos, -cm))]
    n = rule_count(rule, np.asarray(c, dtype=np.float32)[order], param)
    chosen = order[:n]
    new_ids = np.array(ids, dtype=np.int64, copy=True)
    new_masked = masked.copy()
    new_ids[chosen] = np.asarray(amax)[chosen]
    new_masked[chosen] = False
    return chosen, new_ids, new_masked
