"""Test-side glue: builds the oracle's view of the seeded model and compares
GPU results with the oracle's."""
from __future__ import annotations

import numpy as np

import oracle as O
from dynamic_layer_wise_b200 import inputs as I


def oracle_cfg(shape: I.ModelShape, window_mode: int = 0) -> O.Config:
    return O.Config(n_layers=shape.n_layers, d_model=shape.d_model, n_heads=shape.n_heads,
                    n_kv_heads=shape.n_kv_heads, head_dim=shape.head_dim, d_ffn=shape.d_ffn, vocab=shape.vocab,
                    dtype=shape.dtype, rms_eps=shape.rms_eps, rope_theta=shape.rope_theta, window_mode=window_mode)


class LazyRows:
    """Row access to a seeded [vocab][d_model] matrix without materialising it."""

    def __init__(self, shape, seed, name):
        self.shape, self.seed, self.name = shape, seed, name
        self._cache = {}

    def __getitem__(self, rows):
        rows = np.atleast_1d(np.asarray(rows))
        out = np.empty((len(rows), self.shape.d_model))
        for j, r in enumerate(rows):
            r = int(r)
            if r not in self._cache:
                self._cache[r] = I.as_f64(I.weight_values(self.shape, self.seed, self.name, rows=[r])[0],
                                          self.shape.dtype)
            out[j] = self._cache[r]
        return out


class LazyMatrix:
    """Row-slice access to a seeded [rows][cols] weight matrix, generated on
    demand (for the LM head of the 8B shapes)."""

    def __init__(self, shape, seed, name, rows):
        self.spec, self.seed, self.name = shape, seed, name
        self.shape = (rows, shape.d_model)

    def __getitem__(self, sl):
        r0, r1, _ = sl.indices(self.shape[0])
        return I.as_f64(I.weight_rows(self.spec, self.seed, self.name, r0, r1), self.spec.dtype)


def oracle_weights(shape: I.ModelShape, seed: int, lazy_vocab: bool = False, layers=None) -> O.Weights:
    dt = shape.dtype

    def mat(name, l=None):
        return I.as_f64(I.weight_values(shape, seed, name, l), dt)

    ones = np.ones(shape.d_model)
    layer_ids = range(shape.n_layers) if layers is None else layers
    ls = {}
    for l in layer_ids:
        lw = {"attn_norm": ones, "ffn_norm": ones}
        for n in I.LAYER_TENSORS:
            lw[n] = mat(n, l)
        ls[l] = lw
    layer_list = [ls.get(l) for l in range(shape.n_layers)]
    if lazy_vocab:
        return O.Weights(embed=LazyRows(shape, seed, "embed"), lm_head=None, final_norm=ones, layers=layer_list)
    return O.Weights(embed=mat("embed"), lm_head=mat("lm_head"), final_norm=ones, layers=layer_list)


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64).ravel()
    b = np.asarray(b, dtype=np.float64).ravel()
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


def to_np(t):
    import torch
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.cpu().numpy()


def check_selection(sel_gpu, sel_ora, d_ora, keys, bw, budget, mode, N, eps=1e-5, force=None):
    """Selections must match except for indices whose oracle d lies within eps of
    the oracle's k-th boundary value (exact ties are decided by index on both
    sides, so they are not exempt).  Returns the exempt indices."""
    g, o = set(int(i) for i in sel_gpu), set(int(i) for i in sel_ora)
    if g == o:
        return []
    W = O.window_mask(keys, bw, N, mode)
    if force is not None:
        W[force[0]:force[1]] = True
    assert len(g) == len(o), f"selection sizes differ: {len(g)} vs {len(o)}"
    top_o = sorted(o - set(np.flatnonzero(W)), key=lambda i: (-float(d_ora[i]), i))
    boundary = float(d_ora[top_o[-1]]) if top_o else 0.0
    diff = sorted(g ^ o)
    bad = [i for i in diff if abs(float(d_ora[i]) - boundary) > eps]
    assert not bad, f"selection differs beyond the near-boundary exemption at {bad[:10]} (boundary {boundary})"
    return diff


def check_selection_valid(sel_gpu, d_gpu, keys, bw, budget, mode, N):
    """Property of the GPU selection against the GPU's own d (no oracle): it holds
    the whole window, has min(N, |W| + budget) rows, and every selected row
    outside the window ranks above every unselected one by (d desc, index asc)."""
    W = O.window_mask(keys, bw, N, mode)
    sel = np.zeros(N, bool)
    sel[np.asarray(sel_gpu, dtype=np.int64)] = True
    assert np.all(sel[W]), "a window row is not selected"
    assert sel.sum() == min(N, int(W.sum()) + int(budget)), "selection size"
    assert np.all(np.diff(np.asarray(sel_gpu)) > 0), "selection not sorted / has duplicates"
    top = np.flatnonzero(sel & ~W)
    rest = np.flatnonzero(~sel & ~W)
    if len(top) and len(rest):
        d = np.asarray(d_gpu, dtype=np.float32)
        worst_in = max(top, key=lambda i: (-float(d[i]), i))
        best_out = min(rest, key=lambda i: (-float(d[i]), i))
        assert (-float(d[worst_in]), worst_in) < (-float(d[best_out]), best_out), "top-B order violated"


def check_commit(pos_gpu, pos_ora, c_ora, masked, eps=1e-5):
    """Committed sets must match except positions whose oracle confidence is
    within eps of the cut (the confidence of the last committed position)."""
    g, o = list(pos_gpu), list(pos_ora)
    assert len(g) == len(o), f"commit counts differ: {len(g)} vs {len(o)}"
    if set(g) == set(o):
        return []
    cut = float(c_ora[o[-1]])
    diff = sorted(set(g) ^ set(o))
    bad = [p for p in diff if abs(float(c_ora[p]) - cut) > eps]
    assert not bad, f"commit differs beyond the near-boundary exemption at {bad}"
    return diff


# ---------------------------------------------------------------- teacher forcing

class LayerSnap:
    """Host copy (fp64) of what one layer of a DCU step read and wrote on the
    GPU: H_l and H_{l+1}, K_l and V_l before and after the step, and the
    layer's d, selection and counts after it."""

    def __init__(self, before, after, ctx, l, B, N, shape, dcu):
        D, Hkv, hd = shape.d_model, shape.n_kv_heads, shape.head_dim
        f64 = lambda t, *dims: np.asarray(to_np(t), dtype=np.float64).reshape(*dims)  # noqa: E731
        self.l = l
        self.H_old = f64(before[0][l], B, N, D)
        self.H_new = f64(after[0][l], B, N, D)
        self.Hn_old = f64(before[0][l + 1], B, N, D)
        self.Hn_new = f64(after[0][l + 1], B, N, D)
        self.K_old = f64(before[1][l], B, Hkv, N, hd)
        self.V_old = f64(before[2][l], B, Hkv, N, hd)
        self.K_new = f64(after[1][l], B, Hkv, N, hd)
        self.V_new = f64(after[2][l], B, Hkv, N, hd)
        self.d = dcu.dcu_get_tensor(ctx, dcu.DCU_T_D, l).cpu().numpy().reshape(B, N)
        self.sel = dcu.dcu_get_tensor(ctx, dcu.DCU_T_SEL, l).cpu().numpy().reshape(B, N)
        self.cnt = dcu.dcu_get_tensor(ctx, dcu.DCU_T_SEL_COUNT, l).cpu().numpy()


def teacher_forced_layer(snap, lw, cfg_o, s_gpu, budgets, keys, bw, mode, tol, attn_gpu=None, label="", force=None,
                         stale=None, d_atol=2e-7):
    """Per-layer parity with the oracle fed the GPU's own layer inputs (the
    spec parity contract): from the GPU's H_l before and after the step
    the oracle computes d (to 2e-7), s (to 1e-5 relative) and the selection
    with the GPU's budget (exact except indices within 1e-5 of the top-B
    boundary); from the GPU's selection, H_l and pre-step K_l / V_l it
    recomputes the rows, whose H_{l+1}, K_l and V_l must agree within the
    relative-L2 tolerance (and the attention output of the packed rows, when
    given).  Returns the number of exempt near-boundary indices."""
    B, N = snap.d.shape
    g = lw["attn_norm"]
    exempt = 0
    attn_rows, attn_ref = [], []
    for b in range(B):
        if stale is None:
            d_o = O.to_f32(O.cosine_distance(snap.H_new[b], snap.H_old[b], g))
        else:  # select_from = "v": the oracle's Value distance of the stale rows, from the GPU's inputs
            d_o = O.value_dynamics(lw, cfg_o, snap.H_new[b], snap.V_old[b], stale[b])
        err = float(np.max(np.abs(snap.d[b].astype(np.float64) - d_o.astype(np.float64))))
        assert err <= d_atol, f"{label} seq {b}: d differs by {err:.2e}"
        band = 1e-5 if stale is None else max(1e-5, err)
        s_o = O.layer_dynamics(d_o)
        # s is the mean of d: in Value mode its difference is bounded by d's (the Value rounding)
        s_tol = 1e-5 * abs(float(s_o)) + 1e-12 + (err if stale is not None else 0.0)
        assert abs(float(s_gpu[b]) - float(s_o)) <= s_tol, \
            f"{label} seq {b}: s {float(s_gpu[b])} vs oracle {float(s_o)}"
        U = snap.sel[b, :snap.cnt[b]].astype(np.int64)
        ref = O.select_rows(d_o, keys[b], bw, int(budgets[b]), mode, force)
        exempt += len(check_selection(U, ref, d_o, keys[b], bw, int(budgets[b]), mode, N, eps=band, force=force))
        if len(U) == 0:
            continue
        K, V = snap.K_old[b].copy(), snap.V_old[b].copy()
        tr = {}
        y = O.layer_rows(lw, cfg_o, snap.H_new[b][U], U, K, V, trace=tr)
        e = rel_l2(snap.Hn_new[b][U], y)
        assert e <= tol, f"{label} seq {b}: H_{snap.l + 1}[U] rel L2 {e:.3e} > {tol}"
        for name, gpu, o in (("K", snap.K_new[b], K), ("V", snap.V_new[b], V)):
            e = rel_l2(gpu[:, U, :], o[:, U, :])
            assert e <= tol, f"{label} seq {b}: {name}_{snap.l}[U] rel L2 {e:.3e} > {tol}"
        off = np.setdiff1d(np.arange(N), U)
        assert np.array_equal(snap.Hn_new[b][off], snap.Hn_old[b][off]), f"{label}: H_{snap.l + 1} changed off U"
        attn_rows.append(len(U))
        attn_ref.append(tr["attn"])
    if attn_gpu is not None and attn_ref:
        ref = np.concatenate(attn_ref)
        got = np.asarray(attn_gpu, dtype=np.float64)[:len(ref)]
        e = rel_l2(got, ref)
        assert e <= tol, f"{label}: attention output rel L2 {e:.3e} > {tol}"
    return exempt


def dense_layer_check(lw, cfg_o, H0, H1_gpu, K_gpu, V_gpu, sample, tol, label=""):
    """Dense forward, one layer, teacher-forced on the GPU's layer input H0
    ([B, N, D]): the oracle's K/V of every row and the layer output of the
    sampled rows (attending over the oracle's K/V of all rows)."""
    B, N, _ = H0.shape
    pos = np.arange(N)
    for b in range(B):
        K, V = O.kv_rows(lw, cfg_o, H0[b], pos)
        for name, gpu, o in (("K", K_gpu[b], K), ("V", V_gpu[b], V)):
            e = rel_l2(gpu, o)
            assert e <= tol, f"{label} seq {b}: dense {name} rel L2 {e:.3e} > {tol}"
        y = O.layer_rows(lw, cfg_o, H0[b][sample], sample, K.copy(), V.copy())
        e = rel_l2(H1_gpu[b][sample], y)
        assert e <= tol, f"{label} seq {b}: dense H_1 rel L2 {e:.3e} > {tol}"
