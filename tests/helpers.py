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


def check_selection(sel_gpu, sel_ora, d_ora, keys, bw, budget, mode, N, eps=1e-5):
    """Selections must match except for indices whose oracle d lies within eps of
    the oracle's k-th boundary value (exact ties are decided by index on both
    sides, so they are not exempt).  Returns the exempt indices."""
    g, o = set(int(i) for i in sel_gpu), set(int(i) for i in sel_ora)
    if g == o:
        return []
    W = O.window_mask(keys, bw, N, mode)
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
