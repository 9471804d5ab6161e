"""The teacher-forced comparison used by the GPU parity tests, checked on the
CPU: fed a DCU step computed by the oracle itself it must pass, and it must
fail when one recomputed K row, one output row, the attention output, a d
value or a selected index is wrong."""
import types

import numpy as np
import pytest

import oracle as O
from dynamic_layer_wise_b200 import inputs as I

from .helpers import oracle_cfg, oracle_weights, teacher_forced_layer

SHAPE = I.ModelShape(n_layers=2, d_model=64, n_heads=4, n_kv_heads=2, head_dim=16, d_ffn=128, vocab=97,
                     dtype="bf16")


def _oracle_step():
    seed, n_prompt, n_gen = 3, 40, 24
    N = n_prompt + n_gen
    cfg = oracle_cfg(SHAPE)
    w = oracle_weights(SHAPE, seed)
    ids = I.sequence_ids(seed, 0, n_prompt, n_gen, SHAPE.vocab)[None]
    st0 = O.full_forward(w, cfg, ids)
    pos, new = I.unmask_draw(seed, 0, np.arange(n_prompt, N), 3, SHAPE.vocab)
    ids1 = ids.copy()
    ids1[0, pos] = new
    st1, tr = O.dcu_step(w, cfg, st0, ids1, [list(pos)], 6, 4)
    return w, cfg, st0, st1, tr, [list(pos)]


def _snap(st0, st1, tr, l):
    sel = np.zeros((1, st0.H[0].shape[1]), np.int32)
    U = tr.sel[l][0]
    sel[0, :len(U)] = U
    return types.SimpleNamespace(l=l, H_old=st0.H[l].copy(), H_new=st1.H[l].copy(), Hn_old=st0.H[l + 1].copy(),
                                 Hn_new=st1.H[l + 1].copy(), K_old=st0.K[l].copy(), V_old=st0.V[l].copy(),
                                 K_new=st1.K[l].copy(), V_new=st1.V[l].copy(), d=tr.d[l].copy(), sel=sel,
                                 cnt=np.array([len(U)], np.int32))


def _attn(w, cfg, st0, st1, tr, l):
    U = tr.sel[l][0]
    t = {}
    O.layer_rows(w.layers[l], cfg, st1.H[l][0][U], U, st0.K[l][0].copy(), st0.V[l][0].copy(), trace=t)
    return t["attn"]


def test_teacher_forcing_accepts_the_oracle_step():
    w, cfg, st0, st1, tr, keys = _oracle_step()
    for l in range(SHAPE.n_layers):
        sn = _snap(st0, st1, tr, l)
        ex = teacher_forced_layer(sn, w.layers[l], cfg, tr.s[:, l], tr.budgets[:, l], keys, 4, 0, 1e-9,
                                  attn_gpu=_attn(w, cfg, st0, st1, tr, l))
        assert ex == 0


@pytest.mark.parametrize("fault", ["K", "H", "attn", "d", "sel"])
def test_teacher_forcing_rejects_a_planted_error(fault):
    w, cfg, st0, st1, tr, keys = _oracle_step()
    l = 1
    sn = _snap(st0, st1, tr, l)
    attn = _attn(w, cfg, st0, st1, tr, l)
    U = tr.sel[l][0]
    if fault == "K":
        sn.K_new[0][:, U[0], :] *= 1.5
    elif fault == "H":
        sn.Hn_new[0][U[-1]] = -sn.Hn_new[0][U[-1]]
    elif fault == "attn":
        attn = attn.copy()
        attn[0] *= 3.0
    elif fault == "d":
        sn.d[0, U[0]] += 1e-3
    elif fault == "sel":
        i = int(np.setdiff1d(np.arange(sn.d.shape[1]), U)[0])
        sn.sel[0, :len(U)] = np.sort(np.concatenate([U[1:], [i]]))
    with pytest.raises(AssertionError):
        teacher_forced_layer(sn, w.layers[l], cfg, tr.s[:, l], tr.budgets[:, l], keys, 4, 0, 2e-2, attn_gpu=attn)
