"""select_from = "v" (the README's feature source): the token dynamics of a
layer come from the recomputed Value of every stale row (input rewritten
since the layer last recomputed it) against the cached Value.  Checked
teacher-forced against the oracle: from the GPU's stale flags before the step
and its H_l before / after, the oracle derives the stale set at selection
time, the Value distance of those rows, the selection, the recomputed rows,
and the flags after the step (bit-exact).  The Value is rounded to the cache
dtype on both sides after an fp32 (GPU) or fp64 (oracle) dot product, so for
bf16 a few elements may round to neighbouring values and d agrees to ~1e-4
rather than to float32 rounding; the near-boundary band of the selection is
that measured difference."""
import numpy as np
import pytest
import torch

import oracle as O
from dynamic_layer_wise_b200 import dcu
from dynamic_layer_wise_b200 import inputs as I

from .helpers import LayerSnap, oracle_cfg, oracle_weights, teacher_forced_layer

pytestmark = pytest.mark.gpu

SMALL_BF16 = I.ModelShape(n_layers=3, d_model=256, n_heads=4, n_kv_heads=2, head_dim=128, d_ffn=512, vocab=700,
                          dtype="bf16")


def _snapshot(ctx, L):
    return ([dcu.dcu_get_tensor(ctx, dcu.DCU_T_H, l).clone() for l in range(L + 1)],
            [dcu.dcu_get_tensor(ctx, dcu.DCU_T_K, l).clone() for l in range(L)],
            [dcu.dcu_get_tensor(ctx, dcu.DCU_T_V, l).clone() for l in range(L)])


@pytest.mark.parametrize("shape,tol,d_atol,fused", [(SMALL_BF16, 2e-2, 5e-4, False), (SMALL_BF16, 2e-2, 5e-4, True),
                                                   (I.TOY, 1e-4, 1e-6, False)])
def test_value_selection_teacher_forced(shape, tol, d_atol, fused):
    seed, B, n_prompt, n_gen = 12, 2, 180, 60
    N, L = n_prompt + n_gen, shape.n_layers
    B_layer, B_window = 5, 2
    cfg_o = oracle_cfg(shape)
    w_o = oracle_weights(shape, seed)
    W = I.device_weights(shape, seed)
    ctx = dcu.dcu_create(W, I.cfg_dict(shape, B, N))
    dcu.dcu_set_option(ctx, dcu.DCU_OPT_FUSED_EPILOGUE, int(fused))
    dcu.dcu_set_select_from(ctx, dcu.DCU_SELECT_VALUE)
    ids = np.stack([I.sequence_ids(seed, b, n_prompt, n_gen, shape.vocab) for b in range(B)])
    t_ids = torch.tensor(ids, dtype=torch.int32).cuda()
    dcu.dcu_full_forward(ctx, t_ids)
    gen = np.arange(n_prompt, N)
    stale_seen = 0
    for step in range(4):
        keys = []
        for b in range(B):
            pos, new = I.unmask_draw(seed + step, b, gen, 4, shape.vocab)   # more keys than the budget
            ids[b, pos] = new
            keys.append(list(pos))
        kp = np.zeros((B, N), np.int32)
        for b in range(B):
            kp[b, :4] = keys[b]
        stale0 = [dcu.dcu_get_tensor(ctx, dcu.DCU_T_STALE, l).cpu().numpy().reshape(B, N).astype(bool)
                  for l in range(L)]
        before = _snapshot(ctx, L)
        t_ids.copy_(torch.tensor(ids, dtype=torch.int32))
        dcu.dcu_step(ctx, t_ids, torch.tensor(kp).cuda(), torch.full((B,), 4, dtype=torch.int32).cuda(), B_layer,
                     B_window)
        assert dcu.dcu_status(ctx) == 0
        after = _snapshot(ctx, L)
        bud = dcu.dcu_get_tensor(ctx, dcu.DCU_T_BUDGET).cpu().numpy().reshape(B, L)
        s_g = dcu.dcu_get_tensor(ctx, dcu.DCU_T_S).cpu().numpy().reshape(B, L)
        for l in range(L):
            snap = LayerSnap(before, after, ctx, l, B, N, shape, dcu)
            changed = np.any(snap.H_new != snap.H_old, axis=-1)
            stale_sel = stale0[l] | changed
            stale_seen += int(stale_sel.sum())
            teacher_forced_layer(snap, w_o.layers[l], cfg_o, s_g[:, l], bud[:, l], keys, B_window, 0, tol,
                                 label=f"step {step} layer {l}", stale=stale_sel, d_atol=d_atol)
            got = dcu.dcu_get_tensor(ctx, dcu.DCU_T_STALE, l).cpu().numpy().reshape(B, N).astype(bool)
            for b in range(B):
                exp = stale_sel[b].copy()
                exp[snap.sel[b, :snap.cnt[b]]] = False
                np.testing.assert_array_equal(got[b], exp, err_msg=f"step {step} layer {l}: stale flags")
    assert stale_seen > 0
    ctx.close()
