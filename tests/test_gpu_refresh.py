"""Periodic full refresh (the README's prompt_interval_steps /
gen_interval_steps): on a due step the prompt (resp. generated) positions are
forced into every layer's recompute set.  Every step is checked teacher-forced
against the oracle with the same forced range, and a step that refreshes both
blocks must reproduce a dense forward of the same ids."""
import numpy as np
import pytest
import torch

import oracle as O
from dynamic_layer_wise_b200 import dcu
from dynamic_layer_wise_b200 import inputs as I

from .helpers import LayerSnap, oracle_cfg, oracle_weights, rel_l2, teacher_forced_layer, to_np

pytestmark = pytest.mark.gpu

SMALL_BF16 = I.ModelShape(n_layers=2, d_model=256, n_heads=4, n_kv_heads=2, head_dim=64, d_ffn=512, vocab=1000,
                          dtype="bf16")


def _snapshot(ctx, L):
    return ([dcu.dcu_get_tensor(ctx, dcu.DCU_T_H, l).clone() for l in range(L + 1)],
            [dcu.dcu_get_tensor(ctx, dcu.DCU_T_K, l).clone() for l in range(L)],
            [dcu.dcu_get_tensor(ctx, dcu.DCU_T_V, l).clone() for l in range(L)])


@pytest.mark.parametrize("shape,tol,fused", [(SMALL_BF16, 2e-2, False), (SMALL_BF16, 2e-2, True), (I.TOY, 1e-4, False)])
def test_periodic_refresh_teacher_forced(shape, tol, fused):
    seed, B, n_prompt, n_gen = 9, 2, 150, 50
    N, L = n_prompt + n_gen, shape.n_layers
    B_layer, B_window, p_int, g_int = 6, 4, 2, 3
    cfg_o = oracle_cfg(shape)
    w_o = oracle_weights(shape, seed)
    W = I.device_weights(shape, seed)
    ctx = dcu.dcu_create(W, I.cfg_dict(shape, B, N))
    dcu.dcu_set_option(ctx, dcu.DCU_OPT_FUSED_EPILOGUE, int(fused))
    dcu.dcu_set_refresh(ctx, n_prompt, p_int, g_int)
    ids = np.stack([I.sequence_ids(seed, b, n_prompt, n_gen, shape.vocab) for b in range(B)])
    t_ids = torch.tensor(ids, dtype=torch.int32).cuda()
    dcu.dcu_full_forward(ctx, t_ids)
    gen = np.arange(n_prompt, N)
    for step in range(1, 7):
        keys = []
        for b in range(B):
            pos, new = I.unmask_draw(seed + step, b, gen, 2, shape.vocab)
            ids[b, pos] = new
            keys.append(list(pos))
        kp = np.zeros((B, N), np.int32)
        for b in range(B):
            kp[b, :2] = keys[b]
        before = _snapshot(ctx, L)
        t_ids.copy_(torch.tensor(ids, dtype=torch.int32))
        dcu.dcu_step(ctx, t_ids, torch.tensor(kp).cuda(), torch.full((B,), 2, dtype=torch.int32).cuda(), B_layer,
                     B_window)
        assert dcu.dcu_status(ctx) == 0
        after = _snapshot(ctx, L)
        force = O.refresh_range(step, n_prompt, N, p_int, g_int)
        bud = dcu.dcu_get_tensor(ctx, dcu.DCU_T_BUDGET).cpu().numpy().reshape(B, L)
        s_g = dcu.dcu_get_tensor(ctx, dcu.DCU_T_S).cpu().numpy().reshape(B, L)
        for l in range(L):
            snap = LayerSnap(before, after, ctx, l, B, N, shape, dcu)
            teacher_forced_layer(snap, w_o.layers[l], cfg_o, s_g[:, l], bud[:, l], keys, B_window, 0, tol,
                                 label=f"step {step} layer {l}", force=force)
            if force is not None:
                cnt = snap.cnt
                lo, hi = force
                for b in range(B):
                    assert set(range(lo, hi)) <= set(snap.sel[b, :cnt[b]].tolist()), "forced rows not recomputed"
        if force == (0, N):
            # a refresh of both blocks is a dense forward of the same ids
            ref = dcu.dcu_create(W, I.cfg_dict(shape, B, N))
            dcu.dcu_set_option(ref, dcu.DCU_OPT_FUSED_EPILOGUE, int(fused))
            dcu.dcu_full_forward(ref, t_ids)
            for l in range(1, L + 1):
                a = to_np(dcu.dcu_get_tensor(ctx, dcu.DCU_T_H, l))
                r = to_np(dcu.dcu_get_tensor(ref, dcu.DCU_T_H, l))
                assert rel_l2(a, r) <= tol / 10, f"H_{l} after a full refresh vs dense forward"
            ref.close()
    ctx.close()
