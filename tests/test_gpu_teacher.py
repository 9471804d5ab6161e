"""Teacher-forced parity on a small bf16 model with a long sequence (N = 4096),
so that every CTA of both tensor-core attentions walks many key chunks: the
dense forward gives each (kv head, 128-query tile) CTA all 4096 keys (32
chunks of 128 keys on tcgen05, 64 of 64 keys on mma.sync), a DCU step splits
the keys 8 ways (4 or 8 chunks per CTA), so the TMA rings wrap their mbarrier
phases and the online-softmax rescale runs across chunks.  Every layer is compared with the oracle fed the GPU's own layer
inputs; the attention output of the last layer is compared directly."""
import numpy as np
import pytest
import torch

import oracle as O
from dynamic_layer_wise_b200 import dcu
from dynamic_layer_wise_b200 import inputs as I

from .helpers import LayerSnap, dense_layer_check, oracle_cfg, oracle_weights, rel_l2, teacher_forced_layer, to_np

pytestmark = pytest.mark.gpu

LONG_BF16 = I.ModelShape(n_layers=2, d_model=256, n_heads=4, n_kv_heads=2, head_dim=128, d_ffn=512, vocab=640,
                         dtype="bf16")


def _snapshot(ctx, L):
    return ([dcu.dcu_get_tensor(ctx, dcu.DCU_T_H, l).clone() for l in range(L + 1)],
            [dcu.dcu_get_tensor(ctx, dcu.DCU_T_K, l).clone() for l in range(L)],
            [dcu.dcu_get_tensor(ctx, dcu.DCU_T_V, l).clone() for l in range(L)])


@pytest.mark.parametrize("fused,attn", [(False, "tcgen05"), (True, "tcgen05"), (False, "mma_sync")])
@pytest.mark.parametrize("B_layer,B_window", [(32, 32), (200, 16)])
def test_long_sequence_multichunk_attention_teacher_forced(B_layer, B_window, fused, attn):
    shape, seed, n_prompt, n_gen = LONG_BF16, 7, 3840, 256
    N, B = n_prompt + n_gen, 1
    L, D, Hkv, hd, H = shape.n_layers, shape.d_model, shape.n_kv_heads, shape.head_dim, shape.n_heads
    cfg_o = oracle_cfg(shape)
    w_o = oracle_weights(shape, seed)
    W = I.device_weights(shape, seed)
    ctx = dcu.dcu_create(W, I.cfg_dict(shape, B, N))
    dcu.dcu_set_option(ctx, dcu.DCU_OPT_FUSED_EPILOGUE, int(fused))
    dcu.dcu_set_option(ctx, dcu.DCU_OPT_ATTENTION,
                       dcu.DCU_ATTN_TCGEN05 if attn == "tcgen05" else dcu.DCU_ATTN_MMA_SYNC)
    ids = np.stack([I.sequence_ids(seed, 0, n_prompt, n_gen, shape.vocab)])
    t_ids = torch.tensor(ids, dtype=torch.int32).cuda()
    dcu.dcu_full_forward(ctx, t_ids)
    assert dcu.dcu_status(ctx) == 0

    # dense forward: every layer teacher-forced on the GPU's input rows; attention of the last layer directly
    sample = np.unique(np.concatenate([[0, 1, 2047, 2048, N - 1], np.arange(n_prompt - 4, N, 37)]))
    for l in range(L):
        Hl = to_np(dcu.dcu_get_tensor(ctx, dcu.DCU_T_H, l)).reshape(B, N, D)
        Hn = to_np(dcu.dcu_get_tensor(ctx, dcu.DCU_T_H, l + 1)).reshape(B, N, D)
        K = to_np(dcu.dcu_get_tensor(ctx, dcu.DCU_T_K, l)).reshape(B, Hkv, N, hd)
        V = to_np(dcu.dcu_get_tensor(ctx, dcu.DCU_T_V, l)).reshape(B, Hkv, N, hd)
        dense_layer_check(w_o.layers[l], cfg_o, Hl, Hn, K, V, sample, 2e-2, label=f"dense layer {l}")
        if l == L - 1:
            attn = to_np(dcu.dcu_get_tensor(ctx, dcu.DCU_T_ATTN)).reshape(N, H * hd)
            Ko, Vo = O.kv_rows(w_o.layers[l], cfg_o, Hl[0], np.arange(N))
            tr = {}
            O.layer_rows(w_o.layers[l], cfg_o, Hl[0][sample], sample, Ko, Vo, trace=tr)
            e = rel_l2(attn[sample], tr["attn"])
            assert e <= 2e-2, f"dense attention rel L2 {e:.3e}"

    # two DCU steps (uniform split, then the split of the first step's s)
    keys = [[]]
    for step in range(2):
        pos, new = I.unmask_draw(seed + step, 0, np.arange(n_prompt, N), 4, shape.vocab)
        ids[0, pos] = new
        keys = [list(pos)]
        kp = np.zeros((B, N), np.int32)
        kp[0, :len(pos)] = pos
        nk = np.array([len(pos)], np.int32)
        before = _snapshot(ctx, L)
        t_ids.copy_(torch.tensor(ids, dtype=torch.int32))
        dcu.dcu_step(ctx, t_ids, torch.tensor(kp).cuda(), torch.tensor(nk).cuda(), B_layer, B_window)
        assert dcu.dcu_status(ctx) == 0
        after = _snapshot(ctx, L)
        bud = dcu.dcu_get_tensor(ctx, dcu.DCU_T_BUDGET).cpu().numpy().reshape(B, L)
        s_g = dcu.dcu_get_tensor(ctx, dcu.DCU_T_S).cpu().numpy().reshape(B, L)
        if step == 0:
            assert np.all(bud == B_layer)
        else:
            np.testing.assert_array_equal(bud[0], O.split_budget(s_prev, B_layer, False))
        attn = to_np(dcu.dcu_get_tensor(ctx, dcu.DCU_T_ATTN)).reshape(B * N, H * hd)
        for l in range(L):
            snap = LayerSnap(before, after, ctx, l, B, N, shape, dcu)
            teacher_forced_layer(snap, w_o.layers[l], cfg_o, s_g[:, l], bud[:, l], keys, B_window, 0, 2e-2,
                                 attn_gpu=attn if l == L - 1 else None, label=f"step {step} layer {l}")
        s_prev = s_g[0].copy()
    ctx.close()


@pytest.mark.parametrize("attn", ["tcgen05", "mma_sync"])
def test_query_tiles_beyond_the_expected_set_teacher_forced(attn):
    """Many unmasked keys with wide windows and a small budget: each sequence
    recomputes ~250 rows (~500 queries per kv head) while the launch geometry
    is sized for the expected ~25 rows, so every attention CTA walks several
    128-query tiles in turn (and, with 8 key splits, merges each tile in its
    cluster).  Teacher-forced against the oracle, attention output included."""
    shape, seed, n_prompt, n_gen, B = LONG_BF16, 11, 1536, 512, 2
    N, L, H, hd = n_prompt + n_gen, shape.n_layers, shape.n_heads, shape.head_dim
    B_layer, B_window, n_keys = 8, 16, 24
    cfg_o = oracle_cfg(shape)
    w_o = oracle_weights(shape, seed)
    W = I.device_weights(shape, seed)
    ctx = dcu.dcu_create(W, I.cfg_dict(shape, B, N))
    dcu.dcu_set_option(ctx, dcu.DCU_OPT_ATTENTION,
                       dcu.DCU_ATTN_TCGEN05 if attn == "tcgen05" else dcu.DCU_ATTN_MMA_SYNC)
    ids = np.stack([I.sequence_ids(seed, b, n_prompt, n_gen, shape.vocab) for b in range(B)])
    t_ids = torch.tensor(ids, dtype=torch.int32).cuda()
    dcu.dcu_full_forward(ctx, t_ids)
    assert dcu.dcu_status(ctx) == 0
    keys = []
    kp = np.zeros((B, N), np.int32)
    for b in range(B):
        pos, new = I.unmask_draw(seed + 1, b, np.arange(n_prompt, N), n_keys, shape.vocab)
        ids[b, pos] = new
        keys.append(list(pos))
        kp[b, :n_keys] = pos
    before = _snapshot(ctx, L)
    t_ids.copy_(torch.tensor(ids, dtype=torch.int32))
    dcu.dcu_step(ctx, t_ids, torch.tensor(kp).cuda(), torch.full((B,), n_keys, dtype=torch.int32).cuda(), B_layer,
                 B_window)
    assert dcu.dcu_status(ctx) == 0
    after = _snapshot(ctx, L)
    cnt = dcu.dcu_get_tensor(ctx, dcu.DCU_T_SEL_COUNT, 0).cpu().numpy()
    assert int(cnt.min()) > 150, cnt  # >= 3 query tiles per (sequence, kv head)
    bud = dcu.dcu_get_tensor(ctx, dcu.DCU_T_BUDGET).cpu().numpy().reshape(B, L)
    s_g = dcu.dcu_get_tensor(ctx, dcu.DCU_T_S).cpu().numpy().reshape(B, L)
    attn_out = to_np(dcu.dcu_get_tensor(ctx, dcu.DCU_T_ATTN)).reshape(B * N, H * hd)
    for l in range(L):
        snap = LayerSnap(before, after, ctx, l, B, N, shape, dcu)
        teacher_forced_layer(snap, w_o.layers[l], cfg_o, s_g[:, l], bud[:, l], keys, B_window, 0, 2e-2,
                             attn_gpu=attn_out if l == L - 1 else None, label=f"layer {l}")
    ctx.close()
