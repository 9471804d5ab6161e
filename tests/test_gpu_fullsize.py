"""Parity at the full sizes of the benchmark configurations, in the launch
configuration bench.py times (CUDA graphs on, the same context sizes).

The oracle cannot run a whole 32-layer chain at these sizes, so each test
checks (0) the dense forward's first layer teacher-forced on the GPU's H_0
(K/V of every row, H_1 of sampled rows), (1) what the oracle computes from
the seeded inputs alone -- layer-0 dynamics and selections exactly, LM-head
confidence and argmax of sampled masked rows on seeded synthetic final-layer
rows, (1b) teacher-forced layers 0, 1 and L-1 of a DCU step: the oracle is fed
the GPU's layer inputs and must reproduce d, s, the selection (exact up to the
1e-5 near-boundary band), H_{l+1}, K_l and V_l of the recomputed rows and, at
layer L-1, the attention output -- and (2) invariants that hold at any size at
every layer: budgets sum to B_layer * L, stay within one of their quota and
equal the oracle's split of the GPU's s, selections are the window plus the
top-B of the GPU's own d, d^{l+1} is exactly 0 and H_{l+1} / K_l / V_l are
bitwise unchanged at every row layer l did not recompute, and the commit
follows its rule on the GPU's own confidences."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from dynamic_layer_wise_b200 import dcu
from dynamic_layer_wise_b200 import inputs as I

from .helpers import (LayerSnap, LazyMatrix, check_selection_valid, dense_layer_check, oracle_cfg, rel_l2,
                      teacher_forced_layer, to_np)

pytestmark = pytest.mark.gpu

CONFIGS = {
    "llada8b_n1024": dict(shape=I.LLADA_8B, B=1, n_prompt=768, n_gen=256, B_layer=32, B_window=32,
                          rule=O.RULE_FRECHET, param=0.1),
    "llada8b_batch4_n2048": dict(shape=I.LLADA_8B, B=4, n_prompt=1536, n_gen=512, B_layer=64, B_window=32,
                                 rule=O.RULE_THRESHOLD, param=0.9),
    "dream7b_n1024": dict(shape=I.DREAM_7B, B=1, n_prompt=768, n_gen=256, B_layer=32, B_window=32,
                          rule=O.RULE_FACTOR, param=0.9),
    "llada8b_n8192": dict(shape=I.LLADA_8B, B=1, n_prompt=7680, n_gen=512, B_layer=96, B_window=64,
                          rule=O.RULE_FRECHET, param=0.05),
}


def _layer_weights(shape, seed, l, names):
    """fp64 host copies of layer l's matrices, from the host generator (norm gains are ones)."""
    lw = {n: I.as_f64(I.weight_rows(shape, seed, n, 0, shape.weight_shapes()[n][0], layer=l), shape.dtype)
          for n in names}
    lw["attn_norm"] = lw["ffn_norm"] = np.ones(shape.d_model)
    return lw


def _snapshot(ctx, L):
    return ([dcu.dcu_get_tensor(ctx, dcu.DCU_T_H, l).clone() for l in range(L + 1)],
            [dcu.dcu_get_tensor(ctx, dcu.DCU_T_K, l).clone() for l in range(L)],
            [dcu.dcu_get_tensor(ctx, dcu.DCU_T_V, l).clone() for l in range(L)])


@pytest.mark.parametrize("name,fused", [(n, False) for n in CONFIGS] +
                         [("llada8b_n1024", True), ("llada8b_batch4_n2048", True), ("dream7b_n1024", True)])
def test_fullsize_dcu_step(name, fused):
    c = CONFIGS[name]
    shape, B = c["shape"], c["B"]
    N = c["n_prompt"] + c["n_gen"]
    L, D, Hkv, hd = shape.n_layers, shape.d_model, shape.n_kv_heads, shape.head_dim
    seed = 0
    W = I.device_weights(shape, seed)
    ctx = dcu.dcu_create(W, I.cfg_dict(shape, B, N))
    dcu.dcu_set_option(ctx, dcu.DCU_OPT_FUSED_EPILOGUE, int(fused))
    ids0 = np.stack([I.sequence_ids(1 + b, b, c["n_prompt"], c["n_gen"], shape.vocab) for b in range(B)])
    t_ids = torch.tensor(ids0, dtype=torch.int32, device="cuda")
    dcu.dcu_full_forward(ctx, t_ids)
    assert dcu.dcu_status(ctx) == 0
    cfg_o = oracle_cfg(shape)

    # (0) dense forward, layer 0, teacher-forced on the GPU's H_0: K/V of every row and H_1 of sampled rows
    lw0 = _layer_weights(shape, seed, 0, I.LAYER_TENSORS)
    H0 = to_np(dcu.dcu_get_tensor(ctx, dcu.DCU_T_H, 0)).reshape(B, N, D)
    H1 = to_np(dcu.dcu_get_tensor(ctx, dcu.DCU_T_H, 1)).reshape(B, N, D)
    K0 = to_np(dcu.dcu_get_tensor(ctx, dcu.DCU_T_K, 0)).reshape(B, Hkv, N, hd)
    V0 = to_np(dcu.dcu_get_tensor(ctx, dcu.DCU_T_V, 0)).reshape(B, Hkv, N, hd)
    sample = np.unique(np.concatenate([[0, 1, N // 2, N - 2, N - 1], np.linspace(0, N - 1, 7).astype(int)]))
    dense_layer_check(lw0, cfg_o, H0, H1, K0, V0, sample, 2e-2, label=f"{name} dense layer 0")
    del H0, H1, K0, V0

    # synthetic unmasking of 3 generated positions per sequence (the same inputs for the oracle)
    ids1 = ids0.copy()
    keys = []
    for b in range(B):
        pos, new = I.unmask_draw(seed, b, np.arange(c["n_prompt"], N), 3, shape.vocab)
        ids1[b, pos] = new
        keys.append(list(pos))
    kp = np.zeros((B, N), np.int32)
    nk = np.array([len(k) for k in keys], np.int32)
    for b in range(B):
        kp[b, :nk[b]] = keys[b]
    before = _snapshot(ctx, L)
    t_ids.copy_(torch.tensor(ids1, dtype=torch.int32))
    dcu.dcu_step(ctx, t_ids, torch.tensor(kp).cuda(), torch.tensor(nk).cuda(), c["B_layer"], c["B_window"])
    assert dcu.dcu_status(ctx) == 0
    after = _snapshot(ctx, L)

    budgets = dcu.dcu_get_tensor(ctx, dcu.DCU_T_BUDGET).cpu().numpy().reshape(B, L)
    assert np.all(budgets == c["B_layer"])                         # first cached step: uniform split

    # (1) layer 0 from the oracle: d^0 of the key rows and the selection, exactly
    emb = {}
    for b in range(B):
        for p in keys[b]:
            for tok in (ids0[b, p], ids1[b, p]):
                if tok not in emb:
                    emb[tok] = I.as_f64(I.weight_values(shape, seed, "embed", rows=[tok])[0], shape.dtype)
    d0 = dcu.dcu_get_tensor(ctx, dcu.DCU_T_D, 0).cpu().numpy().reshape(B, N)
    sel0 = dcu.dcu_get_tensor(ctx, dcu.DCU_T_SEL, 0).cpu().numpy().reshape(B, N)
    cnt0 = dcu.dcu_get_tensor(ctx, dcu.DCU_T_SEL_COUNT, 0).cpu().numpy()
    for b in range(B):
        d_ora = np.zeros(N, np.float32)
        for p in keys[b]:
            d_ora[p] = O.to_f32(O.cosine_distance(emb[ids1[b, p]], emb[ids0[b, p]], np.ones(D)))[0]
        np.testing.assert_allclose(d0[b], d_ora, rtol=0, atol=2e-7)
        ref = O.select_rows(d_ora, keys[b], c["B_window"], int(budgets[b, 0]), 0)
        np.testing.assert_array_equal(sel0[b, :cnt0[b]], ref)

    # (1b) teacher-forced parity at layers 0, 1 and L-1: the oracle is fed the GPU's H_l (before and
    # after the step), K_l / V_l before it and the GPU's budgets; at layer L-1 the attention output of
    # the recomputed rows is compared too (the tensor-core attention's split and merge path)
    s_gpu = dcu.dcu_get_tensor(ctx, dcu.DCU_T_S).cpu().numpy().reshape(B, L)
    attn = to_np(dcu.dcu_get_tensor(ctx, dcu.DCU_T_ATTN)).reshape(B * N, shape.n_heads * hd)
    exempt = 0
    for l in (0, 1, L - 1):
        lw = lw0 if l == 0 else _layer_weights(shape, seed, l, I.LAYER_TENSORS)
        snap = LayerSnap(before, after, ctx, l, B, N, shape, dcu)
        exempt += teacher_forced_layer(snap, lw, cfg_o, s_gpu[:, l], budgets[:, l], keys, c["B_window"], 0, 2e-2,
                                       attn_gpu=attn if l == L - 1 else None, label=f"{name} layer {l}")
        del snap, lw
    print(f"{name}: teacher-forced layers 0, 1, {L - 1}: {exempt} near-boundary selection differences")
    del lw0

    # (2) invariants at every layer
    for l in range(L):
        d = dcu.dcu_get_tensor(ctx, dcu.DCU_T_D, l).cpu().numpy().reshape(B, N)
        sel = dcu.dcu_get_tensor(ctx, dcu.DCU_T_SEL, l).cpu().numpy().reshape(B, N)
        cnt = dcu.dcu_get_tensor(ctx, dcu.DCU_T_SEL_COUNT, l).cpu().numpy()
        d_next = dcu.dcu_get_tensor(ctx, dcu.DCU_T_D, l + 1).cpu().numpy().reshape(B, N) if l + 1 < L else None
        Hn_b, Hn_a = before[0][l + 1].view(B, N, D), after[0][l + 1].view(B, N, D)
        K_b, K_a = before[1][l].view(B, Hkv, N, hd), after[1][l].view(B, Hkv, N, hd)
        V_b, V_a = before[2][l].view(B, Hkv, N, hd), after[2][l].view(B, Hkv, N, hd)
        for b in range(B):
            U = sel[b, :cnt[b]]
            check_selection_valid(U, d[b], keys[b], c["B_window"], budgets[b, l], 0, N)
            off = np.setdiff1d(np.arange(N), U)
            if d_next is not None:
                assert np.all(d_next[b, off] == 0.0), f"layer {l + 1}: d not 0 off the recomputed rows"
            off_t = torch.tensor(off, device="cuda", dtype=torch.long)
            assert torch.equal(Hn_b[b, off_t], Hn_a[b, off_t]), f"H_{l + 1} changed off U"
            assert torch.equal(K_b[b][:, off_t], K_a[b][:, off_t]), f"K_{l} changed off U"
            assert torch.equal(V_b[b][:, off_t], V_a[b][:, off_t]), f"V_{l} changed off U"
    s = dcu.dcu_get_tensor(ctx, dcu.DCU_T_S).cpu().numpy().reshape(B, L)

    # next step's budgets: exact sum and within one of the proportional quota
    dcu.dcu_step(ctx, t_ids, torch.tensor(kp).cuda(), torch.zeros(B, dtype=torch.int32, device="cuda"),
                 c["B_layer"], c["B_window"])
    b2 = dcu.dcu_get_tensor(ctx, dcu.DCU_T_BUDGET).cpu().numpy().reshape(B, L)
    for b in range(B):
        assert b2[b].sum() == c["B_layer"] * L
        tot = float(np.sum(s[b].astype(np.float64)))
        if tot > 0:
            q = c["B_layer"] * L * s[b].astype(np.float64) / tot
            assert np.all(np.abs(b2[b] - q) < 1.0 + 1e-9)
        # bit-exact against the oracle fed the GPU's s
        np.testing.assert_array_equal(b2[b], O.split_budget(s[b], c["B_layer"], False))

    # (1') commit on seeded synthetic final-layer rows (set through the ABI), sampled vs the oracle
    HL = I.normal_values(seed, 9100, 0, B * N * D, 1.0, shape.dtype)
    HL_t = torch.tensor(HL.view(np.int16)).view(torch.bfloat16).cuda()
    dcu.dcu_set_tensor(ctx, dcu.DCU_T_H, L, HL_t)
    masked = torch.tensor((ids1 == shape.mask_id).astype(np.uint8)).cuda()
    m_before = masked.clone()
    t_pos = torch.zeros((B, N), dtype=torch.int32, device="cuda")
    t_cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
    dcu.commit_select(ctx, c["rule"], c["param"], masked, t_ids, t_pos, t_cnt)
    conf = dcu.dcu_get_tensor(ctx, dcu.DCU_T_CONF).cpu().numpy().reshape(B, N)
    amax = dcu.dcu_get_tensor(ctx, dcu.DCU_T_ARGMAX).cpu().numpy().reshape(B, N)
    assert dcu.dcu_status(ctx) == 0
    lm = LazyMatrix(shape, seed, "lm_head", shape.vocab)
    HL64 = I.as_f64(HL, shape.dtype).reshape(B, N, D)
    mb = m_before.cpu().numpy().astype(bool)
    pos, cnt = t_pos.cpu().numpy(), t_cnt.cpu().numpy()
    for b in range(B):
        mp = np.flatnonzero(mb[b])
        sample = mp[:: max(1, len(mp) // 6)][:6]
        c_o, a_o = O.confidence(HL64[b][sample], np.ones(D), lm, shape.rms_eps)
        np.testing.assert_allclose(conf[b, sample], c_o, rtol=2e-2, atol=0)
        assert np.all(amax[b, sample] == a_o)
        # the commit follows its rule on the GPU's own confidences
        cm = conf[b, mp]
        order = mp[np.lexsort((mp, -cm.astype(np.float64)))]
        assert list(pos[b, :cnt[b]]) == list(order[:cnt[b]])
        cs = conf[b, order].astype(np.float64)
        n = int(cnt[b])
        assert n >= 1
        if c["rule"] == O.RULE_THRESHOLD:
            assert n == max(1, int(np.sum(conf[b, order] >= np.float32(c["param"]))))
        elif c["rule"] == O.RULE_FACTOR:
            assert n == 1 or (n + 1) * (1 - cs[n - 1]) < c["param"]
        else:
            Ln = max(0.0, float(np.sum(cs[:n])) - (n - 1))
            assert n == 1 or Ln - (1 - cs[n - 1]) > c["param"]
    ctx.close()
    del W
    torch.cuda.empty_cache()
