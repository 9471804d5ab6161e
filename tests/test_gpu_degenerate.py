"""Degenerate cases of the DCU step and the commit on the GPU, each reduced to
a property the method fixes ([DLLM] "关键设计 1/2"):
* B_layer = 0 and no window: nothing is recomputed, so every cache but the
  layer-0 input is bitwise unchanged and d is exactly 0 from layer 1 on;
* B_layer = N and no window: every row is recomputed, so the caches equal a
  dense forward over the new ids (bf16 tolerance: different launch shapes);
* no masked position left: the commit commits nothing and changes nothing."""
import numpy as np
import pytest
import torch

from dynamic_layer_wise_b200 import dcu
from dynamic_layer_wise_b200 import inputs as I

from .helpers import rel_l2, to_np

pytestmark = pytest.mark.gpu

SHAPE = I.ModelShape(n_layers=3, d_model=256, n_heads=4, n_kv_heads=2, head_dim=64, d_ffn=512, vocab=1000,
                     dtype="bf16")
SEED, N_PROMPT, N_GEN = 8, 170, 60
N = N_PROMPT + N_GEN


def _caches(ctx):
    L = SHAPE.n_layers
    return ([dcu.dcu_get_tensor(ctx, dcu.DCU_T_H, l).clone() for l in range(L + 1)],
            [dcu.dcu_get_tensor(ctx, dcu.DCU_T_K, l).clone() for l in range(L)],
            [dcu.dcu_get_tensor(ctx, dcu.DCU_T_V, l).clone() for l in range(L)])


def _setup(W):
    ctx = dcu.dcu_create(W, I.cfg_dict(SHAPE, 1, N))
    ids0 = I.sequence_ids(SEED, 0, N_PROMPT, N_GEN, SHAPE.vocab)[None]
    ids = torch.tensor(ids0, dtype=torch.int32).cuda()
    dcu.dcu_full_forward(ctx, ids)
    pos, new = I.unmask_draw(SEED, 0, np.arange(N_PROMPT, N), 4, SHAPE.vocab)
    ids1 = ids0.copy()
    ids1[0, pos] = new
    keys = np.zeros((1, N), np.int32)
    keys[0, :len(pos)] = pos
    return ctx, ids, ids1, torch.tensor(keys).cuda(), torch.tensor([len(pos)], dtype=torch.int32).cuda(), pos


def test_zero_budget_no_window_keeps_every_cache_but_h0():
    W = I.device_weights(SHAPE, SEED)
    ctx, ids, ids1, keys, nkeys, pos = _setup(W)
    before = _caches(ctx)
    ids.copy_(torch.tensor(ids1, dtype=torch.int32))
    dcu.dcu_step(ctx, ids, keys, nkeys, 0, 0)
    assert dcu.dcu_status(ctx) == 0
    after = _caches(ctx)
    L = SHAPE.n_layers
    for l in range(1, L + 1):
        assert torch.equal(before[0][l], after[0][l]), f"H_{l} changed"
    for l in range(L):
        assert torch.equal(before[1][l], after[1][l]) and torch.equal(before[2][l], after[2][l]), f"K/V_{l} changed"
    h0b, h0a = before[0][0].view(N, -1), after[0][0].view(N, -1)
    changed = np.flatnonzero((h0b != h0a).any(dim=1).cpu().numpy())
    assert set(changed) <= set(pos.tolist())          # only the refreshed key rows of H_0
    for l in range(L):
        cnt = dcu.dcu_get_tensor(ctx, dcu.DCU_T_SEL_COUNT, l).cpu().numpy()
        assert cnt[0] == 0
    for l in range(1, L):
        assert not dcu.dcu_get_tensor(ctx, dcu.DCU_T_D, l).view(-1)[:N].any()
    ctx.close()


def test_full_budget_no_window_equals_a_dense_forward():
    W = I.device_weights(SHAPE, SEED)
    ctx, ids, ids1, keys, nkeys, _ = _setup(W)
    ids.copy_(torch.tensor(ids1, dtype=torch.int32))
    dcu.dcu_step(ctx, ids, keys, nkeys, N, 0)          # first cached step: uniform budgets of N each
    assert dcu.dcu_status(ctx) == 0
    for l in range(SHAPE.n_layers):
        assert dcu.dcu_get_tensor(ctx, dcu.DCU_T_SEL_COUNT, l).cpu().numpy()[0] == N
    step = _caches(ctx)
    ref = dcu.dcu_create(W, I.cfg_dict(SHAPE, 1, N))
    dcu.dcu_full_forward(ref, torch.tensor(ids1, dtype=torch.int32).cuda())
    dense = _caches(ref)
    for kind, a, b in (("H", step[0], dense[0]), ("K", step[1], dense[1]), ("V", step[2], dense[2])):
        for l, (x, y) in enumerate(zip(a, b)):
            e = rel_l2(to_np(x), to_np(y))
            assert e <= 2e-2, f"{kind}_{l}: rel L2 {e:.3e}"
    ctx.close()
    ref.close()


def test_commit_with_nothing_masked_commits_nothing():
    W = I.device_weights(SHAPE, SEED)
    ctx = dcu.dcu_create(W, I.cfg_dict(SHAPE, 1, N))
    ids = torch.tensor(I.sequence_ids(SEED, 0, N_PROMPT, N_GEN, SHAPE.vocab)[None], dtype=torch.int32).cuda()
    dcu.dcu_full_forward(ctx, ids)
    masked = torch.zeros((1, N), dtype=torch.uint8, device="cuda")
    ids_before = ids.clone()
    pos = torch.full((1, N), -1, dtype=torch.int32, device="cuda")
    cnt = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    for rule, param in ((dcu.DCU_FRECHET, 0.1), (dcu.DCU_THRESHOLD, 0.9), (dcu.DCU_FACTOR, 0.9)):
        dcu.commit_select(ctx, rule, param, masked, ids, pos, cnt)
        assert dcu.dcu_status(ctx) == 0
        assert cnt.item() == 0
        assert torch.equal(ids, ids_before) and not masked.any()
    ctx.close()
