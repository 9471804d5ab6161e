"""Block-wise schedule of the commit ([README] "Quick Start": generate_mode
"default"; [FRECHET] "实验关键数据": block size 32) on the GPU against the
oracle: the stateless rule on seeded confidences and the full commit_select
on a small bf16 model."""
import numpy as np
import pytest
import torch

import oracle as O
from dynamic_layer_wise_b200 import dcu
from dynamic_layer_wise_b200 import inputs as I

from .helpers import LazyMatrix

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rule,param", [(O.RULE_FRECHET, 0.1), (O.RULE_THRESHOLD, 0.9), (O.RULE_FACTOR, 0.9)])
@pytest.mark.parametrize("N,gen_start,block_len", [(7, 2, 3), (300, 236, 32), (1000, 500, 64), (4096, 3000, 32),
                                                   (256, 0, 256), (64, 10, 1)])
def test_block_commit_rule_parity(rule, param, N, gen_start, block_len):
    rng = np.random.default_rng(N + block_len + rule)
    for trial in range(4):
        B = int(rng.integers(1, 4))
        c = rng.choice([0.5, 0.9, 0.95, 0.99], (B, N)).astype(np.float32) if trial % 2 else \
            rng.beta(12, 1, (B, N)).astype(np.float32)
        masked = np.zeros((B, N), np.uint8)
        masked[:, gen_start:] = rng.random((B, N - gen_start)) < (0.7 if trial < 3 else 0.0)
        if trial == 1 and N - gen_start > block_len:   # first block already done
            masked[:, gen_start:gen_start + block_len] = 0
        amax = rng.integers(0, 1000, (B, N)).astype(np.int32)
        ids = rng.integers(0, 1000, (B, N)).astype(np.int32)
        tm, ti = torch.tensor(masked).cuda(), torch.tensor(ids).cuda()
        pos = torch.full((B, N), -1, dtype=torch.int32, device="cuda")
        cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
        dcu.dcu_commit_rule_block(rule, param, gen_start, block_len, torch.tensor(c).cuda(), torch.tensor(amax).cuda(),
                                  tm, ti, pos, cnt)
        pos, cnt, tm, ti = pos.cpu().numpy(), cnt.cpu().numpy(), tm.cpu().numpy(), ti.cpu().numpy()
        for b in range(B):
            rp, rid, rm = O.commit(c[b], amax[b], masked[b], ids[b], rule, param, gen_start=gen_start,
                                   block_len=block_len)
            assert cnt[b] == len(rp)
            np.testing.assert_array_equal(pos[b, :cnt[b]], rp)
            np.testing.assert_array_equal(ti[b], rid)
            np.testing.assert_array_equal(tm[b].astype(bool), rm)


SHAPE = I.ModelShape(n_layers=2, d_model=256, n_heads=4, n_kv_heads=2, head_dim=64, d_ffn=512, vocab=1000,
                     dtype="bf16")


def test_commit_select_block_matches_oracle_on_the_open_block():
    """commit_select_block computes the LM head only on the open block's
    masked rows and commits there; confidences / argmax of those rows match
    the oracle, and the committed set is the oracle's block commit on the
    GPU's own confidences."""
    seed, n_prompt, n_gen, blen = 4, 200, 96, 32
    N = n_prompt + n_gen
    W = I.device_weights(SHAPE, seed)
    ctx = dcu.dcu_create(W, I.cfg_dict(SHAPE, 2, N))
    ids0 = np.stack([I.sequence_ids(seed + b, b, n_prompt, n_gen, SHAPE.vocab) for b in range(2)])
    ids = torch.tensor(ids0, dtype=torch.int32).cuda()
    dcu.dcu_full_forward(ctx, ids)
    masked = (ids == SHAPE.mask_id).to(torch.uint8)
    masked[1, n_prompt:n_prompt + blen] = 0                # sequence 1: first block already committed
    m_before = masked.cpu().numpy().astype(bool)
    pos = torch.zeros((2, N), dtype=torch.int32, device="cuda")
    cnt = torch.zeros(2, dtype=torch.int32, device="cuda")
    dcu.commit_select_block(ctx, O.RULE_FRECHET, 0.1, n_prompt, blen, masked, ids, pos, cnt)
    assert dcu.dcu_status(ctx) == 0
    conf = dcu.dcu_get_tensor(ctx, dcu.DCU_T_CONF).cpu().numpy().reshape(2, N)
    amax = dcu.dcu_get_tensor(ctx, dcu.DCU_T_ARGMAX).cpu().numpy().reshape(2, N)
    HL = dcu.dcu_get_tensor(ctx, dcu.DCU_T_H, SHAPE.n_layers).view(2, N, SHAPE.d_model).float().cpu().numpy()
    lm = LazyMatrix(SHAPE, seed, "lm_head", SHAPE.vocab)
    pos, cnt = pos.cpu().numpy(), cnt.cpu().numpy()
    for b in range(2):
        b0, b1 = O.active_block(m_before[b], n_prompt, blen)
        assert b0 == n_prompt + (blen if b == 1 else 0)
        rows = np.flatnonzero(m_before[b, b0:b1]) + b0
        c_o, a_o = O.confidence(HL[b][rows].astype(np.float64), np.ones(SHAPE.d_model), lm, SHAPE.rms_eps)
        np.testing.assert_allclose(conf[b, rows], c_o, rtol=2e-2, atol=0)
        # the argmax is decided in float32 on bf16-rounded inputs: where the two
        # largest logits are that close, either id is a correct maximum, so the
        # GPU's id must reach the oracle's maximum logit within the bf16 input
        # rounding (|dz| ~ |z| 2^-8), and must equal the oracle's id elsewhere
        z = O.rmsnorm(HL[b][rows].astype(np.float64), np.ones(SHAPE.d_model), SHAPE.rms_eps) @ lm[0:SHAPE.vocab].T
        zg = z[np.arange(len(rows)), amax[b, rows]]
        zmax = z.max(axis=1)
        assert np.all(zg >= zmax - 5e-3), float(np.max(zmax - zg))
        second = np.sort(z, axis=1)[:, -2]
        clear = zmax - second > 5e-3
        assert np.all(amax[b, rows][clear] == a_o[clear])
        ref = O.commit(conf[b], amax[b], m_before[b], ids0[b], O.RULE_FRECHET, 0.1, gen_start=n_prompt,
                       block_len=blen)[0]
        np.testing.assert_array_equal(pos[b, :cnt[b]], ref)
        assert all(b0 <= p < b1 for p in pos[b, :cnt[b]])
    ctx.close()
