"""The pass sweep of the layer GEMMs and of the LM head
(DCU_OPT_GEMM_PASS_SWEEP): when the rows span more than one 256-row token
pass, two passes share each weight tile in shared memory, each with its own
tensor-memory accumulator.  Every accumulator still receives the same
tensor-core instructions in the same k order as with one pass per weight
stream, and the LM head folds each token's logits over the vocabulary tiles in
the same order, so caches, confidences, argmaxes and commits must be
bit-identical with the sweep on and off -- over a dense forward (5 passes:
groups of 2, 2 and 1), LM heads over 600 and fewer masked rows (3 passes) and
DCU steps whose recompute sets span 2 and 3 passes."""
import numpy as np
import pytest
import torch

import oracle as O
from dynamic_layer_wise_b200 import dcu
from dynamic_layer_wise_b200 import inputs as I

pytestmark = pytest.mark.gpu

SWEEP_BF16 = I.ModelShape(n_layers=2, d_model=256, n_heads=4, n_kv_heads=2, head_dim=64, d_ffn=512, vocab=800,
                          dtype="bf16")


def _caches(ctx, L):
    return ([dcu.dcu_get_tensor(ctx, dcu.DCU_T_H, l).clone() for l in range(L + 1)] +
            [dcu.dcu_get_tensor(ctx, dcu.DCU_T_K, l).clone() for l in range(L)] +
            [dcu.dcu_get_tensor(ctx, dcu.DCU_T_V, l).clone() for l in range(L)] +
            [dcu.dcu_get_tensor(ctx, dcu.DCU_T_D, l).clone() for l in range(L)])


@pytest.mark.parametrize("B_layer", [150, 280])
def test_pass_sweep_is_bit_identical(B_layer):
    shape, seed, B, n_prompt, n_gen = SWEEP_BF16, 13, 2, 300, 300
    N, L = n_prompt + n_gen, shape.n_layers
    W = I.device_weights(shape, seed)
    ids = np.stack([I.sequence_ids(seed, b, n_prompt, n_gen, shape.vocab) for b in range(B)])
    runs = []
    for sweep in (1, 0):
        ctx = dcu.dcu_create(W, I.cfg_dict(shape, B, N))
        dcu.dcu_set_option(ctx, dcu.DCU_OPT_GEMM_PASS_SWEEP, sweep)
        t_ids = torch.tensor(ids, dtype=torch.int32).cuda()
        masked = (t_ids == shape.mask_id).to(torch.uint8)
        pos = torch.zeros((B, N), dtype=torch.int32, device="cuda")
        cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
        dcu.dcu_full_forward(ctx, t_ids)
        snaps = [_caches(ctx, L)]
        for step in range(3):
            was = masked.reshape(-1).bool().clone()  # conf / argmax are written at these positions
            n_masked = int(was.sum().item())
            dcu.commit_select(ctx, O.RULE_FRECHET, 0.1, masked, t_ids, pos, cnt)
            assert dcu.dcu_status(ctx) == 0
            if step == 0:
                assert n_masked > 512, n_masked  # the LM head takes three 256-row passes
            snaps.append([dcu.dcu_get_tensor(ctx, dcu.DCU_T_CONF).reshape(-1)[was].clone(),
                          dcu.dcu_get_tensor(ctx, dcu.DCU_T_ARGMAX).reshape(-1)[was].clone(), pos.clone(),
                          cnt.clone(), t_ids.clone(), masked.clone()])
            dcu.dcu_step(ctx, t_ids, pos, cnt, B_layer, 8)
            assert dcu.dcu_status(ctx) == 0
            rows = max(int(dcu.dcu_get_tensor(ctx, dcu.DCU_T_SEL_COUNT, l).cpu().numpy().sum()) for l in range(L))
            # the recompute set spans more than one 256-row token pass
            assert rows > 256, rows
            snaps.append(_caches(ctx, L))
        torch.cuda.synchronize()
        runs.append(snaps)
        del ctx
    for k, (a, b) in enumerate(zip(*runs)):
        for i, (x, y) in enumerate(zip(a, b)):
            assert torch.equal(x, y), f"snapshot {k} tensor {i} differs between sweep on and off"
