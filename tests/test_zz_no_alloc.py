"""The allocation-free LM-head confidence entry point (for callers that cannot
call cudaMalloc) against the allocating path of commit_select.

Collected last on purpose: if it fails, a run that stops at the first failure
has already run every other test."""
import numpy as np
import pytest
import torch

from dynamic_layer_wise_b200 import dcu
from dynamic_layer_wise_b200 import inputs as I

pytestmark = pytest.mark.gpu

SHAPE = I.ModelShape(n_layers=2, d_model=256, n_heads=4, n_kv_heads=2, head_dim=64, d_ffn=512, vocab=10000,
                     dtype="bf16")


def test_noalloc_confidence_matches_commit_select_twice():
    seed, n_prompt, n_gen = 21, 200, 100
    N = n_prompt + n_gen
    W = I.device_weights(SHAPE, seed)
    ctx = dcu.dcu_create(W, I.cfg_dict(SHAPE, 1, N))
    ids = torch.tensor(I.sequence_ids(seed, 0, n_prompt, n_gen, SHAPE.vocab)[None], dtype=torch.int32).cuda()
    masked = (ids == SHAPE.mask_id).to(torch.uint8)
    pos = torch.zeros((1, N), dtype=torch.int32, device="cuda")
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    dcu.dcu_full_forward(ctx, ids)
    mpos = torch.nonzero(masked[0]).flatten()
    dcu.commit_select(ctx, dcu.DCU_FRECHET, 0.1, masked, ids, pos, cnt)
    conf_ref = dcu.dcu_get_tensor(ctx, dcu.DCU_T_CONF)[mpos]
    amax_ref = dcu.dcu_get_tensor(ctx, dcu.DCU_T_ARGMAX)[mpos]
    h_last = dcu.dcu_get_tensor(ctx, dcu.DCU_T_H, SHAPE.n_layers).view(N, SHAPE.d_model)[mpos].contiguous()
    assert dcu.dcu_status(ctx) == 0
    for call in range(2):                      # two calls in a row share the static scratch
        conf, amax = dcu.dcu_lm_confidence_noalloc(h_last, W["final_norm"], W["lm_head"], SHAPE.rms_eps)
        torch.cuda.synchronize()
        np.testing.assert_allclose(conf.cpu().numpy(), conf_ref.cpu().numpy(), rtol=1e-5, atol=0,
                                   err_msg=f"call {call}")
        np.testing.assert_array_equal(amax.cpu().numpy(), amax_ref.cpu().numpy(), err_msg=f"call {call}")
    with pytest.raises(dcu.DcuError):
        dcu.dcu_lm_confidence_noalloc(torch.zeros((300, SHAPE.d_model), dtype=torch.bfloat16, device="cuda"),
                                      W["final_norm"], W["lm_head"])
    ctx.close()
