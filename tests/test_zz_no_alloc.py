"""The allocation-free LM-head confidence entry point, for callers that cannot
call cudaMalloc (a host framework that owns every device allocation, a serving
process whose allocator is frozen).  Checked against the allocating LM-head
path of commit_select and against the oracle, on two calls in a row (the
calls share the library's static scratch), for bf16 with a ragged last
vocabulary chunk and for float32 with a single partial chunk; misaligned and
oversized inputs must be refused.

Collected last on purpose: if it fails, a run that stops at the first failure
has already run every other test."""
import numpy as np
import pytest
import torch

import oracle as O
from dynamic_layer_wise_b200 import dcu
from dynamic_layer_wise_b200 import inputs as I

from .helpers import LazyMatrix

pytestmark = pytest.mark.gpu


def _argmax_ok(amax, rows64, lm, V, eps):
    """The id must be the oracle's wherever its two largest logits are more
    than eps apart; elsewhere it must reach the oracle's maximum within eps
    (either id is then a correct maximum at the kernel's precision)."""
    z = O.rmsnorm(rows64, np.ones(rows64.shape[1]), 1e-5) @ lm[0:V].T
    zmax = z.max(axis=1)
    zg = z[np.arange(len(amax)), amax]
    assert np.all(zg >= zmax - eps), float(np.max(zmax - zg))
    second = np.sort(z, axis=1)[:, -2]
    clear = zmax - second > eps
    assert np.all(amax[clear] == np.argmax(z, axis=1)[clear])


@pytest.mark.parametrize("dtype,vocab,rtol,eps", [("bf16", 10000, 2e-2, 5e-3), ("f32", 3000, 1e-4, 1e-4)])
def test_noalloc_confidence_matches_commit_select_twice(dtype, vocab, rtol, eps):
    shape = I.ModelShape(n_layers=2, d_model=256, n_heads=4, n_kv_heads=2, head_dim=64, d_ffn=512, vocab=vocab,
                         dtype=dtype)
    seed, n_prompt, n_gen = 21, 200, 100
    N, D, L = n_prompt + n_gen, shape.d_model, shape.n_layers
    W = I.device_weights(shape, seed)
    ctx = dcu.dcu_create(W, I.cfg_dict(shape, 1, N))
    ids = torch.tensor(I.sequence_ids(seed, 0, n_prompt, n_gen, vocab)[None], dtype=torch.int32).cuda()
    dcu.dcu_full_forward(ctx, ids)
    # seeded synthetic final-layer rows, set through the ABI, so both paths and the oracle see the same rows
    HL = I.normal_values(seed, 9200, 0, N * D, 1.0, dtype)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    HL_t = (torch.tensor(HL.view(np.int16)).view(torch.bfloat16) if dtype == "bf16" else torch.tensor(HL)).cuda()
    dcu.dcu_set_tensor(ctx, dcu.DCU_T_H, L, HL_t)
    masked = (ids == shape.mask_id).to(torch.uint8)
    mpos = torch.nonzero(masked[0]).flatten()
    pos = torch.zeros((1, N), dtype=torch.int32, device="cuda")
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    dcu.commit_select(ctx, dcu.DCU_FRECHET, 0.1, masked, ids, pos, cnt)
    conf_ref = dcu.dcu_get_tensor(ctx, dcu.DCU_T_CONF)[mpos].cpu().numpy()
    assert dcu.dcu_status(ctx) == 0
    h_rows = HL_t.view(N, D)[mpos].contiguous()
    assert h_rows.dtype == tdt
    rows64 = I.as_f64(HL, dtype).reshape(N, D)[mpos.cpu().numpy()]
    c_o, _ = O.confidence(rows64, np.ones(D), LazyMatrix(shape, seed, "lm_head", vocab), shape.rms_eps)
    lm = LazyMatrix(shape, seed, "lm_head", vocab)
    for call in range(2):                      # two calls in a row share the static scratch
        conf, amax = dcu.dcu_lm_confidence_noalloc(h_rows, W["final_norm"], W["lm_head"], shape.rms_eps)
        torch.cuda.synchronize()
        conf, amax = conf.cpu().numpy(), amax.cpu().numpy()
        np.testing.assert_allclose(conf, conf_ref, rtol=1e-5, atol=0, err_msg=f"call {call} vs commit_select")
        np.testing.assert_allclose(conf, c_o, rtol=rtol, atol=0, err_msg=f"call {call} vs oracle")
        _argmax_ok(amax, rows64, lm, vocab, eps)
    ctx.close()


def test_noalloc_refuses_misaligned_and_oversized_inputs():
    shape = I.ModelShape(n_layers=1, d_model=256, n_heads=4, n_kv_heads=2, head_dim=64, d_ffn=512, vocab=5000,
                         dtype="bf16")
    W = I.device_weights(shape, 4)
    D = shape.d_model
    flat = torch.zeros(8 * D + 8, dtype=torch.bfloat16, device="cuda")
    misaligned = flat[1:1 + 8 * D].view(8, D)          # 2 bytes past a 16-byte boundary
    assert misaligned.data_ptr() % 16 != 0
    with pytest.raises(dcu.DcuError):
        dcu.dcu_lm_confidence_noalloc(misaligned, W["final_norm"], W["lm_head"])
    with pytest.raises(dcu.DcuError):
        dcu.dcu_lm_confidence_noalloc(torch.zeros((300, D), dtype=torch.bfloat16, device="cuda"),
                                      W["final_norm"], W["lm_head"])
    with pytest.raises(ValueError):                     # lm_head in another dtype than the rows
        dcu.dcu_lm_confidence_noalloc(torch.zeros((4, D), dtype=torch.float32, device="cuda"),
                                      W["final_norm"], W["lm_head"])
    # the library still works after the refusals
    conf, amax = dcu.dcu_lm_confidence_noalloc(flat[:8 * D].view(8, D), W["final_norm"], W["lm_head"])
    torch.cuda.synchronize()
    assert np.allclose(conf.cpu().numpy(), 1.0 / shape.vocab, rtol=1e-5)   # zero rows: uniform softmax
    assert np.all(amax.cpu().numpy() == 0)
