"""Adaptive parallel decoding (APD, [DLLM] "关键设计 3") on the GPU against the
oracle, teacher-forced at every commit: from the GPU's final-layer rows of
the candidates (this commit and the previous one) the oracle computes the
logits, the concentration c = 1 - p_second and the instability H = 1 -
cos(p, p_prev); the GPU's thresholds must equal the oracle's update of the
GPU's previous thresholds (within the propagated tolerance of c and H), and
the committed set must be exactly the oracle's APD selection fed the GPU's
own confidences and thresholds.  DCU steps between the commits change the
final-layer rows, so H is exercised."""
import numpy as np
import pytest
import torch

import oracle as O
from dynamic_layer_wise_b200 import dcu
from dynamic_layer_wise_b200 import inputs as I

from .helpers import oracle_weights, to_np

pytestmark = pytest.mark.gpu

SMALL_BF16 = I.ModelShape(n_layers=2, d_model=256, n_heads=4, n_kv_heads=2, head_dim=64, d_ffn=512, vocab=700,
                          dtype="bf16")


# tau0 sits just above the seeded models' confidences (about 0.0035 / 0.0032 and 0.0025 / 0.0029 for the two
# sequences), so that after the first update some positions pass their threshold and others do not
@pytest.mark.parametrize("shape,c_atol,h_atol,tau0", [(SMALL_BF16, 1e-4, 2e-3, 0.00358), (I.TOY, 1e-6, 1e-5, 0.00259)])
def test_apd_commits_teacher_forced(shape, c_atol, h_atol, tau0):
    seed, B, n_prompt, n_gen = 4, 2, 100, 40
    N, L, D, V = n_prompt + n_gen, shape.n_layers, shape.d_model, shape.vocab
    alpha, beta = 1e-4, 0.05
    w_o = oracle_weights(shape, seed)
    W = I.device_weights(shape, seed)
    ctx = dcu.dcu_create(W, I.cfg_dict(shape, B, N))
    with pytest.raises(dcu.DcuError):                 # the APD rule needs dcu_set_apd first
        dcu.commit_select(ctx, dcu.DCU_APD, 0.0, torch.zeros((B, N), dtype=torch.uint8, device="cuda"),
                          torch.zeros((B, N), dtype=torch.int32, device="cuda"),
                          torch.zeros((B, N), dtype=torch.int32, device="cuda"),
                          torch.zeros(B, dtype=torch.int32, device="cuda"))
    dcu.dcu_set_apd(ctx, alpha, beta, tau0)
    ids = np.stack([I.sequence_ids(seed, b, n_prompt, n_gen, V) for b in range(B)])
    t_ids = torch.tensor(ids, dtype=torch.int32).cuda()
    dcu.dcu_full_forward(ctx, t_ids)
    masked = (ids == shape.mask_id)
    t_m = torch.tensor(masked.astype(np.uint8)).cuda()
    pos = torch.zeros((B, N), dtype=torch.int32, device="cuda")
    cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
    tau_prev = np.full((B, N), tau0, np.float32)
    z_prev = [dict() for _ in range(B)]               # position -> oracle logits at the previous commit
    multi = 0
    for it in range(4):
        HL = np.asarray(to_np(dcu.dcu_get_tensor(ctx, dcu.DCU_T_H, L)), dtype=np.float64).reshape(B, N, D)
        m_before = masked.copy()
        dcu.commit_select(ctx, dcu.DCU_APD, 0.0, t_m, t_ids, pos, cnt)
        assert dcu.dcu_status(ctx) == 0
        conf = dcu.dcu_get_tensor(ctx, dcu.DCU_T_CONF).cpu().numpy().reshape(B, N)
        amax = dcu.dcu_get_tensor(ctx, dcu.DCU_T_ARGMAX).cpu().numpy().reshape(B, N)
        tau = dcu.dcu_get_tensor(ctx, dcu.DCU_T_APD_TAU).cpu().numpy().reshape(B, N)
        cg = dcu.dcu_get_tensor(ctx, dcu.DCU_T_APD_C).cpu().numpy().reshape(B, N)
        hg = dcu.dcu_get_tensor(ctx, dcu.DCU_T_APD_H).cpu().numpy().reshape(B, N)
        gpos, gcnt = pos.cpu().numpy(), cnt.cpu().numpy()
        for b in range(B):
            mp = np.flatnonzero(m_before[b])
            z = O.logits(HL[b][mp], w_o.final_norm, w_o.lm_head, shape.rms_eps)
            c_o, h_o = O.apd_signals(z, [z_prev[b].get(int(p)) for p in mp])
            np.testing.assert_allclose(cg[b, mp], c_o, rtol=0, atol=c_atol, err_msg=f"commit {it}: c")
            np.testing.assert_allclose(hg[b, mp], h_o, rtol=0, atol=h_atol, err_msg=f"commit {it}: H")
            if it == 0:
                assert np.all(hg[b, mp] == 0.0)
            tau_o = O.apd_update(tau_prev[b, mp], c_o, h_o, alpha, beta)
            np.testing.assert_allclose(tau[b, mp], tau_o, rtol=0, atol=alpha * c_atol + beta * h_atol + 1e-6)
            # the selector fed the GPU's own confidences and thresholds: exact
            ref = O.apd_commit(conf[b], amax[b], m_before[b], ids[b], tau[b])
            np.testing.assert_array_equal(gpos[b, :gcnt[b]], ref[0], err_msg=f"commit {it}: committed positions")
            multi += int(gcnt[b] > 1)
            ids[b], masked[b] = ref[1], ref[2]
            for k, p in enumerate(mp):
                z_prev[b][int(p)] = z[k]
            tau_prev[b] = tau[b]
        # the next DCU step reads the committed positions as keys
        t_ids.copy_(torch.tensor(ids, dtype=torch.int32))
        dcu.dcu_step(ctx, t_ids, pos, cnt, 6, 4)
        assert dcu.dcu_status(ctx) == 0
    assert multi > 0, "no commit passed more than one threshold: the adaptive path was not exercised"
    # a dense forward starts a new generation: thresholds back to tau0
    dcu.dcu_full_forward(ctx, t_ids)
    tau = dcu.dcu_get_tensor(ctx, dcu.DCU_T_APD_TAU).cpu().numpy()
    assert np.all(tau == np.float32(tau0))
    ctx.close()
