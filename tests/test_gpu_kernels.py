"""Per-kernel parity of the CUDA path (through the C ABI) with the oracle on
seeded synthetic inputs."""
import numpy as np
import pytest
import torch

import oracle as O
from dynamic_layer_wise_b200 import dcu
from dynamic_layer_wise_b200 import inputs as I

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("M,K,Nout", [(1, 64, 128), (17, 256, 1000), (65, 4096, 384), (128, 512, 256),
                                      (130, 1024, 640), (300, 128, 200), (1024, 256, 128),
                                      (520, 192, 130), (777, 128, 384)])
def test_linear_parity(dtype, M, K, Nout):
    """The recompute GEMM (tcgen05 for bf16) against an fp64 product of the same
    stored values; fp32 accumulation bounds the error by ~K * 2^-24 * sum|x||w|."""
    rng = np.random.default_rng(M * 7 + K)
    x = O.store(rng.standard_normal((M, K)), dtype)
    w = O.store(rng.standard_normal((Nout, K)) * 0.02, dtype)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    y = dcu.dcu_linear(torch.tensor(x).to(tdt).cuda(), torch.tensor(w).to(tdt).cuda()).cpu().numpy()
    ref = x @ w.T
    bound = np.abs(x) @ np.abs(w).T * (K * 2.0 ** -23 + 1e-7)
    assert np.all(np.abs(y - ref) <= bound), float(np.max(np.abs(y - ref) / bound))


def test_device_generator_matches_host_bits():
    for dtype, tdt in (("bf16", torch.bfloat16), ("f32", torch.float32)):
        for seed, tid, start, n in ((0, 1, 0, 100003), (7, 123, 5_000_000, 4099), (2**31 + 5, 77, 2**33, 1000)):
            t = torch.empty(n, dtype=tdt, device="cuda")
            I.device_normal_(t, seed, tid, 0.02, start=start)
            host = I.normal_values(seed, tid, start, n, 0.02, dtype)
            if dtype == "bf16":
                got = t.view(torch.int16).cpu().numpy().view(np.uint16)
            else:
                got = t.cpu().numpy()
            np.testing.assert_array_equal(got.view(np.uint16 if dtype == "bf16" else np.uint32),
                                          host.view(np.uint16 if dtype == "bf16" else np.uint32))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("D", [8, 256, 4096, 3584])
def test_cosine_distance_parity(dtype, D):
    rows = 37
    rng = np.random.default_rng(D)
    x = rng.standard_normal((rows, D))
    y = x + rng.standard_normal((rows, D)) * rng.choice([0.0, 1e-3, 0.1, 1.0], (rows, 1))
    y[3] = -x[3]
    x[5] = 0.0
    x[6] = 0.0
    y[6] = 0.0
    g = rng.uniform(0.5, 1.5, D)
    xs, ys = O.store(x, dtype), O.store(y, dtype)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    tx = torch.tensor(xs, dtype=torch.float64).to(tdt).cuda()
    ty = torch.tensor(ys, dtype=torch.float64).to(tdt).cuda()
    d = dcu.dcu_cosine_distance(tx, ty, torch.tensor(g, dtype=torch.float32).cuda()).cpu().numpy()
    ref = O.cosine_distance(xs, ys, np.asarray(torch.tensor(g, dtype=torch.float32), dtype=np.float64))
    np.testing.assert_allclose(d, ref.astype(np.float32), rtol=0, atol=2e-7)
    assert d[0] == 0.0 or not np.array_equal(xs[0], ys[0])
    assert d[5] == 1.0 and d[6] == 0.0


def test_budget_split_parity():
    rng = np.random.default_rng(1)
    for trial in range(40):
        B, L = int(rng.integers(1, 5)), int(rng.integers(1, 80))
        Bl = int(rng.integers(0, 200))
        s = rng.exponential(1.0, (B, L)).astype(np.float32)
        s[rng.random((B, L)) < 0.3] = 0.0
        if trial % 5 == 0:
            s[:] = np.float32(0.25)                       # equal fractional parts: ties -> lower layer
        if trial % 7 == 0:
            s[0] = 0.0                                    # all-zero row -> uniform
        uniform = trial % 11 == 0
        got = dcu.dcu_budget_split(torch.tensor(s).cuda(), Bl, uniform).cpu().numpy()
        for b in range(B):
            ref = O.split_budget(s[b], Bl, uniform)
            np.testing.assert_array_equal(got[b], ref)
            assert got[b].sum() == Bl * L


def _select_case(rng, B, N, ties):
    d = (rng.choice([0.0, 0.125, 0.5], (B, N)) if ties else rng.exponential(0.01, (B, N))).astype(np.float32)
    d[rng.random((B, N)) < 0.5] = 0.0
    keys = np.zeros((B, N), dtype=np.int32)
    nk = np.zeros(B, dtype=np.int32)
    for b in range(B):
        k = int(rng.integers(0, min(N, 6) + 1))
        keys[b, :k] = rng.choice(N, k, replace=False)
        nk[b] = k
    budgets = rng.integers(0, N + 5, B).astype(np.int32)
    return d, keys, nk, budgets


@pytest.mark.parametrize("N", [1, 5, 64, 257, 1024, 1531, 8192, 16384])
def test_select_tokens_parity(N):
    rng = np.random.default_rng(N)
    for trial in range(6):
        B = int(rng.integers(1, 4))
        d, keys, nk, budgets = _select_case(rng, B, N, ties=trial % 2 == 0)
        bw = int(rng.integers(0, 40))
        mode = trial % 2
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        idx, cnt, s = dcu.dcu_select_tokens(torch.tensor(d).cuda(), torch.tensor(keys).cuda(),
                                            torch.tensor(nk).cuda(), torch.tensor(budgets).cuda(), bw, mode, status)
        idx, cnt, s = idx.cpu().numpy(), cnt.cpu().numpy(), s.cpu().numpy()
        assert status.item() == 0
        for b in range(B):
            ref = O.select_rows(d[b], list(keys[b, :nk[b]]), bw, int(budgets[b]), mode)
            assert cnt[b] == len(ref)
            np.testing.assert_array_equal(idx[b, :cnt[b]], ref)
            assert s[b] == O.layer_dynamics(d[b])


def test_select_tokens_flags_bad_keys():
    d = torch.zeros((1, 32), dtype=torch.float32, device="cuda")
    keys = torch.tensor([[3, 40, -1] + [0] * 29], dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx, cnt, _ = dcu.dcu_select_tokens(d, keys, torch.tensor([3], dtype=torch.int32, device="cuda"),
                                        torch.tensor([2], dtype=torch.int32, device="cuda"), 4, 0, status)
    assert status.item() & dcu.DCU_ST_BAD_KEY
    ref = O.select_rows(np.zeros(32, np.float32), [3], 4, 2, 0)
    np.testing.assert_array_equal(idx.cpu().numpy()[0, :cnt.item()], ref)


def _commit_case(rng, B, N, kind):
    if kind == "profile":
        c = rng.beta(12, 1, (B, N))
    elif kind == "ties":
        c = rng.choice([0.5, 0.9, 0.99], (B, N))
    else:
        c = rng.uniform(1e-5, 1e-3, (B, N))
    c = c.astype(np.float32)
    masked = (rng.random((B, N)) < 0.6).astype(np.uint8)
    amax = rng.integers(0, 1000, (B, N)).astype(np.int32)
    ids = rng.integers(0, 1000, (B, N)).astype(np.int32)
    return c, masked, amax, ids


@pytest.mark.parametrize("rule,param", [(O.RULE_FRECHET, 0.1), (O.RULE_FRECHET, 0.0), (O.RULE_FRECHET, 0.3),
                                        (O.RULE_THRESHOLD, 0.9), (O.RULE_FACTOR, 0.9), (O.RULE_FACTOR, 0.75)])
@pytest.mark.parametrize("N", [1, 7, 256, 1000, 4096])
def test_commit_rule_parity(rule, param, N):
    rng = np.random.default_rng(N * 10 + rule)
    for kind in ("profile", "ties", "flat_low"):
        B = int(rng.integers(1, 4))
        c, masked, amax, ids = _commit_case(rng, B, N, kind)
        tm, ti = torch.tensor(masked).cuda(), torch.tensor(ids).cuda()
        pos = torch.full((B, N), -1, dtype=torch.int32, device="cuda")
        cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
        dcu.dcu_commit_rule(rule, param, torch.tensor(c).cuda(), torch.tensor(amax).cuda(), tm, ti, pos, cnt)
        pos, cnt, tm, ti = pos.cpu().numpy(), cnt.cpu().numpy(), tm.cpu().numpy(), ti.cpu().numpy()
        for b in range(B):
            rp, rid, rm = O.commit(c[b], amax[b], masked[b], ids[b], rule, param)
            assert cnt[b] == len(rp)
            np.testing.assert_array_equal(pos[b, :cnt[b]], rp)
            np.testing.assert_array_equal(ti[b], rid)
            np.testing.assert_array_equal(tm[b].astype(bool), rm)


def test_commit_rule_worked_profile():
    prof = np.array([0.99, 0.95, 0.82, 0.78, 0.74], dtype=np.float32)
    for rule, param, want in ((O.RULE_FRECHET, 0.1, 4), (O.RULE_FACTOR, 0.9, 3), (O.RULE_FRECHET, 0.3, 4),
                              (O.RULE_FACTOR, 0.7, 2), (O.RULE_THRESHOLD, 0.9, 2)):
        c = torch.tensor(prof[::-1].copy())[None].cuda()          # shuffled order on the device
        masked = torch.ones((1, 5), dtype=torch.uint8, device="cuda")
        ids = torch.zeros((1, 5), dtype=torch.int32, device="cuda")
        amax = torch.arange(5, dtype=torch.int32, device="cuda")[None] + 10
        pos = torch.zeros((1, 5), dtype=torch.int32, device="cuda")
        cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
        dcu.dcu_commit_rule(rule, param, c, amax, masked, ids, pos, cnt)
        assert cnt.item() == want
        assert list(pos[0, :want].cpu().numpy()) == [4, 3, 2, 1, 0][:want]


def test_bounded_wait_expires_and_reports_timeout():
    """Failure detection without a fault: a wait on a barrier that nothing
    arrives on gives up after its wall-clock bound (~1 s), reports
    DCU_ST_TIMEOUT and the kernel finishes; the context keeps working."""
    import time
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    dcu.dcu_selftest_wait_timeout(status)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert status.item() == dcu.DCU_ST_TIMEOUT
    assert 0.5 < dt < 10.0
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum().item()) == 8.0                  # the context is usable afterwards


def test_options_refuse_bad_values():
    """dcu_set_option: unknown options and values out of range are refused
    (DCU_EINVAL); the context stays usable and a valid setting is accepted."""
    shape = I.ModelShape(n_layers=1, d_model=256, n_heads=4, n_kv_heads=2, head_dim=64, d_ffn=512, vocab=500,
                         dtype="bf16")
    ctx = dcu.dcu_create(I.device_weights(shape, 2), I.cfg_dict(shape, 1, 64))
    for opt, val in [(dcu.DCU_OPT_ATTENTION, 2), (dcu.DCU_OPT_ATTENTION, -1), (dcu.DCU_OPT_FUSED_EPILOGUE, 3),
                     (dcu.DCU_OPT_L2_PREFETCH, -1), (dcu.DCU_OPT_L2_PREFETCH, 4097), (dcu.DCU_OPT_GEMM_SMEM_KB, 135),
                     (dcu.DCU_OPT_GEMM_SMEM_KB, 221), (99, 0)]:
        with pytest.raises(dcu.DcuError):
            dcu.dcu_set_option(ctx, opt, val)
    dcu.dcu_set_option(ctx, dcu.DCU_OPT_ATTENTION, dcu.DCU_ATTN_MMA_SYNC)
    dcu.dcu_set_option(ctx, dcu.DCU_OPT_ATTENTION, dcu.DCU_ATTN_TCGEN05)
    dcu.dcu_set_option(ctx, dcu.DCU_OPT_GEMM_SMEM_KB, 160)
    ctx.close()
