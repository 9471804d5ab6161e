"""Pins of the fp64 oracle against facts that do not come from the oracle itself:
closed forms, invariants, library routines, brute force and the worked profile
printed on the Fast-dLLM++ page."""
import itertools
import math
import os

import numpy as np
import pytest
import scipy.spatial.distance
import scipy.special
import torch
import torch.nn.functional as F

import oracle as O
from dynamic_layer_wise_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, *v = line.split()
            out[k] = [float(x) for x in v]
    return out


# ------------------------------------------------------------------ E1: cosine distance

def test_cosine_distance_closed_forms():
    rng = np.random.default_rng(0)
    g = np.ones(64)
    x = rng.standard_normal(64)
    assert O.cosine_distance(x, x, g)[0] == 0.0                        # identical -> 0
    assert O.cosine_distance(x, -x, g)[0] == pytest.approx(2.0, abs=1e-15)   # antiparallel -> 2
    e1, e2 = np.eye(64)[0], np.eye(64)[1]
    assert O.cosine_distance(e1, e2, g)[0] == pytest.approx(1.0, abs=1e-15)  # orthogonal -> 1
    y = rng.standard_normal(64)
    for a in (1e-3, 0.5, 7.0, 1e4):                                     # positive scale invariance
        assert O.cosine_distance(x, a * y, g)[0] == pytest.approx(O.cosine_distance(x, y, g)[0], rel=1e-12)
    assert O.cosine_distance(np.zeros(8), np.zeros(8), np.ones(8))[0] == 0.0
    assert O.cosine_distance(np.zeros(8), np.ones(8), np.ones(8))[0] == 1.0


def test_cosine_distance_matches_scipy_with_gain():
    rng = np.random.default_rng(1)
    for _ in range(20):
        x, y, g = rng.standard_normal(33), rng.standard_normal(33), rng.uniform(0.2, 3.0, 33)
        ref = scipy.spatial.distance.cosine(g * x, g * y)
        assert O.cosine_distance(x, y, g)[0] == pytest.approx(ref, abs=1e-13)


def test_layer_dynamics_is_mean():
    d = np.array([0.5, 0.25, 0.0, 1.0], dtype=np.float32)
    assert O.layer_dynamics(d) == np.float32(0.4375)


# ------------------------------------------------------------------ E3: budget split

def test_budget_uniform_and_first_step():
    assert list(O.split_budget(np.zeros(8, np.float32), 32, uniform=False)) == [32] * 8
    s = np.linspace(0.1, 1.0, 8).astype(np.float32)
    assert list(O.split_budget(s, 16, uniform=True)) == [16] * 8
    assert list(O.split_budget(np.full(5, 0.3, np.float32), 7, uniform=False)) == [7] * 5


def test_budget_hand_example():
    # T = 2 * 3 = 6; q = (1.5, 1.5, 3.0): floors (1, 1, 3), one left, equal fractions -> lower layer.
    assert list(O.split_budget(np.array([1, 1, 2], np.float32), 2, False)) == [2, 1, 3]
    # T = 4 * 4 = 16; q = 16 * (0.1, 0.2, 0.3, 0.4) = (1.6, 3.2, 4.8, 6.4): floors 14, two left -> layers 0, 2.
    assert list(O.split_budget(np.array([0.1, 0.2, 0.3, 0.4], np.float32), 4, False)) == [2, 3, 5, 6]


def test_budget_conservation_and_quota():
    rng = np.random.default_rng(2)
    for trial in range(300):
        L = int(rng.integers(1, 40))
        Bl = int(rng.integers(0, 100))
        s = rng.exponential(1.0, L).astype(np.float32)
        s[rng.random(L) < 0.2] = 0.0
        b = O.split_budget(s, Bl, False)
        assert b.sum() == Bl * L
        if s.astype(np.float64).sum() > 0:
            q = Bl * L * s.astype(np.float64) / s.astype(np.float64).sum()
            assert np.all(b >= np.floor(q) - 1e-9) and np.all(b <= np.ceil(q) + 1e-9)   # quota property


def test_budget_is_min_l1_apportionment_bruteforce():
    """Largest remainder is the integer vector with the given total closest to the
    real quotas in L1 (brute force over all compositions for tiny L, T)."""
    rng = np.random.default_rng(3)
    for _ in range(60):
        L = int(rng.integers(2, 5))
        Bl = int(rng.integers(1, 4))
        T = Bl * L
        s = rng.uniform(0.01, 1.0, L).astype(np.float32)
        q = T * s.astype(np.float64) / s.astype(np.float64).sum()
        best = min(sum(abs(c[l] - q[l]) for l in range(L))
                   for c in itertools.product(range(T + 1), repeat=L) if sum(c) == T)
        b = O.split_budget(s, Bl, False)
        assert sum(abs(b[l] - q[l]) for l in range(L)) == pytest.approx(best, abs=1e-9)


# ------------------------------------------------------------------ E4 + top-k

def test_window_closed_forms():
    assert O.window_mask([10], 4, 30, 0).sum() == 5            # B_w + 1 positions (inclusive bounds)
    assert O.window_mask([10], 4, 30, 1).sum() == 4            # B_w positions
    assert list(np.flatnonzero(O.window_mask([0, 10], 4, 20, 0))) == [0, 1, 2, 8, 9, 10, 11, 12]
    assert list(np.flatnonzero(O.window_mask([0, 10], 4, 20, 1))) == [0, 1, 8, 9, 10, 11]
    assert list(np.flatnonzero(O.window_mask([19], 6, 20, 0))) == [16, 17, 18, 19]
    assert O.window_mask([3, 4], 0, 20, 0).sum() == 0          # B_w = 0: no window
    assert O.window_mask([5, 7], 4, 20, 0).sum() == 7          # overlapping windows union: 3..9


def _brute_select(d, keys, bw, budget, mode):
    N = len(d)
    W = set()
    if bw > 0:
        h = bw // 2
        for p in keys:
            hi = p + h if mode == 0 else p - h + bw - 1
            W.update(i for i in range(p - h, hi + 1) if 0 <= i < N)
    rest = sorted((i for i in range(N) if i not in W), key=lambda i: (-float(d[i]), i))
    k = min(budget, N - len(W))
    return sorted(W | set(rest[:k]))


def test_select_bruteforce_with_ties():
    rng = np.random.default_rng(4)
    for trial in range(300):
        N = int(rng.integers(1, 70))
        d = rng.choice([0.0, 0.25, 0.5, 1.0], N) if trial % 2 else rng.uniform(0, 2, N)
        d = d.astype(np.float32)
        d[rng.random(N) < 0.4] = 0.0
        keys = [int(k) for k in rng.choice(N, size=min(N, int(rng.integers(0, 4))), replace=False)]
        bw = int(rng.integers(0, 9))
        budget = int(rng.integers(0, N + 3))
        mode = int(rng.integers(0, 2))
        got = list(O.select_rows(d, keys, bw, budget, mode))
        assert got == _brute_select(d, keys, bw, budget, mode)
        W = O.window_mask(keys, bw, N, mode)
        assert len(got) == min(N, int(W.sum()) + budget)


# ------------------------------------------------------------------ Fréchet / threshold / factor

def test_frechet_worked_profile_from_page():
    g = _golden("frechet_profile.txt")
    prof = np.array(g["profile"], dtype=np.float32)
    delta = g["claim_delta"][0]
    assert O.frechet_count(prof, delta) == int(g["claim_frechet_n"][0])
    assert O.factor_count(prof, 1.0 - delta) == int(g["claim_matched_factor_n"][0])


def test_frechet_profile_values_by_hand():
    prof = np.array([0.99, 0.95, 0.82, 0.78, 0.74])
    L, U, G = O.frechet_profile(prof)
    # L_n = sum - (n-1): 0.99, 0.94, 0.76, 0.54, 0.28;  U_n = 1 - c_(n)
    np.testing.assert_allclose(L, [0.99, 0.94, 0.76, 0.54, 0.28], atol=1e-12)
    np.testing.assert_allclose(U, [0.01, 0.05, 0.18, 0.22, 0.26], atol=1e-12)
    np.testing.assert_allclose(G, [0.98, 0.89, 0.58, 0.32, 0.02], atol=1e-12)
    p32 = prof.astype(np.float32)
    assert O.frechet_count(p32, 0.1) == 4
    assert O.factor_count(p32, 0.9) == 3          # (n+1)(1-c): 0.02, 0.15, 0.72, 1.10, 1.56
    assert O.frechet_count(p32, 0.25) == 4
    assert O.factor_count(p32, 0.75) == 3
    assert O.frechet_count(p32, 0.99) == 1        # nothing passes -> 1 (progress)
    assert O.threshold_count(p32, 0.9) == 2
    assert O.threshold_count(p32, 0.999) == 1     # nothing passes -> top one
    assert O.frechet_count(np.zeros(0, np.float32), 0.1) == 0


def test_frechet_decomposition_and_dominance():
    """G_n = F_n + B_n while L_n > 0 (Proposition 4.3); Fréchet(delta) commits at
    least as many as factor(1 - delta), strictly more exactly when
    F_n <= delta < F_n + B_n at its n* (Corollary 4.4); flat profiles tie."""
    rng = np.random.default_rng(5)
    for _ in range(500):
        m = int(rng.integers(1, 40))
        c = np.sort(rng.beta(8, 1, m))[::-1].astype(np.float32)
        cd = c.astype(np.float64)
        Ls, _, G = O.frechet_profile(cd)
        for n in range(1, m + 1):
            Fn = (n + 1) * cd[n - 1] - n
            Bn = float(np.sum(cd[:n - 1] - cd[n - 1]))
            if Ls[n - 1] > 0:
                assert G[n - 1] == pytest.approx(Fn + Bn, abs=1e-12)
        delta = float(rng.uniform(0.0, 0.5))
        nf = O.frechet_count(c, delta)
        nq = O.factor_count(c, 1.0 - delta)
        assert nf >= nq
        if nf > nq:
            n = nf
            Fn = (n + 1) * cd[n - 1] - n
            Bn = float(np.sum(cd[:n - 1] - cd[n - 1]))
            assert Fn <= delta + 1e-12 and delta < Fn + Bn + 1e-12
        flat = np.full(m, np.float32(rng.uniform(0.5, 1.0)))
        assert O.frechet_count(flat, delta) == O.factor_count(flat, 1.0 - delta)


def test_commit_hand_case():
    c = np.array([0.1, 0.9, 0.5, 0.9, 0.2, 0.95], dtype=np.float32)
    masked = np.array([1, 1, 1, 1, 0, 1], dtype=bool)
    amax = np.array([7, 8, 9, 10, 11, 12])
    ids = np.array([5, 5, 5, 5, 3, 5])
    # sorted masked: pos5 (0.95), pos1 (0.9), pos3 (0.9), pos2 (0.5), pos0 (0.1);
    # threshold 0.85 -> 3 positions (tie 0.9 broken by position).
    pos, nid, nm = O.commit(c, amax, masked, ids, O.RULE_THRESHOLD, 0.85)
    assert list(pos) == [5, 1, 3]
    assert list(nid) == [5, 8, 5, 10, 3, 12]
    assert list(nm) == [True, False, True, False, False, False]
    pos, _, _ = O.commit(c, amax, np.zeros(6, bool), ids, O.RULE_FRECHET, 0.1)
    assert len(pos) == 0


# ------------------------------------------------------------------ softmax-max

def test_confidence_matches_scipy_softmax_and_argmax_tie():
    rng = np.random.default_rng(6)
    D, V = 16, 37
    lm = rng.standard_normal((V, D))
    lm[20] = lm[9]                                  # planted exact tie between ids 9 and 20
    h = rng.standard_normal((5, D))
    g = np.ones(D)
    c, a = O.confidence(h, g, lm, 1e-5)
    hn = F.rms_norm(torch.tensor(h), (D,), torch.tensor(g), 1e-5).numpy()
    z = hn @ lm.T
    np.testing.assert_allclose(c, scipy.special.softmax(z, axis=1).max(axis=1).astype(np.float32), rtol=1e-6)
    assert list(a) == list(np.argmax(z, axis=1))
    hz = lm[9] * 50.0                               # makes ids 9 and 20 the joint maximum
    _, a2 = O.confidence(hz[None, :], g, lm, 1e-5)
    assert a2[0] == 9


# ------------------------------------------------------------------ model pieces vs torch library routines

def test_rmsnorm_matches_torch():
    rng = np.random.default_rng(7)
    x, g = rng.standard_normal((4, 24)), rng.uniform(0.5, 2.0, 24)
    ref = F.rms_norm(torch.tensor(x), (24,), torch.tensor(g), 1e-5).numpy()
    np.testing.assert_allclose(O.rmsnorm(x, g, 1e-5), ref, rtol=1e-13)


def test_silu_matches_torch():
    x = np.linspace(-20, 20, 101)
    np.testing.assert_allclose(O.silu(x), F.silu(torch.tensor(x)).numpy(), rtol=1e-13, atol=1e-300)


def test_attention_matches_torch_sdpa_gqa():
    rng = np.random.default_rng(8)
    M, N, H, Hkv, hd = 5, 11, 8, 2, 16
    q = rng.standard_normal((M, H, hd))
    K = rng.standard_normal((Hkv, N, hd))
    V = rng.standard_normal((Hkv, N, hd))
    out = O.attend(q, K, V)
    tq = torch.tensor(q).permute(1, 0, 2)[None]                    # [1, H, M, hd]
    rep = H // Hkv
    tk = torch.tensor(K).repeat_interleave(rep, dim=0)[None]       # kv head of query head h = h // rep
    tv = torch.tensor(V).repeat_interleave(rep, dim=0)[None]
    ref = F.scaled_dot_product_attention(tq, tk, tv)[0].permute(1, 0, 2).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_rope_invariants():
    rng = np.random.default_rng(9)
    hd = 16
    q = rng.standard_normal((1, 1, hd))
    k = rng.standard_normal((1, 1, hd))
    np.testing.assert_array_equal(O.rope(q, np.array([0]), 10000.0), q)          # position 0: identity
    for p in (1, 5, 300):                                                       # norm-preserving
        assert np.linalg.norm(O.rope(q, np.array([p]), 10000.0)) == pytest.approx(np.linalg.norm(q), rel=1e-13)
    dots = []
    for m, n in ((3, 1), (10, 8), (102, 100)):                                  # depends on m - n only
        dots.append(float(np.sum(O.rope(q, np.array([m]), 10000.0) * O.rope(k, np.array([n]), 10000.0))))
    assert dots[0] == pytest.approx(dots[1], rel=1e-10) and dots[1] == pytest.approx(dots[2], rel=1e-10)
    # head_dim 2: a plain rotation by the position (theta^0 = 1)
    v = np.array([[[1.0, 0.0]]])
    np.testing.assert_allclose(O.rope(v, np.array([2]), 10000.0)[0, 0], [math.cos(2), math.sin(2)], atol=1e-15)


def _tiny_model(seed=0, L=2, D=32, H=4, Hkv=2, hd=8, Fd=48, V=50, dtype="f32", gains=False):
    cfg = O.Config(n_layers=L, d_model=D, n_heads=H, n_kv_heads=Hkv, head_dim=hd, d_ffn=Fd, vocab=V, dtype=dtype)
    rng = np.random.default_rng(seed)
    def mat(o, i):
        return O.store(rng.normal(0, 0.3, (o, i)), dtype)
    gain = (lambda: rng.uniform(0.5, 1.5, D)) if gains else (lambda: np.ones(D))
    layers = [dict(attn_norm=gain(), wq=mat(H * hd, D), wk=mat(Hkv * hd, D), wv=mat(Hkv * hd, D),
                   wo=mat(D, H * hd), ffn_norm=gain(), w_gate=mat(Fd, D), w_up=mat(Fd, D), w_down=mat(D, Fd))
              for _ in range(L)]
    w = O.Weights(embed=mat(V, D), lm_head=mat(V, D), final_norm=gain(), layers=layers)
    return cfg, w


def test_full_forward_matches_torch_layer_stack():
    cfg, w = _tiny_model(gains=True)
    N = 9
    ids = np.array([[3, 7, 1, 0, 49, 49, 12, 5, 8]])
    st = O.full_forward(w, cfg, ids)
    t = lambda a: torch.tensor(np.asarray(a, dtype=np.float64))
    h = t(w.embed[ids[0]])
    hd, H, Hkv = cfg.head_dim, cfg.n_heads, cfg.n_kv_heads
    pos = np.arange(N)
    for l, lw in enumerate(w.layers):
        n = F.rms_norm(h, (cfg.d_model,), t(lw["attn_norm"]), cfg.rms_eps)
        q = F.linear(n, t(lw["wq"])).reshape(N, H, hd).numpy()
        k = F.linear(n, t(lw["wk"])).reshape(N, Hkv, hd).numpy()
        v = F.linear(n, t(lw["wv"])).reshape(N, Hkv, hd)
        q, k = t(O.rope(q, pos, cfg.rope_theta)), t(O.rope(k, pos, cfg.rope_theta))
        rep = H // Hkv
        a = F.scaled_dot_product_attention(q.permute(1, 0, 2)[None], k.permute(1, 0, 2).repeat_interleave(rep, 0)[None],
                                           v.permute(1, 0, 2).repeat_interleave(rep, 0)[None])[0].permute(1, 0, 2)
        h = h + F.linear(a.reshape(N, H * hd), t(lw["wo"]))
        m = F.rms_norm(h, (cfg.d_model,), t(lw["ffn_norm"]), cfg.rms_eps)
        h = h + F.linear(F.silu(F.linear(m, t(lw["w_gate"]))) * F.linear(m, t(lw["w_up"])), t(lw["w_down"]))
        np.testing.assert_allclose(st.H[l + 1][0], h.numpy().astype(np.float32), rtol=2e-6, atol=1e-6)
        h = t(st.H[l + 1][0])      # continue from the stored (float32-rounded) value


# ------------------------------------------------------------------ storage rounding

def test_bf16_store_matches_torch_on_float32_inputs():
    rng = np.random.default_rng(10)
    x = (rng.standard_normal(20000) * 10.0 ** rng.integers(-6, 6, 20000)).astype(np.float32)
    ref = torch.tensor(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.store(x.astype(np.float64), "bf16"), ref)
    # ties to even: 1 + 2^-8 lies halfway between 1 and 1 + 2^-7 -> 1; 1 + 3*2^-8 -> 1 + 2^-6
    assert O.store(np.array([1 + 2.0 ** -8]), "bf16")[0] == 1.0
    assert O.store(np.array([1 + 3 * 2.0 ** -8]), "bf16")[0] == 1 + 2.0 ** -6
    # generator's bf16 rounding (a separate implementation) agrees on fp64 inputs
    y = rng.standard_normal(20000) * 0.05
    np.testing.assert_array_equal(I.as_f64(I.f64_to_bf16_bits(y), "bf16"), O.store(y, "bf16"))


# ------------------------------------------------------------------ DCU step invariants

def _ids_and_keys(V, N, n_gen, seed=0, n_unmask=2):
    rng = np.random.default_rng(seed)
    ids0 = np.concatenate([rng.integers(0, V - 1, N - n_gen), np.full(n_gen, V - 1)])
    keys = np.sort(rng.choice(np.arange(N - n_gen, N), n_unmask, replace=False))
    ids1 = ids0.copy()
    ids1[keys] = rng.integers(0, V - 1, n_unmask)
    return ids0[None], ids1[None], [list(keys)]


def test_dcu_full_budget_equals_dense_forward():
    """B^l = N with no window on the first cached (uniform) step recomputes every
    row of every layer, so it must equal a dense forward on the new ids."""
    cfg, w = _tiny_model(seed=1, L=3, gains=True)
    N = 12
    ids0, ids1, keys = _ids_and_keys(cfg.vocab, N, 5)
    st0 = O.full_forward(w, cfg, ids0)
    st1, tr = O.dcu_step(w, cfg, st0, ids1, keys, B_layer=N, B_window=0)
    dense = O.full_forward(w, cfg, ids1)
    for l in range(cfg.n_layers + 1):
        np.testing.assert_allclose(st1.H[l], dense.H[l], rtol=0, atol=1e-6)
    for l in range(cfg.n_layers):
        np.testing.assert_allclose(st1.K[l], dense.K[l], rtol=0, atol=1e-6)
        np.testing.assert_allclose(st1.V[l], dense.V[l], rtol=0, atol=1e-6)
        assert list(tr.sel[l][0]) == list(range(N))


def test_dcu_zero_budget_keeps_cache():
    cfg, w = _tiny_model(seed=2, L=3)
    N = 12
    ids0, ids1, keys = _ids_and_keys(cfg.vocab, N, 5)
    st0 = O.full_forward(w, cfg, ids0)
    st1, tr = O.dcu_step(w, cfg, st0, ids1, keys, B_layer=0, B_window=0)
    assert not np.array_equal(st1.H[0], st0.H[0])          # the key rows' embeddings changed
    for l in range(1, cfg.n_layers + 1):
        np.testing.assert_array_equal(st1.H[l], st0.H[l])
    for l in range(cfg.n_layers):
        np.testing.assert_array_equal(st1.K[l], st0.K[l])
        np.testing.assert_array_equal(st1.V[l], st0.V[l])
        assert len(tr.sel[l][0]) == 0


def test_dcu_stuck_in_mud_and_budget_conservation():
    """d^{l+1} = 0 exactly at every row that layer l did not recompute, and the
    per-layer budgets of every step sum to B_layer * L."""
    cfg, w = _tiny_model(seed=3, L=4, dtype="bf16")
    N = 24
    ids0, ids1, keys = _ids_and_keys(cfg.vocab, N, 8, seed=3)
    st, _ = O.full_forward(w, cfg, ids0), None
    B_layer, Bw = 3, 2
    for step in range(3):
        st, tr = O.dcu_step(w, cfg, st, ids1 if step == 0 else st.ids, keys if step == 0 else [[]], B_layer, Bw)
        assert tr.budgets.sum() == B_layer * cfg.n_layers
        for l in range(cfg.n_layers - 1):
            off = np.setdiff1d(np.arange(N), tr.sel[l][0])
            assert np.all(tr.d[l + 1][0][off] == 0.0)
        d0 = tr.d[0][0]
        assert (np.count_nonzero(d0) == len(keys[0])) if step == 0 else (np.count_nonzero(d0) == 0)
    assert not st.first


def test_rope_matches_transformers_rotate_half():
    """The rotate-half RoPE of the Llama implementation in ``transformers`` (a
    library routine) with theta = 10000."""
    from transformers import LlamaConfig
    from transformers.models.llama import modeling_llama as ml
    hd, H, N = 16, 2, 7
    cfg = LlamaConfig(hidden_size=hd * H, num_attention_heads=H, num_key_value_heads=H, rope_theta=10000.0)
    emb = ml.LlamaRotaryEmbedding(cfg)
    rng = np.random.default_rng(11)
    q = rng.standard_normal((N, H, hd))
    k = rng.standard_normal((N, H, hd))
    pos = torch.arange(N)[None]
    x = torch.tensor(q).permute(1, 0, 2)[None]
    cos, sin = emb(x, pos)
    rq, rk = ml.apply_rotary_pos_emb(x, torch.tensor(k).permute(1, 0, 2)[None], cos.double(), sin.double())
    np.testing.assert_allclose(O.rope(q, np.arange(N), 10000.0), rq[0].permute(1, 0, 2).numpy(), rtol=1e-6, atol=1e-6)
    np.testing.assert_allclose(O.rope(k, np.arange(N), 10000.0), rk[0].permute(1, 0, 2).numpy(), rtol=1e-6, atol=1e-6)


# ---- block-wise schedule ([README] "Quick Start", generate_mode "default")

def test_block_commit_worked_example():
    """N = 10, generation from 4, blocks of 3: [4, 7) [7, 10).  Masked 5, 8, 9:
    the open block is [4, 7), so only position 5 can be committed; once it is
    unmasked the open block moves to [7, 10)."""
    N = 10
    masked = np.zeros(N, bool)
    masked[[5, 8, 9]] = True
    c = np.full(N, 0.5, np.float32)
    c[[8, 9]] = 0.99                      # higher confidence outside the open block
    amax = np.arange(N) + 100
    ids = np.zeros(N, np.int64)
    assert O.active_block(masked, 4, 3) == (4, 7)
    pos, new_ids, new_masked = O.commit(c, amax, masked, ids, O.RULE_THRESHOLD, 0.9, gen_start=4, block_len=3)
    assert list(pos) == [5] and new_ids[5] == 105 and not new_masked[5] and new_masked[8] and new_masked[9]
    assert O.active_block(new_masked, 4, 3) == (7, 10)
    pos2, _, m2 = O.commit(c, amax, new_masked, new_ids, O.RULE_THRESHOLD, 0.9, gen_start=4, block_len=3)
    assert sorted(pos2) == [8, 9] and not m2.any()
    assert O.active_block(m2, 4, 3) is None
    assert len(O.commit(c, amax, m2, ids, O.RULE_FRECHET, 0.1, gen_start=4, block_len=3)[0]) == 0


def test_block_commit_reduces_to_plain_commit_and_stays_in_block():
    """A block covering the whole generation region is the plain commit; any
    block size commits only inside the leftmost block that holds a masked
    position (brute force over the blocks)."""
    rng = np.random.default_rng(5)
    for trial in range(200):
        N = int(rng.integers(1, 60))
        g0 = int(rng.integers(0, N))
        masked = np.zeros(N, bool)
        masked[g0:] = rng.random(N - g0) < 0.6
        c = rng.choice([0.2, 0.5, 0.95, 0.99], N).astype(np.float32)
        amax = rng.integers(0, 50, N)
        ids = rng.integers(0, 50, N)
        rule, param = [(O.RULE_FRECHET, 0.1), (O.RULE_THRESHOLD, 0.9), (O.RULE_FACTOR, 0.9)][trial % 3]
        full = O.commit(c, amax, masked, ids, rule, param)
        whole = O.commit(c, amax, masked, ids, rule, param, gen_start=g0, block_len=N)
        np.testing.assert_array_equal(full[0], whole[0])
        blen = int(rng.integers(1, 9))
        pos, _, _ = O.commit(c, amax, masked, ids, rule, param, gen_start=g0, block_len=blen)
        blocks = [(b, min(N, b + blen)) for b in range(g0, N, blen)]
        open_ = next(((a, b) for a, b in blocks if masked[a:b].any()), None)
        if open_ is None:
            assert len(pos) == 0
        else:
            assert len(pos) >= 1 and all(open_[0] <= p < open_[1] and masked[p] for p in pos)
            inside = np.flatnonzero(masked[open_[0]:open_[1]]) + open_[0]
            ref = O.commit(np.where(np.isin(np.arange(N), inside), c, 0).astype(np.float32), amax,
                           np.isin(np.arange(N), inside), ids, rule, param)
            np.testing.assert_array_equal(pos, ref[0])


# ------------------------------------------------------------------ periodic full refresh

def test_refresh_range_schedule():
    """Closed forms of the refresh schedule: the prompt block every
    prompt_interval steps, the generated block every gen_interval steps,
    both together on common multiples, nothing when an interval is 0."""
    N, g0 = 100, 70
    got = [O.refresh_range(t, g0, N, 2, 3) for t in range(1, 7)]
    assert got == [None, (0, 70), (70, 100), (0, 70), None, (0, 100)]
    assert all(O.refresh_range(t, g0, N, 0, 0) is None for t in range(1, 20))
    assert O.refresh_range(5000, g0, N, 5000, 5000) == (0, N)        # the README's setting: every 5000 steps


def test_forced_range_selection_bruteforce():
    """A forced range joins the window: the top-B is taken outside both, so
    |U| = min(N, |W u F| + B), and U holds all of F."""
    rng = np.random.default_rng(11)
    for _ in range(200):
        N = int(rng.integers(1, 40))
        d = rng.integers(0, 4, N).astype(np.float32) / 4
        keys = list(rng.integers(0, N, int(rng.integers(0, 3))))
        bw, B = int(rng.integers(0, 6)), int(rng.integers(0, N + 2))
        lo = int(rng.integers(0, N + 1))
        hi = int(rng.integers(lo, N + 1))
        U = O.select_rows(d, keys, bw, B, 0, force=(lo, hi))
        W = O.window_mask(keys, bw, N, 0)
        W[lo:hi] = True
        assert set(np.flatnonzero(W)) <= set(U)
        assert len(U) == min(N, int(W.sum()) + B)
        # brute force: the rest are the top-B of (d desc, index asc) outside W u F
        rest = sorted(np.flatnonzero(~W), key=lambda i: (-float(d[i]), i))[:max(0, min(B, N - int(W.sum())))]
        assert set(U) == set(np.flatnonzero(W)) | set(rest)


def test_full_refresh_equals_dense_forward_and_keeps_dynamics():
    """A refresh of both blocks recomputes every row of every layer, so the step
    equals a dense forward on the new ids whatever the budget; d and s are
    still those of the step (the next budgets follow it)."""
    cfg, w = _tiny_model(seed=4, L=3, gains=True)
    N = 12
    ids0, ids1, keys = _ids_and_keys(cfg.vocab, N, 5)
    st0 = O.full_forward(w, cfg, ids0)
    force = O.refresh_range(6, 7, N, 2, 3)
    assert force == (0, N)
    st1, tr = O.dcu_step(w, cfg, st0, ids1, keys, B_layer=1, B_window=0, force=force)
    dense = O.full_forward(w, cfg, ids1)
    for l in range(cfg.n_layers + 1):
        np.testing.assert_allclose(st1.H[l], dense.H[l], rtol=0, atol=1e-6)
    for l in range(cfg.n_layers):
        np.testing.assert_allclose(st1.K[l], dense.K[l], rtol=0, atol=1e-6)
        assert list(tr.sel[l][0]) == list(range(N))
    # the dynamics are the step's: layer-0 d at the key rows only, and s their mean
    assert np.count_nonzero(tr.d[0][0]) == len(keys[0])
    np.testing.assert_allclose(tr.s[0, 0], np.mean(tr.d[0][0].astype(np.float64)), rtol=1e-6)
    # a prompt-only refresh leaves the generated rows to the budget
    st2, tr2 = O.dcu_step(w, cfg, st0, ids1, keys, B_layer=0, B_window=0, force=(0, 7))
    for l in range(cfg.n_layers):
        assert list(tr2.sel[l][0]) == list(range(7))


# ------------------------------------------------------------------ select_from = "v"

def test_value_dynamics_reduces_to_input_dynamics_for_identity_values():
    """With W_v = I (Hkv * hd = D), unit gains and float32 storage, the Value of a
    row is its RMS-normalised input, a positive multiple of it, so the Value
    cosine distance equals the input cosine distance at every stale row."""
    cfg, w = _tiny_model(seed=5, L=2, D=16, H=4, Hkv=2, hd=8)
    for lw in w.layers:
        lw["wv"] = np.eye(16)
    N = 10
    ids0, ids1, keys = _ids_and_keys(cfg.vocab, N, 4, seed=5, n_unmask=3)
    st0 = O.full_forward(w, cfg, ids0)
    st1, tr_v = O.dcu_step(w, cfg, st0, ids1, keys, B_layer=2, B_window=0, select_from="v")
    _, tr_x = O.dcu_step(w, cfg, st0, ids1, keys, B_layer=2, B_window=0)
    np.testing.assert_allclose(tr_v.d[0], tr_x.d[0], rtol=0, atol=2e-6)
    for l in range(cfg.n_layers):
        assert tr_v.sel[l][0].tolist() == tr_x.sel[l][0].tolist()


def test_value_dynamics_invariants():
    """d = 0 wherever the row is not stale; scaling W_v by a > 0 changes nothing;
    a rewritten row that its own layer skipped stays stale into the next step,
    where the Value proxy still sees it (d > 0) while the input proxy gives 0."""
    cfg, w = _tiny_model(seed=6, L=3, D=32)
    N = 16
    ids0, ids1, keys = _ids_and_keys(cfg.vocab, N, 6, seed=6, n_unmask=4)
    st0 = O.full_forward(w, cfg, ids0)
    st1, tr = O.dcu_step(w, cfg, st0, ids1, keys, B_layer=2, B_window=0, select_from="v")
    # layer 0: stale = the rows whose id (hence embedding) changed
    assert set(np.flatnonzero(tr.d[0][0])) <= set(keys[0])
    w2 = O.Weights(w.embed, w.lm_head, w.final_norm, [dict(lw, wv=lw["wv"] * 4.0) for lw in w.layers])
    st0b = O.full_forward(w2, cfg, ids0)
    _, tr2 = O.dcu_step(w2, cfg, st0b, ids1, keys, B_layer=2, B_window=0, select_from="v")
    np.testing.assert_allclose(tr2.d[0], tr.d[0], rtol=1e-6, atol=1e-7)
    # stale bookkeeping: rows recomputed by layer l are clean; rows rewritten into H_l (layer 0:
    # a changed id) but not recomputed by layer l stay stale
    skipped = []
    for l in range(cfg.n_layers):
        U = set(tr.sel[l][0])
        rewritten = set(keys[0]) if l == 0 else set(tr.sel[l - 1][0])
        for i in range(N):
            if i in U:
                assert not st1.stale[l][0][i]
            elif i not in rewritten:
                assert not st1.stale[l][0][i]
        skipped += [(l, i) for i in rewritten - U if st1.stale[l][0][i]]
    assert skipped, "no skipped stale row in this seeded case"
    # next step with nothing new and no budget: the Value proxy still sees them, the input proxy gives 0
    _, tr3 = O.dcu_step(w, cfg, st1, st1.ids, [[]], B_layer=0, B_window=0, select_from="v")
    _, tr4 = O.dcu_step(w, cfg, st1, st1.ids, [[]], B_layer=0, B_window=0)
    for l, i in skipped:
        assert tr3.d[l][0][i] > 0 and tr4.d[l][0][i] == 0


def test_value_mode_full_budget_equals_dense_forward():
    cfg, w = _tiny_model(seed=7, L=2, gains=True)
    N = 10
    ids0, ids1, keys = _ids_and_keys(cfg.vocab, N, 4, seed=7)
    st0 = O.full_forward(w, cfg, ids0)
    st1, _ = O.dcu_step(w, cfg, st0, ids1, keys, B_layer=N, B_window=0, select_from="v")
    dense = O.full_forward(w, cfg, ids1)
    for l in range(cfg.n_layers + 1):
        np.testing.assert_allclose(st1.H[l], dense.H[l], rtol=0, atol=1e-6)
    assert not any(x.any() for x in st1.stale)


# ------------------------------------------------------------------ APD (adaptive parallel decoding)

def test_apd_concentration_closed_forms():
    """c = 1 - (second-highest probability): p = (0.6, 0.3, 0.1) -> 0.7; a tie at
    the top makes the second-highest the top probability: (0.4, 0.4, 0.2) -> 0.6."""
    c, H = O.apd_signals(np.log([[0.6, 0.3, 0.1], [0.4, 0.4, 0.2]]), None)
    np.testing.assert_allclose(c, [0.7, 0.6], rtol=0, atol=1e-12)
    assert np.all(H == 0.0)                                # first visit: no instability yet


def test_apd_instability_closed_forms_and_scipy():
    """H = 1 - cos(p, p_prev): 0 for identical distributions; p = (1/2, 1/2, 0)
    against (1/2, 0, 1/2) gives cos = 1/2; random logits agree with
    scipy.spatial.distance.cosine of the softmax vectors."""
    z = np.log(np.array([[0.5, 0.5, 1e-300], [0.2, 0.3, 0.5]]))
    zp = [np.log(np.array([0.5, 1e-300, 0.5])), np.log(np.array([0.2, 0.3, 0.5]))]
    _, H = O.apd_signals(z, zp)
    np.testing.assert_allclose(H, [0.5, 0.0], rtol=0, atol=1e-12)
    rng = np.random.default_rng(3)
    z = rng.normal(0, 3, (5, 40))
    zp = [rng.normal(0, 3, 40) for _ in range(5)]
    _, H = O.apd_signals(z, zp)
    ref = [scipy.spatial.distance.cosine(scipy.special.softmax(z[i]), scipy.special.softmax(zp[i])) for i in range(5)]
    np.testing.assert_allclose(H, ref, rtol=1e-9, atol=1e-12)
    _, H = O.apd_signals(z, [None, zp[1], None, zp[3], None])
    assert H[0] == 0.0 and H[2] == 0.0 and H[1] > 0


def test_apd_update_and_commit_reduce_to_threshold_rule():
    """alpha = beta = 0 keeps tau; with H = 0 the threshold drops by alpha c; a
    constant tau makes the APD commit the threshold rule (a different code path:
    the sorted prefix with c >= tau); random per-position tau commits exactly
    {i : c_i >= tau_i} (brute force), else the most confident position."""
    tau = np.full(6, 0.9, dtype=np.float32)
    c = np.linspace(0.1, 0.6, 6)
    np.testing.assert_array_equal(O.apd_update(tau, c, np.ones(6), 0.0, 0.0), tau)
    np.testing.assert_allclose(O.apd_update(tau, c, np.zeros(6), 0.5, 1.0), 0.9 - 0.5 * c, rtol=0, atol=1e-7)
    rng = np.random.default_rng(5)
    for _ in range(300):
        N = int(rng.integers(1, 30))
        conf = (rng.integers(0, 8, N) / 8).astype(np.float32)
        masked = rng.random(N) < 0.7
        ids = np.zeros(N, np.int64)
        amax = rng.integers(0, 50, N)
        t0 = float(rng.integers(0, 9) / 8)
        a = O.apd_commit(conf, amax, masked, ids, np.full(N, t0, np.float32))
        b = O.commit(conf, amax, masked, ids, O.RULE_THRESHOLD, t0)
        assert list(a[0]) == list(b[0])
        tau = (rng.integers(0, 9, N) / 8).astype(np.float32)
        got = set(O.apd_commit(conf, amax, masked, ids, tau)[0].tolist())
        want = {i for i in range(N) if masked[i] and conf[i] >= tau[i]}
        if not want and masked.any():
            mp = np.flatnonzero(masked)
            want = {int(sorted(mp, key=lambda i: (-float(conf[i]), i))[0])}
        assert got == want
