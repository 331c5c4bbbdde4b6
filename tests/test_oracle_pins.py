"""Pins of the CPU oracle against what the pages and mathematics fix.

No GPU.  Each check compares the oracle with something other than itself: a
truth table written by hand from the pages' mask definitions, values the pages
print, closed forms, a library routine for a special case (torch's SDPA,
scipy's logsumexp, torch's bf16 cast), a full recompute, or brute force.
"""
import json
import os

import numpy as np
import pytest
import scipy.special
import torch

from oracle import step, theory

RNG = np.random.default_rng(1234)


# ----------------------------------------------------------------- rounding

def test_bf16_rounding_matches_torch_cast():
    x = RNG.standard_normal(20000).astype(np.float32)
    # exact ties between two bf16 neighbours, both parities of the kept bit
    bits = RNG.integers(0x3C000000, 0x42000000, 2000, dtype=np.uint32)
    ties = ((bits & 0xFFFF0000) | 0x8000).view(np.float32)
    x = np.concatenate([x, ties, -ties, np.float32([0.0, 1.0, -2.5, 3.0e-3])])
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = step.round_bf16(x.astype(np.float64))
    assert np.array_equal(got, want)


# -------------------------------------------------------------- attention

def _random_visible(n, m):
    vis = RNG.random((n, m)) < 0.6
    vis[np.arange(n), RNG.integers(0, m, n)] = True
    return vis


def test_masked_attention_matches_torch_sdpa():
    for (n, m, d) in [(8, 72, 32), (5, 300, 128), (1, 1, 16)]:
        q, k, v = (RNG.standard_normal(s) for s in [(n, d), (m, d), (m, d)])
        vis = _random_visible(n, m)
        got = step.masked_attention(q, k, v, vis)
        want = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q)[None], torch.from_numpy(k)[None],
            torch.from_numpy(v)[None], attn_mask=torch.from_numpy(vis)[None]
        )[0].numpy()
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-13)


def test_attention_single_visible_key_returns_its_value():
    q, k, v = (RNG.standard_normal(s) for s in [(3, 16), (10, 16), (10, 16)])
    vis = np.zeros((3, 10), bool)
    vis[:, 7] = True
    np.testing.assert_allclose(step.masked_attention(q, k, v, vis),
                               np.repeat(v[7:8], 3, axis=0), rtol=0, atol=1e-15)


def test_attention_zero_query_averages_visible_values():
    k, v = RNG.standard_normal((12, 8)), RNG.standard_normal((12, 8))
    vis = _random_visible(4, 12)
    got = step.masked_attention(np.zeros((4, 8)), k, v, vis)
    want = np.stack([v[vis[i]].mean(axis=0) for i in range(4)])
    np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-14)


def _prefixcache_inputs(B=2, Hq=6, Hkv=2, d=16, cap=40, n=20, D=8):
    q = RNG.standard_normal((B, n, Hq, d))
    k_pre, v_pre = RNG.standard_normal((2, B, Hkv, cap, d))
    k_new, v_new = RNG.standard_normal((2, B, Hkv, n, d))
    lens = np.array([cap - 7, 0][:B])
    return q, k_pre, v_pre, lens, k_new, v_new, D


def test_prefixcache_attention_matches_torch_sdpa_with_gqa():
    """Full attention of every recomputed row over [prefix | fresh rows]
    against SDPA with the KV heads repeated for their query groups."""
    q, k_pre, v_pre, lens, k_new, v_new, _ = _prefixcache_inputs()
    got = step.prefixcache_attention(q, k_pre, v_pre, lens, k_new, v_new)
    group = q.shape[2] // k_pre.shape[1]
    for b in range(q.shape[0]):
        K = np.concatenate([k_pre[b, :, :lens[b]], k_new[b]], axis=1).repeat(group, axis=0)
        V = np.concatenate([v_pre[b, :, :lens[b]], v_new[b]], axis=1).repeat(group, axis=0)
        want = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[b].transpose(1, 0, 2)), torch.from_numpy(K),
            torch.from_numpy(V)).numpy().transpose(1, 0, 2)
        np.testing.assert_allclose(got[b], want, rtol=1e-12, atol=1e-13)


def test_prefixcache_block_rows_equal_dualcache_with_the_same_suffix():
    """When the suffix cache holds exactly the K/V that PrefixCache
    recomputes, the active block's rows see the same keys under both schemes
    (technical review, section 3: the two differ only in what is refreshed)."""
    q, k_pre, v_pre, lens, k_new, v_new, D = _prefixcache_inputs()
    pc = step.prefixcache_attention(q, k_pre, v_pre, lens, k_new, v_new)
    q_off, q_len = 2, 4
    dc = step.attention_step(q[:, q_off:q_off + q_len], k_pre, v_pre, lens, lens,
                             k_new[:, :, :D], v_new[:, :, :D], q_off,
                             k_suf=k_new[:, :, D:], v_suf=v_new[:, :, D:],
                             len_suf=np.full(q.shape[0], q.shape[1] - D))
    np.testing.assert_allclose(pc[:, q_off:q_off + q_len], dc, rtol=1e-13, atol=1e-14)


# ------------------------------------------------------------------ masks

def test_training_mask_truth_table(golden_dir):
    rows = []
    with open(os.path.join(golden_dir, "training_mask_L6_D2.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            rows.append([c == "1" for c in line.strip().replace(" ", "")])
    assert np.array_equal(step.training_mask(6, 2), np.array(rows))


def test_training_mask_quadrant_properties():
    L, D = 64, 8
    M = step.training_mask(L, D)
    blk = np.arange(L) // D
    assert not M[L:, :L].any()                                # clean never sees noised
    assert np.array_equal(M[L:, L:], np.tril(M[L:, L:]) | M[L:, L:])
    for i in range(L):
        assert M[i, :L].sum() == D                            # own block only
        assert M[i, L:].sum() == D * blk[i]                   # strictly earlier clean blocks
        assert M[L + i, L:].sum() == D * (blk[i] + 1)         # same or earlier


def test_inference_visibility_is_block_causal():
    P, D = 13, 4
    pos = np.arange(P + 5 * D)
    active = 3                                                # block index 3
    q_pos = P + (active - 1) * D + np.arange(D)
    vis = step.inference_visibility(q_pos, pos, P, D, full=False)
    kb = step.block_ids(pos, P, D)
    assert np.array_equal(vis, np.broadcast_to(kb <= active, vis.shape))
    assert vis[:, : P + active * D].all() and not vis[:, P + active * D:].any()
    assert step.inference_visibility(q_pos, pos, P, D, full=True).all()


def _single_layer(X, Wq, Wk, Wv, mask):
    return step.masked_attention(X @ Wq, X @ Wk, X @ Wv, mask)


def test_training_forward_equals_cached_inference_path():
    """One fp64 layer over [x_t ; x_0] with M_full gives, for the noised rows
    of block b, exactly what the cached inference path gives with prefix =
    clean blocks < b and block = noised block b (digest, Figure 7b)."""
    L, D, dm, d = 16, 4, 24, 16
    Wq, Wk, Wv = (RNG.standard_normal((dm, d)) for _ in range(3))
    x0 = RNG.standard_normal((L, dm))
    xt = x0.copy()
    noised = RNG.random(L) < 0.5
    xt[noised] = RNG.standard_normal(dm)                      # a shared [MASK] embedding
    X = np.concatenate([xt, x0])
    full = _single_layer(X, Wq, Wk, Wv, step.training_mask(L, D))
    for b in range(L // D):
        Lp = b * D
        q = (xt[Lp:Lp + D] @ Wq)[None, :, None, :]
        kp = (x0[:Lp] @ Wk)[None, None]
        vp = (x0[:Lp] @ Wv)[None, None]
        kb = (xt[Lp:Lp + D] @ Wk)[None, None]
        vb = (xt[Lp:Lp + D] @ Wv)[None, None]
        cached = step.attention_step(q, kp, vp, [Lp], [0], kb, vb, 0)[0, :, 0, :]
        np.testing.assert_allclose(cached, full[Lp:Lp + D], rtol=1e-12, atol=1e-12)


def _two_layer_rows(X, W, mask):
    """Two attention layers with residuals; returns per-layer K, V and output."""
    h, kv = X, []
    for (Wq, Wk, Wv) in W:
        kv.append((h @ Wk, h @ Wv))
        h = h + step.masked_attention(h @ Wq, h @ Wk, h @ Wv, mask)
    return h, kv


@pytest.mark.parametrize("full", [False, True])
def test_block_cache_exact_only_when_block_causal(full):
    """v2 digest, Level 3: the block-level KV cache equals a recompute, because
    later blocks are invisible to earlier ones.  Under full attention (v1
    DualCache on LLaDA-style models) the cached prefix is stale from layer 2 on
    (technical review, section 3), so the two must differ."""
    P, D, dm = 6, 4, 16
    n_blocks = 4
    Ltot = P + n_blocks * D
    W = [tuple(RNG.standard_normal((dm, dm)) / 4 for _ in range(3)) for _ in range(2)]
    X = RNG.standard_normal((Ltot, dm))
    pos = np.arange(Ltot)
    mask = step.inference_visibility(pos, pos, P, D, full=full)
    _, kv_full = _two_layer_rows(X, W, mask)
    Lp = P + (n_blocks - 1) * D                               # active = last block
    pre = np.arange(Lp)
    _, kv_prefix_only = _two_layer_rows(X[:Lp], W,
                                        step.inference_visibility(pre, pre, P, D, full=full))
    diff = max(np.abs(kv_prefix_only[layer][t] - kv_full[layer][t][:Lp]).max()
               for layer in range(2) for t in range(2))
    if full:
        assert diff > 1e-3
    else:
        assert diff < 1e-12


def test_gqa_equals_mha_with_repeated_kv_heads():
    B, q_len, Hq, Hkv, d, D, cap = 2, 3, 6, 2, 8, 4, 9
    q = RNG.standard_normal((B, q_len, Hq, d))
    kp, vp = RNG.standard_normal((2, B, Hkv, cap, d))
    kb, vb = RNG.standard_normal((2, B, Hkv, D, d))
    lp, pl = np.array([9, 5]), np.array([1, 1])
    got = step.attention_step(q, kp, vp, lp, pl, kb, vb, 1)
    rep = lambda t: np.repeat(t, Hq // Hkv, axis=1)
    want = step.attention_step(q, rep(kp), rep(vp), lp, pl, rep(kb), rep(vb), 1)
    np.testing.assert_allclose(got, want, rtol=0, atol=0)
    # and each head against the plain eq. (3) over its own key list
    b, h = 1, 5
    K = np.concatenate([kp[b, h // 3, :5], kb[b, h // 3]])
    Vv = np.concatenate([vp[b, h // 3, :5], vb[b, h // 3]])
    s = q[b, :, h] @ K.T / np.sqrt(d)
    p = np.exp(s - s.max(1, keepdims=True))
    np.testing.assert_allclose(got[b, :, h], (p / p.sum(1, keepdims=True)) @ Vv,
                               rtol=1e-12)


def test_token_shift_rows():
    src = RNG.standard_normal((2, 4, 3))
    hp = RNG.standard_normal((2, 3))
    assert np.array_equal(step.shifted_rows(src, hp, 0), src)
    r = step.shifted_rows(src, hp, 1)
    assert np.array_equal(r[:, 0], hp) and np.array_equal(r[:, 1:], src[:, :-1])


# -------------------------------------------------------- LM head softmax

def test_confidence_is_exp_of_max_minus_logsumexp():
    rows = RNG.standard_normal((5, 32))
    w = RNG.standard_normal((1000, 32)) * 0.7
    tok, conf, gap = step.lmhead_confidence(rows, w)
    logits = rows @ w.T
    np.testing.assert_array_equal(tok, logits.argmax(1))
    want = np.exp(logits.max(1) - scipy.special.logsumexp(logits, axis=1))
    np.testing.assert_allclose(conf, want, rtol=1e-12)
    srt = np.sort(logits, axis=1)
    np.testing.assert_allclose(gap, srt[:, -1] - srt[:, -2], rtol=0, atol=1e-12)


def test_confidence_special_cases():
    V, H = 257, 4
    rows = np.ones((1, H))
    tok, conf, _ = step.lmhead_confidence(rows, np.ones((V, H)))
    assert tok[0] == 0 and conf[0] == pytest.approx(1.0 / V, rel=1e-14)
    w = np.zeros((V, H))
    w[100, 0] = 50.0
    tok, conf, _ = step.lmhead_confidence(rows, w)
    assert tok[0] == 100
    assert conf[0] == pytest.approx(1.0 / (1.0 + (V - 1) * np.exp(-50.0)), rel=1e-14)
    w[37, 0] = 50.0                                            # exact two-way tie
    tok, conf, gap = step.lmhead_confidence(rows, w)
    assert tok[0] == 37 and gap[0] == 0.0
    assert conf[0] == pytest.approx(1.0 / (2.0 + (V - 2) * np.exp(-50.0)), rel=1e-14)


# ----------------------------------------------------------------- commit

def _commit(conf_row, tok_row, tokens, tau, q_off=0, mask=9):
    q_len = len(conf_row)
    return step.threshold_commit(np.array([tokens]), np.array([conf_row]),
                                 np.array([tok_row]), q_off, q_len, mask, tau)


def test_commit_all_above_threshold_commit_together():
    new, comm, n, left = _commit([0.95, 0.91, 0.5, 0.99], [1, 2, 3, 4], [9, 9, 9, 9], 0.9)
    assert new[0].tolist() == [1, 2, 9, 4] and comm[0].tolist() == [1, 1, 0, 1]
    assert n[0] == 3 and left[0] == 1


def test_commit_fallback_picks_single_most_confident():
    new, comm, n, left = _commit([0.3, 0.8, 0.5, 0.7], [1, 2, 3, 4], [9, 9, 9, 9], 0.9)
    assert new[0].tolist() == [9, 2, 9, 9] and n[0] == 1 and left[0] == 3


def test_commit_fallback_tie_goes_to_lowest_position():
    new, _, n, _ = _commit([0.4, 0.6, 0.6, 0.1], [1, 2, 3, 4], [9, 9, 9, 9], 0.9)
    assert new[0].tolist() == [9, 2, 9, 9] and n[0] == 1


def test_commit_threshold_is_inclusive():
    new, _, n, _ = _commit([0.9, 0.95, 0.2], [5, 6, 7], [9, 9, 9], 0.9)
    assert new[0].tolist() == [5, 6, 9] and n[0] == 2


def test_commit_only_masked_positions_are_candidates():
    # position 0 already decoded (token 3): its confidence is ignored even
    # though it is the largest; the fallback picks among masked positions only
    new, comm, n, left = _commit([0.99, 0.2, 0.4], [7, 1, 2], [3, 9, 9], 0.995)
    assert new[0].tolist() == [3, 9, 2] and comm[0].tolist() == [0, 0, 1]
    assert n[0] == 1 and left[0] == 1


def test_commit_no_masked_positions_is_noop():
    new, comm, n, left = _commit([0.1, 0.2], [1, 2], [4, 5], 0.9)
    assert new[0].tolist() == [4, 5] and not comm.any() and n[0] == 0 and left[0] == 0


def test_commit_tau_one_decodes_one_token_per_step():
    """digest, Level 2: with tau = 1.0 parallel decoding is disabled."""
    rng = np.random.default_rng(5)
    tokens = [9] * 8
    for stepno in range(8):
        conf = list(rng.uniform(0.1, 0.999, 8))
        new, _, n, left = _commit(conf, list(range(8)), tokens, 1.0)
        assert n[0] == 1 and left[0] == 8 - stepno - 1
        tokens = new[0].tolist()


def test_commit_respects_unit_offset():
    # unit [4, 8) of a block of 8; positions outside the unit are never touched
    toks = [1, 9, 9, 9, 9, 9, 9, 9]
    new, comm, n, left = step.threshold_commit(np.array([toks]),
                                               np.array([[0.95, 0.1, 0.2, 0.3]]),
                                               np.array([[11, 12, 13, 14]]), 4, 4, 9, 0.9)
    assert new[0].tolist() == [1, 9, 9, 9, 11, 9, 9, 9]
    assert comm[0].tolist() == [0, 0, 0, 0, 1, 0, 0, 0] and n[0] == 1 and left[0] == 3


# ------------------------------------------------- selection mathematics

def _bits(s):
    return tuple(int(c) for c in s)


def test_toy_joint_values_printed_in_section_4(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "toy_joint.json")))
    p = np.zeros((2, 2))
    for k, v in g["joint"].items():
        p[_bits(k)] = v
    for m in theory.marginals(p):
        assert m[0] == pytest.approx(g["marginal_prob_of_zero"], abs=1e-12)
    q = theory.product_of_marginals(p)
    for k, v in g["product_of_marginals"].items():
        assert q[_bits(k)] == pytest.approx(v, abs=1e-12)
    assert theory.tv_distance(p, q) == pytest.approx(g["total_variation"], abs=1e-12)
    assert theory.argmax_product(p) == _bits(g["independent_greedy_choice"])
    assert theory.argmax_joint(p) in [_bits(s) for s in g["joint_maximisers"]]
    assert not theory.agreement_certified(p)


def test_group_bound_printed_in_section_6(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "group_bound.json")))
    assert theory.max_certified_group(g["eps"]) == g["max_certified_n"]
    for n, c in g["boundary_confidence"].items():
        assert int(n) / (int(n) + 1) == pytest.approx(c, abs=1e-12)
        assert theory.max_certified_group(1.0 - c) == int(n)


def _concentrated_joint(n, k, rng):
    """A random joint whose mass concentrates on one random string."""
    p = rng.random((k,) * n) ** 8
    mode = tuple(rng.integers(0, k, n))
    p[mode] += rng.uniform(0.0, 50.0) * p.sum()
    return p / p.sum()


def test_agreement_theorem_by_brute_force():
    """Eq. (8): whenever (n+1) eps <= 1 (strict marginals), the joint argmax
    equals the product argmax.  Brute force over n <= 4, alphabets 2 and 3."""
    rng = np.random.default_rng(7)
    certified = 0
    for _ in range(3000):
        n, k = int(rng.integers(1, 5)), int(rng.integers(2, 4))
        p = _concentrated_joint(n, k, rng)
        if theory.agreement_certified(p):
            certified += 1
            assert theory.argmax_joint(p) == theory.argmax_product(p)
    assert certified > 300


def test_eta_family_breaks_agreement_just_outside_the_bound():
    for n in (2, 3, 5):
        p = theory.eta_family(n, 0.01)
        assert p.sum() == pytest.approx(1.0, abs=1e-15)
        assert theory.argmax_product(p) == (0,) * n           # every coordinate prefers 0
        assert sum(theory.argmax_joint(p)) == 1                # a single-one string wins
        assert not theory.agreement_certified(p)
        eps = 1.0 - min(m.max() for m in theory.marginals(p))
        assert eps == pytest.approx(1.0 / (n + 1) + 0.01 / n, abs=1e-12)


def test_heterogeneous_budget_certifies_agreement():
    """Eq. (9): sum eps_j + max eps_j < 1 suffices; with equal eps_j it is
    the uniform condition (n+1) eps < 1."""
    rng = np.random.default_rng(11)
    hits = 0
    for _ in range(3000):
        n, k = int(rng.integers(1, 5)), int(rng.integers(2, 4))
        p = _concentrated_joint(n, k, rng)
        eps = [1.0 - m.max() for m in theory.marginals(p)]
        if theory.heterogeneous_budget_ok(eps):
            hits += 1
            assert theory.argmax_joint(p) == theory.argmax_product(p)
    assert hits > 300
    for n in range(1, 10):
        e = 1.0 / (n + 1)
        assert not theory.heterogeneous_budget_ok([e * 1.001] * n)
        assert theory.heterogeneous_budget_ok([e * 0.999] * n)


def test_factor_rule_eq13():
    conf = {0: 0.99, 1: 0.95, 2: 0.6, 3: 0.97}
    c = conf.__getitem__
    # sorted: 0 (0.99), 3 (0.97), 1 (0.95), 2 (0.6)
    # n=1: 2*0.01=0.02; n=2: 3*0.03=0.09; n=3: 4*0.05=0.2; n=4: 5*0.4=2
    assert theory.factor_select([0, 1, 2, 3], c, 1.0) == [0, 3, 1]
    assert theory.factor_select([0, 1, 2, 3], c, 0.1) == [0, 3]
    assert theory.factor_select([0, 1, 2, 3], c, 0.01) == [0]   # fallback: first alone
    assert theory.factor_select([0, 1, 2, 3], c, 3.0) == [0, 3, 1, 2]
    # with every confidence just below the boundary n/(n+1), f = 1 admits groups of
    # size m only while (m+1)/(n+1) < 1, i.e. m = n - 1 (or the first alone)
    for n in range(1, 12):
        cc = {i: n / (n + 1) - 1e-9 for i in range(n)}
        got = theory.factor_select(list(range(n)), cc.__getitem__, 1.0)
        assert len(got) == max(n - 1, 1)


def test_threshold_select_is_algorithm_2():
    c = {1: 0.2, 4: 0.95, 6: 0.9}.__getitem__
    assert step.threshold_select([1, 4, 6], c, 0.9) == [4, 6]
    assert step.threshold_select([1, 4, 6], c, 0.96) == [4]
    assert step.threshold_select([], c, 0.5) == []


# ------------------------------------------------------ teaching roofline

def test_teaching_roofline_constants(golden_dir):
    """The FAQ page's H100 roofline model: the weight-read floor and the
    per-position compute time reproduce from 14 GB / 3.35 TB/s and
    2 x 7e9 FLOP / 989 TFLOP/s; our roofline helper uses the same formulas."""
    import bench
    g = json.load(open(os.path.join(golden_dir, "teaching_roofline.json")))
    floor_ms = bench.roofline_seconds(bytes_moved=14e9, flops=0, hbm_bps=3.35e12,
                                      flops_per_s=989e12) * 1e3
    per_pos_ms = bench.roofline_seconds(bytes_moved=0, flops=2 * 7e9, hbm_bps=3.35e12,
                                        flops_per_s=989e12) * 1e3
    assert floor_ms == pytest.approx(g["weight_read_floor_ms"], abs=5e-3)
    # 2 * 7e9 / 989e12 s = 0.0141557 ms; the page prints it cut to 0.01415
    assert per_pos_ms == pytest.approx(g["ms_per_position"], abs=1e-5)
    assert floor_ms / per_pos_ms == pytest.approx(g["crossover_positions"], abs=1.0)


def test_budget_rule_eq9_selection():
    # eps sorted: 0.01, 0.02, 0.05, 0.3 -> n=1: .01+.01; n=2: .03+.02; n=3: .08+.05;
    # n=4: .38+.3 = .68 < 1 -> all four admissible
    c = {0: 0.95, 1: 0.99, 2: 0.7, 3: 0.98}.__getitem__
    assert theory.budget_select([0, 1, 2, 3], c) == [1, 3, 0, 2]
    c2 = {0: 0.6, 1: 0.99, 2: 0.55}.__getitem__
    # n=2: eps .01+.4 = .41 + max .4 = .81 < 1; n=3: .86 + .45 = 1.31
    assert theory.budget_select([0, 1, 2], c2) == [1, 0]
    c3 = {0: 0.4, 1: 0.3}.__getitem__
    assert theory.budget_select([0, 1], c3) == [0]       # 0.6 + 0.6 >= 1: first alone
    # the certificate it uses implies agreement (eq. 8 generalised), by brute force
    assert theory.heterogeneous_budget_ok([0.01, 0.02, 0.05, 0.3])


def test_select_commit_matches_threshold_commit_for_algorithm_2():
    rng = np.random.default_rng(3)
    for _ in range(50):
        conf = rng.uniform(0, 1, (3, 8))
        tok = rng.integers(0, 100, (3, 8))
        bt = np.where(rng.random((3, 16)) < 0.5, 99, rng.integers(0, 99, (3, 16)))
        a = step.threshold_commit(bt, conf, tok, 4, 8, 99, 0.7)
        b = step.select_commit(bt, conf, tok, 4, 8, 99, step.RULE_THRESHOLD, 0.7)
        for x, y in zip(a, b):
            assert np.array_equal(x, y)
