"""Plant plausible mistakes in the oracle (on the CPU) and check that a pin
catches each one.  Shows the pins are not vacuous."""
import numpy as np
import pytest

import tests.test_oracle_pins as pins
from oracle import step


def _expect_pin_failure(fn, *args):
    with pytest.raises(AssertionError):
        fn(*args)


def test_dropped_softmax_scale_is_caught(monkeypatch):
    orig = step.masked_attention

    def no_scale(q, k, v, visible):
        return orig(np.asarray(q) * np.sqrt(np.asarray(q).shape[-1]), k, v, visible)
    monkeypatch.setattr(step, "masked_attention", no_scale)
    _expect_pin_failure(pins.test_masked_attention_matches_torch_sdpa)


def test_inclusive_offset_block_causal_is_caught(monkeypatch, golden_dir):
    def wrong(L, D):
        blk = np.arange(L) // D
        top = np.concatenate([blk[:, None] == blk[None, :], blk[None, :] <= blk[:, None]], 1)
        bot = np.concatenate([np.zeros((L, L), bool), blk[None, :] <= blk[:, None]], 1)
        return np.concatenate([top, bot], 0)
    monkeypatch.setattr(step, "training_mask", wrong)
    _expect_pin_failure(pins.test_training_mask_truth_table, golden_dir)
    _expect_pin_failure(pins.test_training_forward_equals_cached_inference_path)


def test_last_index_argmax_is_caught(monkeypatch):
    orig = step.lmhead_confidence

    def last_on_tie(rows, w, chunk=8192):
        tok, conf, gap = orig(rows, w, chunk)
        logits = np.asarray(rows, np.float64) @ np.asarray(w, np.float64).T
        rev = logits.shape[1] - 1 - logits[:, ::-1].argmax(1)
        return rev, conf, gap
    monkeypatch.setattr(step, "lmhead_confidence", last_on_tie)
    _expect_pin_failure(pins.test_confidence_special_cases)


def test_strict_threshold_is_caught(monkeypatch):
    def strict(masked_positions, conf_of, tau):
        M = list(masked_positions)
        S = [p for p in M if conf_of(p) > tau]
        if not S and M:
            S = [max(M, key=lambda p: (conf_of(p), -p))]
        return S
    monkeypatch.setattr(step, "threshold_select", strict)
    _expect_pin_failure(pins.test_commit_threshold_is_inclusive)


def test_fallback_to_highest_position_is_caught(monkeypatch):
    def highest(masked_positions, conf_of, tau):
        M = list(masked_positions)
        S = [p for p in M if conf_of(p) >= tau]
        if not S and M:
            S = [max(M, key=lambda p: (conf_of(p), p))]
        return S
    monkeypatch.setattr(step, "threshold_select", highest)
    _expect_pin_failure(pins.test_commit_fallback_tie_goes_to_lowest_position)


def test_wrong_gqa_map_is_caught(monkeypatch):
    orig = step.attention_step

    def interleaved(q, k_pre, v_pre, len_pre, prompt_len, k_blk, v_blk, q_off, *a):
        # query head h reads KV head h % Hkv instead of h // group
        Hq, Hkv = q.shape[2], k_pre.shape[1]
        idx = np.arange(Hq) % Hkv
        order = np.argsort(idx, kind="stable")
        out = orig(q[:, :, order], k_pre, v_pre, len_pre, prompt_len, k_blk, v_blk, q_off, *a)
        res = np.empty_like(out)
        res[:, :, order] = out
        return res
    monkeypatch.setattr(step, "attention_step", interleaved)
    _expect_pin_failure(pins.test_gqa_equals_mha_with_repeated_kv_heads)


def test_shift_in_wrong_direction_is_caught(monkeypatch):
    def wrong(src, h_prev, shift):
        src = np.asarray(src)
        if not shift:
            return src.copy()
        rows = np.empty_like(src)
        rows[:, -1] = h_prev
        rows[:, :-1] = src[:, 1:]
        return rows
    monkeypatch.setattr(step, "shifted_rows", wrong)
    _expect_pin_failure(pins.test_token_shift_rows)


def test_prefixcache_with_block_causal_mask_is_caught(monkeypatch):
    """PrefixCache computed as if the recomputed rows were one block under a
    causal-across-blocks mask (suffix rows hidden from earlier rows)."""
    def causal(q, k_pre, v_pre, len_pre, k_fresh, v_fresh):
        B, n, Hq, d = q.shape
        group = Hq // k_pre.shape[1]
        out = np.empty((B, n, Hq, d))
        for b in range(B):
            Lp = int(len_pre[b])
            vis = np.ones((n, Lp + n), bool)
            vis[:, Lp:] = np.tril(np.ones((n, n), bool))
            for h in range(Hq):
                K = np.concatenate([k_pre[b, h // group, :Lp], k_fresh[b, h // group]])
                V = np.concatenate([v_pre[b, h // group, :Lp], v_fresh[b, h // group]])
                out[b, :, h] = step.masked_attention(q[b, :, h], K, V, vis)
        return out
    monkeypatch.setattr(step, "prefixcache_attention", causal)
    _expect_pin_failure(pins.test_prefixcache_attention_matches_torch_sdpa_with_gqa)


def test_factor_rule_with_n_instead_of_n_plus_1_is_caught(monkeypatch):
    """Eq. 13 with the group-size factor off by one: n (1 - c_(n)) < f."""
    from oracle import theory

    def off_by_one(masked_positions, conf_of, f):
        order = sorted(masked_positions, key=lambda p: (-conf_of(p), p))
        best = 0
        for n in range(1, len(order) + 1):
            if n * (1.0 - conf_of(order[n - 1])) < f:
                best = n
        return order[:best] if best else order[:1]
    monkeypatch.setattr(theory, "factor_select", off_by_one)
    _expect_pin_failure(pins.test_factor_rule_eq13)


def test_budget_rule_without_the_max_term_is_caught(monkeypatch):
    """Eq. 9 with the max_j eps_j term dropped (sum only)."""
    from oracle import theory
    monkeypatch.setattr(theory, "heterogeneous_budget_ok",
                        lambda eps: sum(float(e) for e in eps) < 1.0)
    _expect_pin_failure(pins.test_budget_rule_eq9_selection)


def test_dualcache_without_its_suffix_is_caught(monkeypatch):
    orig = step.attention_step

    def no_suffix(q, k_pre, v_pre, len_pre, prompt_len, k_blk, v_blk, q_off,
                  k_suf=None, v_suf=None, len_suf=None):
        return orig(q, k_pre, v_pre, len_pre, prompt_len, k_blk, v_blk, q_off)
    monkeypatch.setattr(step, "attention_step", no_suffix)
    _expect_pin_failure(pins.test_prefixcache_block_rows_equal_dualcache_with_the_same_suffix)


def test_prefixcache_over_the_whole_cache_capacity_is_caught(monkeypatch):
    orig = step.prefixcache_attention

    def whole_cap(q, k_pre, v_pre, len_pre, k_fresh, v_fresh):
        cap = np.asarray(k_pre).shape[2]
        return orig(q, k_pre, v_pre, np.full(len(len_pre), cap), k_fresh, v_fresh)
    monkeypatch.setattr(step, "prefixcache_attention", whole_cap)
    _expect_pin_failure(pins.test_prefixcache_attention_matches_torch_sdpa_with_gqa)
