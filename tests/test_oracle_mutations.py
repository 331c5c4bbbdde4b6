"""Plant plausible mistakes in the C++ oracle (on the CPU) and check that a
pin catches each one.  Shows the pins are not vacuous.

Each mutant is the oracle's own source, ``oracle/step.cc``, with one small
edit (every edited snippet must occur exactly once, so a mutant never drifts
silently when the source changes), compiled with the oracle's own flags into
a temporary library; the pins then run against that library.
"""
import concurrent.futures
import os
import tempfile

import pytest

import tests.test_oracle_pins as pins
from oracle import build, step

# name -> ([(original snippet, mutated snippet), ...], [pins that must fail])
MUTANTS = {
    "dropped_softmax_scale": (
        [("s[j] = dot / scale;", "s[j] = dot;")],
        ["test_masked_attention_matches_torch_sdpa"]),
    "inclusive_offset_block_causal": (
        [("else if (qi_noised) v = bj < bi;", "else if (qi_noised) v = bj <= bi;")],
        ["test_training_mask_truth_table"]),
    "block_causal_strict": (
        [("return block_id(k_pos, prompt_len, D) <= block_id(q_pos, prompt_len, D);",
          "return block_id(k_pos, prompt_len, D) < block_id(q_pos, prompt_len, D);")],
        ["test_inference_visibility_is_block_causal",
         "test_training_forward_equals_cached_inference_path"]),
    "last_index_argmax": (
        [("if (l[v] > top1) {", "if (l[v] >= top1) {")],
        ["test_confidence_special_cases"]),
    "confidence_without_max_shift": (
        [("sum += std::exp(l[v] - top1);", "sum += std::exp(l[v]);")],
        ["test_confidence_is_exp_of_max_minus_logsumexp"]),
    "bf16_ties_away_from_zero": (
        [("std::nearbyint(m * 256.0)", "std::round(m * 256.0)")],
        ["test_bf16_rounding_matches_torch_cast"]),
    "strict_threshold": (
        [("if (c[p] >= tau) S.push_back(p);", "if (c[p] > tau) S.push_back(p);")],
        ["test_commit_threshold_is_inclusive"]),
    "fallback_to_highest_position": (
        [("if (c[p] > c[best]) best = p;", "if (c[p] >= c[best]) best = p;")],
        ["test_commit_fallback_tie_goes_to_lowest_position"]),
    "every_unit_position_a_candidate": (
        [("if (bt[p] == mask_id) M.push_back(p);", "M.push_back(p);")],
        ["test_commit_only_masked_positions_are_candidates"]),
    "interleaved_gqa": (
        [("h = static_cast<int>(bh % a.Hq);\n    const int kvh = h / group;",
          "h = static_cast<int>(bh % a.Hq);\n    const int kvh = h % a.Hkv;")],
        ["test_gqa_equals_mha_with_repeated_kv_heads"]),
    "shift_in_wrong_direction": (
        [("else if (i == 0) from = h_prev", "else if (i == q_len - 1) from = h_prev"),
         ("(static_cast<size_t>(b) * q_len + i - 1) * H;",
          "(static_cast<size_t>(b) * q_len + i + 1) * H;")],
        ["test_token_shift_rows"]),
    "prefixcache_causal_over_fresh_rows": (
        [("      const size_t q0 = ((static_cast<size_t>(b) * n + r) * Hq + h) * d;",
          "      for (int64_t j = Lp; j < n_keys; ++j) vis[j] = (j - Lp) <= r;\n"
          "      const size_t q0 = ((static_cast<size_t>(b) * n + r) * Hq + h) * d;")],
        ["test_prefixcache_attention_matches_torch_sdpa_with_gqa"]),
    "prefixcache_over_whole_capacity": (
        [("const int64_t Lp = len_pre[b];\n    const int64_t n_keys = Lp + n;",
          "const int64_t Lp = cap_pre;\n    const int64_t n_keys = Lp + n;")],
        ["test_prefixcache_attention_matches_torch_sdpa_with_gqa"]),
    "dualcache_without_suffix": (
        [("const int64_t Ls = dual ? len_suf[b] : 0;", "const int64_t Ls = 0;")],
        ["test_prefixcache_block_rows_equal_dualcache_with_the_same_suffix"]),
    "factor_rule_n_not_n_plus_1": (
        [("static_cast<double>(n + 1) * (1.0 - c[order[n - 1]]) < f",
          "static_cast<double>(n) * (1.0 - c[order[n - 1]]) < f")],
        ["test_factor_rule_eq13"]),
    "budget_rule_without_max_term": (
        [("return sum + mx < 1.0;", "return sum < 1.0;")],
        ["test_budget_rule_eq9_selection", "test_heterogeneous_budget_certifies_agreement"]),
}


def _mutant_source(edits):
    with open(build.SRC) as f:
        src = f.read()
    for old, new in edits:
        assert src.count(old) == 1, f"snippet not found exactly once: {old!r}"
        src = src.replace(old, new)
    return src


@pytest.fixture(scope="module")
def mutant_libs():
    """Every mutant compiled once (in parallel) into a temporary directory."""
    tmp = tempfile.mkdtemp(prefix="oracle_mutants_")

    def make(name):
        src = os.path.join(tmp, name + ".cc")
        with open(src, "w") as f:
            f.write(_mutant_source(MUTANTS[name][0]))
        out = os.path.join(tmp, name + ".so")
        build.compile_source(src, out)
        return name, out

    with concurrent.futures.ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
        paths = dict(ex.map(make, MUTANTS))
    return {name: step.load(path) for name, path in paths.items()}


def _call_pin(name, golden_dir):
    fn = getattr(pins, name)
    if "golden_dir" in fn.__code__.co_varnames[:fn.__code__.co_argcount]:
        return fn(golden_dir)
    if fn.__code__.co_argcount:
        return fn(False)                       # the parametrised block-cache pin
    return fn()


def test_every_pin_passes_on_the_unmutated_oracle(golden_dir):
    for _, names in MUTANTS.values():
        for name in names:
            _call_pin(name, golden_dir)


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_mutant_is_caught(mutant, mutant_libs, golden_dir):
    _, names = MUTANTS[mutant]
    with step.using(mutant_libs[mutant]):
        for name in names:
            with pytest.raises(AssertionError):
                _call_pin(name, golden_dir)
