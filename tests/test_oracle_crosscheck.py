"""The C++ oracle against the independent numpy restatement of the same
definitions (``oracle/step_np.py``), on seeded cases that cover both storage
dtypes, GQA, the token shift, DualCache, attention chained as the LM-head
input, and the incremental recompute the margin repair uses.  The two share
nothing but the definitions on the pages, so agreement to ~1e-12 checks the
C++ program's indexing and composition end to end."""
import numpy as np
import pytest
import torch

from block_diffusion_decoding_causal_b200 import synth
from oracle import cases, step, step_np

SMALL = dict(batch=3, n_q_heads=6, n_kv_heads=2, head_dim=64, block_size=16, q_len=8,
             q_off=None, prefix=(0, 300), cap_prefix=300, suffix=0, cap_suffix=0,
             hidden=384, vocab=5000, mask_id=4999, shift=1, tau=0.8, w_scale=8.0,
             dtype="bf16", masked=(2, 8))
DUAL = dict(SMALL, suffix=50, cap_suffix=60, shift=0)


def _np(t):
    if t is None:
        return None
    return t.to(torch.float64).numpy()


def _numpy_step(case):
    return step_np.denoise_step(
        case.cfg, _np(case.q), _np(case.k_pre), _np(case.v_pre), case.len_pre.numpy(),
        case.prompt_len.numpy(), _np(case.k_blk), _np(case.v_blk), _np(case.hidden),
        _np(case.h_prev), _np(case.w_lm), case.block_tokens.numpy(), _np(case.k_suf),
        _np(case.v_suf), None if case.len_suf is None else case.len_suf.numpy())


def _agree(a, b):
    act = b["active"]
    for k in ["attn", "attn_rounded", "rows", "conf", "logit_gap"]:
        x, y = np.asarray(a[k]), np.asarray(b[k])
        if k == "logit_gap":
            x, y = x[act], y[act]
        err = np.abs(x - y).max() / max(1e-300, np.abs(y).max())
        assert err < 1e-12, (k, err)
    for k in ["tok", "block_tokens", "committed", "n_committed", "n_masked_left", "active"]:
        assert np.array_equal(np.asarray(a[k]), np.asarray(b[k])), k


@pytest.mark.parametrize("name,cfg,as_hidden", [
    ("tiny", None, False), ("tiny", None, True), ("small", SMALL, False),
    ("small", SMALL, True), ("dual", DUAL, False), ("dual", DUAL, True)])
def test_cpp_oracle_equals_numpy_restatement(name, cfg, as_hidden):
    for seed in (3, 4):
        case = synth.make_case(name, seed, cfg=cfg, attn_as_hidden=as_hidden)
        _agree(cases.run_oracle(case), _numpy_step(case))


def test_margin_repaired_case_equals_a_full_recompute():
    """The repair recomputes only redrawn rows; the final result must equal a
    fresh full oracle call on the repaired inputs."""
    for as_hidden in (False, True):
        case, res, redrawn = cases.parity_case("small", 7, cfg=SMALL,
                                               attn_as_hidden=as_hidden)
        full = cases.run_oracle(case)
        assert redrawn > 0
        for k in ["attn", "conf", "logit_gap", "tok", "block_tokens", "n_committed"]:
            assert np.array_equal(res[k], full[k]), k


def test_selection_rules_equal_numpy_restatement():
    from oracle import theory
    rng = np.random.default_rng(9)
    for _ in range(300):
        n = int(rng.integers(0, 12))
        M = sorted(rng.choice(32, n, replace=False).tolist())
        conf = rng.uniform(0.0, 1.0, 32) ** rng.uniform(0.1, 2.0)
        conf[rng.integers(0, 32)] = conf[rng.integers(0, 32)]       # ties now and then
        c = lambda p: float(conf[p])
        f = float(rng.uniform(0.05, 3.0))
        tau = float(rng.uniform(0.3, 1.0))
        assert step.threshold_select(M, c, tau) == step_np.threshold_select(M, c, tau)
        assert theory.factor_select(M, c, f) == (step_np.factor_select(M, c, f) if M else [])
        assert theory.budget_select(M, c) == (step_np.budget_select(M, c) if M else [])
