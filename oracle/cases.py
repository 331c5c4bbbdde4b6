"""Parity cases: synthetic step inputs whose decisions have margins.

TEST INFRASTRUCTURE, like the rest of ``oracle``.

The committed tokens must match bit for bit between the GPU (fp32 arithmetic
on bf16/fp32 inputs) and this fp64 oracle.  That is only well defined when
no decision sits on a rounding boundary, so after drawing a case we run the
oracle and redraw the input row behind every active row whose

* top-1 minus top-2 logit gap is below ``GAP`` (the argmax),
* confidence lies within ``CONF_MARGIN`` of tau (the threshold test),
* predicted token equals the mask id (a commit that leaves a mask),

and, for a unit where the fallback fires, the row behind the best candidate
when the two best confidences differ by less than ``CAND_REL`` of the best
(relative, because fallback confidences can be ~1/V).  We repeat until every
margin holds and report how many rows were redrawn.
"""
from __future__ import annotations

import numpy as np
from block_diffusion_decoding_causal_b200 import synth
from . import step

GAP = 0.05
CONF_MARGIN = 5e-3
CAND_REL = 2e-3


def run_oracle(case: synth.Case, previous: dict = None, redo_q=None, redo_lm=None,
               threads: int = 0) -> dict:
    """The oracle's denoise step on a synthetic case (inputs as stored).

    With ``previous`` and the [B, q_len] flags ``redo_q`` / ``redo_lm`` only
    the flagged query rows and LM-head rows are recomputed (see
    ``step.denoise_step``)."""
    c = case.cfg
    return step.denoise_step(
        c, case.q, case.k_pre, case.v_pre, case.len_pre.numpy(),
        case.prompt_len.numpy(), case.k_blk, case.v_blk, case.hidden, case.h_prev,
        case.w_lm, case.block_tokens.numpy(), case.k_suf, case.v_suf,
        None if case.len_suf is None else case.len_suf.numpy(), threads=threads,
        previous=previous, redo_q=redo_q, redo_lm=redo_lm)


def _violations(case: synth.Case, res: dict):
    """Unit rows (b, i) whose decisions are too close to call."""
    c = case.cfg
    tau = res["tau"]
    bad = set()
    act = res["active"]
    B, q_len = act.shape
    for b in range(B):
        for i in range(q_len):
            if not act[b, i]:
                continue
            if (res["logit_gap"][b, i] < GAP
                    or abs(res["conf"][b, i] - tau) < CONF_MARGIN
                    or res["tok"][b, i] == c["mask_id"]):
                bad.add((b, i))
        if res["cand_gap"][b] < CAND_REL:
            conf_b = np.where(act[b], res["conf"][b], -np.inf)
            bad.add((b, int(np.argmax(conf_b))))
    return sorted(bad)


def _redraw_source(case: synth.Case, b: int, i: int, attempt: int, redo_q, redo_lm):
    """Redraw the input row that feeds LM-head row (b, i) and flag the rows
    whose results that changes."""
    shift = case.cfg["shift"]
    q_len = case.cfg["q_len"]
    if shift and i == 0:
        synth.redraw_row(case, "h_prev", (b,), attempt)
        redo_lm[b, 0] = 1
        return
    src = i - 1 if shift else i
    if case.hidden is not None:
        synth.redraw_row(case, "hidden", (b, src), attempt)
    else:
        synth.redraw_row(case, "q", (b, src), attempt)
        redo_q[b, src] = 1
    if src + shift < q_len:
        redo_lm[b, src + shift] = 1


def parity_case(name: str, seed: int, cfg=None, attn_as_hidden: bool = False,
                max_rounds: int = 40, **overrides):
    """A synthetic case with every decision margin satisfied.

    Returns (case, oracle result, number of redrawn rows).  After the first
    full oracle run, each round recomputes only the rows it redrew.
    """
    case = synth.make_case(name, seed, cfg=cfg, attn_as_hidden=attn_as_hidden,
                           **overrides)
    redrawn = 0
    res = run_oracle(case)
    B, q_len = case.cfg["batch"], case.cfg["q_len"]
    for attempt in range(max_rounds):
        bad = _violations(case, res)
        if not bad:
            return case, res, redrawn
        redo_q = np.zeros((B, q_len), dtype=np.uint8)
        redo_lm = np.zeros((B, q_len), dtype=np.uint8)
        for (b, i) in bad:
            _redraw_source(case, b, i, attempt, redo_q, redo_lm)
            redrawn += 1
        res = run_oracle(case, previous=res, redo_q=redo_q, redo_lm=redo_lm)
    raise RuntimeError(f"margin repair did not converge for {name} seed {seed}")
