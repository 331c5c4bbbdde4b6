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
import torch

from block_diffusion_decoding_causal_b200 import synth
from . import step

GAP = 0.05
CONF_MARGIN = 5e-3
CAND_REL = 2e-3


def _np(t, dtype=np.float64):
    if t is None:
        return None
    if t.dtype in (torch.bfloat16, torch.float16):
        t = t.to(torch.float32)
    return t.numpy().astype(dtype, copy=False)


def run_oracle(case: synth.Case) -> dict:
    """The oracle's denoise step on a synthetic case (inputs upcast exactly)."""
    c = case.cfg
    w = case.w_lm
    w_np = (w.to(torch.float32) if w.dtype != torch.float32 else w).numpy()
    return step.denoise_step(
        c, _np(case.q), _np(case.k_pre), _np(case.v_pre),
        case.len_pre.numpy(), case.prompt_len.numpy(), _np(case.k_blk),
        _np(case.v_blk), _np(case.hidden), _np(case.h_prev), w_np,
        case.block_tokens.numpy(), _np(case.k_suf), _np(case.v_suf),
        None if case.len_suf is None else case.len_suf.numpy())


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


def _redraw_source(case: synth.Case, b: int, i: int, attempt: int) -> None:
    """Redraw the input row that feeds LM-head row (b, i)."""
    shift = case.cfg["shift"]
    if shift and i == 0:
        synth.redraw_row(case, "h_prev", (b,), attempt)
        return
    src = i - 1 if shift else i
    if case.hidden is not None:
        synth.redraw_row(case, "hidden", (b, src), attempt)
    else:
        synth.redraw_row(case, "q", (b, src), attempt)


def parity_case(name: str, seed: int, cfg=None, attn_as_hidden: bool = False,
                max_rounds: int = 40, **overrides):
    """A synthetic case with every decision margin satisfied.

    Returns (case, oracle result, number of redrawn rows).
    """
    case = synth.make_case(name, seed, cfg=cfg, attn_as_hidden=attn_as_hidden,
                           **overrides)
    redrawn = 0
    for attempt in range(max_rounds):
        res = run_oracle(case)
        bad = _violations(case, res)
        if not bad:
            return case, res, redrawn
        for (b, i) in bad:
            _redraw_source(case, b, i, attempt)
            redrawn += 1
    raise RuntimeError(f"margin repair did not converge for {name} seed {seed}")
