"""Independent numpy restatement of the oracle (fp64), kept as a second check.

The oracle proper is the plain C++ program in ``step.cc`` (``step.py`` is its
binding); this module writes the same definitions again in numpy, and a CPU
test compares the two on seeded cases.

TEST INFRASTRUCTURE.  Only the tests, the smoke check and the CPU-baseline leg
of the benchmark may import this package.  The CUDA library never calls it and
shares no code with it.

Every function below writes out the plain definition the pages give; nothing is
blocked, fused or reordered.  Sources (page title, then the passage):

* "Fast-dLLM v2: Efficient Block-Diffusion LLM" (paper digest), section 3.4:
  "Attention Mask Design" with the inference-time mask of Figure 7b;
  "Step 5: Token shift for prediction"; "Inference Pipeline", Levels 1-3.
* "Fast-dLLM: Reusing Bidirectional State and Spending Confidence on Parallel
  Tokens" (technical review), section 2 eq. (3) (attention), section 3
  (PrefixCache / DualCache), section 4 Algorithm 2 (threshold selection).

Readings where the pages are silent (each is listed in the design notes):
* GQA: query head h reads KV head h // (Hq / Hkv).
* argmax over the full vocabulary, lowest index on a tie; confidence is the
  largest softmax probability 1 / sum_v exp(l_v - l_max).
* commit compares conf >= tau, with tau as the float32 the library receives;
  the fallback picks the lowest position among equal confidences.
* token shift: the row that predicts unit position q_off + i is the hidden state
  of position q_off + i - 1; for i = 0 it is the caller's h_prev.
* attention output is rounded once to the storage dtype (bf16: round to
  nearest even) before it is used as an LM-head row.

Parity of that last rounding point and of the GPU's fp32 exponentials is
unpinned by the pages: tolerances and decision margins cover both.
"""
from __future__ import annotations

import numpy as np

# ----------------------------------------------------------------- rounding


def round_bf16(x) -> np.ndarray:
    """Round fp64 values to bfloat16 (8 significant bits, ties to even).

    bfloat16 keeps the fp32 exponent range and 1 + 7 mantissa bits.  Written
    as: x = m * 2**e with 0.5 <= |m| < 1, keep round(m * 2**8) (numpy's rint
    rounds half to even).  Valid for normal numbers, which is all the step
    produces; bf16 subnormals (|x| < 2**-126) are not modelled.
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    return np.ldexp(np.rint(m * 256.0), e - 8)


def round_to(x, dtype: str) -> np.ndarray:
    """Round fp64 values to the storage dtype ("f32" or "bf16")."""
    if dtype == "bf16":
        return round_bf16(x)
    if dtype == "f32":
        return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)
    raise ValueError(dtype)


# ------------------------------------------------------------------ masks


def training_mask(L: int, D: int) -> np.ndarray:
    """M_full over the concatenation [x_t ; x_0] of length 2L (v2 digest,
    "Attention Mask Design"): [[M_BD, M_OBC], [0, M_BC]].

    M_BD: noised i sees noised j iff same block.  M_OBC: noised i sees clean j
    iff j's block is strictly before i's.  M_BC: clean i sees clean j iff j's
    block is the same or earlier.  Clean never sees noised (zero quadrant).
    """
    blk = np.arange(L) // D
    same = blk[:, None] == blk[None, :]
    before = blk[None, :] < blk[:, None]
    same_or_before = blk[None, :] <= blk[:, None]
    top = np.concatenate([same, before], axis=1)
    bottom = np.concatenate([np.zeros((L, L), dtype=bool), same_or_before], axis=1)
    return np.concatenate([top, bottom], axis=0)


def block_ids(pos: np.ndarray, prompt_len: int, D: int) -> np.ndarray:
    """Block index of absolute positions: the prompt is block 0, then the
    generated answer is cut into blocks of D (v2 digest, Level 1)."""
    pos = np.asarray(pos)
    return np.where(pos < prompt_len, 0, 1 + (pos - prompt_len) // D)


def inference_visibility(q_pos, k_pos, prompt_len: int, D: int,
                         full: bool) -> np.ndarray:
    """Which keys each query of the active block may attend to.

    Block-causal (v2, Figure 7b): a query sees every key in its own block
    (bidirectional) and every key in an earlier block (causal across blocks).
    ``full``: v1 DualCache over a full-attention dLLM, where every position of
    the sequence (prefix, block, masked suffix) is visible (technical review,
    section 3).
    """
    q_pos = np.asarray(q_pos)
    k_pos = np.asarray(k_pos)
    if full:
        return np.ones((q_pos.size, k_pos.size), dtype=bool)
    qb = block_ids(q_pos, prompt_len, D)
    kb = block_ids(k_pos, prompt_len, D)
    return kb[None, :] <= qb[:, None]


# -------------------------------------------------------------- attention


def masked_attention(q, k, v, visible) -> np.ndarray:
    """softmax(q k^T / sqrt(d)) v, blocked pairs at -inf before the softmax
    (technical review eq. (3); v2 digest "Attention Mask Design")."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    s = q @ k.T / np.sqrt(q.shape[-1])
    s = np.where(visible, s, -np.inf)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=1, keepdims=True)
    return p @ v


def attention_step(q, k_pre, v_pre, len_pre, prompt_len, k_blk, v_blk, q_off,
                   k_suf=None, v_suf=None, len_suf=None) -> np.ndarray:
    """Attention output of the active unit's queries, fp64, [B, q_len, Hq, d].

    Keys of sequence b = prefix cache rows [0, len_pre[b]) followed by the D
    block rows (and, for DualCache, the suffix cache rows [0, len_suf[b])).
    Absolute positions: prefix 0..Lp-1, block Lp..Lp+D-1, suffix after it.
    Query r of the unit sits at position Lp + q_off + r.  With a suffix the
    mask is full attention, otherwise block-causal.
    """
    B, q_len, Hq, d = q.shape
    Hkv = k_pre.shape[1]
    D = k_blk.shape[2]
    group = Hq // Hkv
    dual = k_suf is not None
    out = np.empty((B, q_len, Hq, d), dtype=np.float64)
    for b in range(B):
        Lp = int(len_pre[b])
        Ls = int(len_suf[b]) if dual else 0
        k_pos = np.arange(Lp + D + Ls)
        q_pos = Lp + q_off + np.arange(q_len)
        vis = inference_visibility(q_pos, k_pos, int(prompt_len[b]), D, full=dual)
        for h in range(Hq):
            kvh = h // group
            parts_k = [k_pre[b, kvh, :Lp], k_blk[b, kvh]]
            parts_v = [v_pre[b, kvh, :Lp], v_blk[b, kvh]]
            if dual:
                parts_k.append(k_suf[b, kvh, :Ls])
                parts_v.append(v_suf[b, kvh, :Ls])
            K = np.concatenate(parts_k, axis=0)
            Vv = np.concatenate(parts_v, axis=0)
            out[b, :, h, :] = masked_attention(q[b, :, h, :], K, Vv, vis)
    return out


def prefixcache_attention(q, k_pre, v_pre, len_pre, k_fresh, v_fresh) -> np.ndarray:
    """PrefixCache attention of v1 (technical review, section 3 and
    Algorithm 1, the PrefixCache branch), fp64, [B, n, Hq, d].

    Only the prompt and the finished answer prefix are cached; the active
    block and the still-masked suffix after it (n positions in all) are
    recomputed every step.  Their queries attend, with full (bidirectional)
    attention, to the cached prefix rows [0, len_pre[b]) followed by the n
    recomputed rows' own fresh K/V.
    """
    B, n, Hq, d = q.shape
    Hkv = k_pre.shape[1]
    group = Hq // Hkv
    out = np.empty((B, n, Hq, d), dtype=np.float64)
    for b in range(B):
        Lp = int(len_pre[b])
        vis = np.ones((n, Lp + n), dtype=bool)
        for h in range(Hq):
            kvh = h // group
            K = np.concatenate([k_pre[b, kvh, :Lp], k_fresh[b, kvh]], axis=0)
            Vv = np.concatenate([v_pre[b, kvh, :Lp], v_fresh[b, kvh]], axis=0)
            out[b, :, h, :] = masked_attention(q[b, :, h, :], K, Vv, vis)
    return out


# ------------------------------------------------------- LM head + commit


def shifted_rows(src, h_prev, shift: int) -> np.ndarray:
    """LM-head input row for each unit position (v2 digest, section 3.4
    Step 5): position q_off + i is predicted from the hidden state at the
    position before it.  ``src`` is [B, q_len, H]; with shift the first row
    comes from ``h_prev`` [B, H]."""
    src = np.asarray(src)
    if not shift:
        return src.copy()
    rows = np.empty_like(src)
    rows[:, 0] = h_prev
    rows[:, 1:] = src[:, :-1]
    return rows


def lmhead_confidence(rows, w, chunk: int = 8192):
    """Greedy prediction and its confidence for each row (v2 digest, Level 2;
    technical review, section 4, Algorithm 2).

    logits l = W h over the full vocabulary; token = argmax l (lowest index
    on a tie, numpy's argmax); confidence = the probability softmax(l) gives
    that token = 1 / sum_v exp(l_v - l_max).  Also returns the top-1 minus
    top-2 logit gap (a decision margin for the tests).
    """
    rows = np.asarray(rows, dtype=np.float64)
    R = rows.shape[0]
    V = w.shape[0]
    logits = np.empty((R, V), dtype=np.float64)
    for c0 in range(0, V, chunk):
        c1 = min(V, c0 + chunk)
        logits[:, c0:c1] = rows @ np.asarray(w[c0:c1], dtype=np.float64).T
    tok = logits.argmax(axis=1)
    lmax = logits[np.arange(R), tok]
    conf = 1.0 / np.exp(logits - lmax[:, None]).sum(axis=1)
    second = np.partition(logits, V - 2, axis=1)[:, V - 2] if V > 1 else lmax
    return tok.astype(np.int64), conf, lmax - second


def threshold_select(masked_positions, conf_of, tau: float):
    """Technical review Algorithm 2: S = {i in M : c_i >= tau}; if S is empty
    (and M is not), S = {the position with maximum c_i}.  Ties in the
    fallback go to the lowest position."""
    M = list(masked_positions)
    S = [p for p in M if conf_of(p) >= tau]
    if not S and M:
        best = M[0]
        for p in M[1:]:
            if conf_of(p) > conf_of(best):
                best = p
        S = [best]
    return S


def threshold_commit(block_tokens, conf, tok, q_off: int, q_len: int,
                     mask_id: int, tau: float):
    """Commit step over the active unit [q_off, q_off + q_len) of each block.

    Candidates are the unit's positions still holding the mask token (v2
    digest Level 1: undecoded positions hold the mask token).  The sub-block is the
    thresholding unit (v2 digest, "Sub-block size as a decoding granularity
    knob").  conf / tok are [B, q_len], indexed by unit position.
    Returns new block tokens, the committed bitmap over the whole block,
    the commit count and the masked count left in the unit.
    """
    bt = np.array(block_tokens, dtype=np.int64)
    B, D = bt.shape
    new = bt.copy()
    committed = np.zeros((B, D), dtype=np.uint8)
    n_comm = np.zeros(B, dtype=np.int64)
    n_left = np.zeros(B, dtype=np.int64)
    for b in range(B):
        M = [p for p in range(q_off, q_off + q_len) if bt[b, p] == mask_id]
        S = threshold_select(M, lambda p: conf[b, p - q_off], tau)
        for p in S:
            new[b, p] = tok[b, p - q_off]
            committed[b, p] = 1
        n_comm[b] = len(S)
        n_left[b] = sum(1 for p in range(q_off, q_off + q_len) if new[b, p] == mask_id)
    return new, committed, n_comm, n_left


def select_commit(block_tokens, conf, tok, q_off: int, q_len: int, mask_id: int,
                  select):
    """Commit step with any selection rule ``select(masked, conf_of)`` over
    the unit's still-masked positions (technical review, Algorithms 2 and 3;
    eq. 9).  Same outputs as ``threshold_commit``."""
    bt = np.array(block_tokens, dtype=np.int64)
    B, D = bt.shape
    new = bt.copy()
    committed = np.zeros((B, D), dtype=np.uint8)
    n_comm = np.zeros(B, dtype=np.int64)
    n_left = np.zeros(B, dtype=np.int64)
    for b in range(B):
        M = [p for p in range(q_off, q_off + q_len) if bt[b, p] == mask_id]
        S = select(M, lambda p: conf[b, p - q_off]) if M else []
        for p in S:
            new[b, p] = tok[b, p - q_off]
            committed[b, p] = 1
        n_comm[b] = len(S)
        n_left[b] = sum(1 for p in range(q_off, q_off + q_len) if new[b, p] == mask_id)
    return new, committed, n_comm, n_left


def lmhead_stage(rows, w, active, tau=None):
    """LM-head stage outputs as the library reports them: rows whose target
    position is not masked get conf = -1 and tok = -1."""
    B, q_len, H = rows.shape
    tok, conf, gap = lmhead_confidence(rows.reshape(B * q_len, H), w)
    tok = tok.reshape(B, q_len)
    conf = conf.reshape(B, q_len)
    gap = gap.reshape(B, q_len)
    active = np.asarray(active, dtype=bool)
    return (np.where(active, conf, -1.0), np.where(active, tok, -1), gap)


def denoise_step(c: dict, q, k_pre, v_pre, len_pre, prompt_len, k_blk, v_blk,
                 hidden, h_prev, w_lm, block_tokens, k_suf=None, v_suf=None,
                 len_suf=None) -> dict:
    """One denoising step of the active unit, written from its definition.

    1. attention of the unit's queries over prefix (+ suffix) cache and block;
    2. that output rounded to the storage dtype;
    3. LM-head rows: ``hidden`` if given, else the attention output (the
       single-layer chaining), then the token shift;
    4. full-vocabulary argmax and confidence;
    5. the threshold commit (tau as float32).
    Also returns the decision margins the parity tests rely on.
    """
    dtype = c["dtype"]
    q_off, q_len, mask_id = int(c["q_off"]), int(c["q_len"]), int(c["mask_id"])
    tau = float(np.float32(c["tau"]))
    attn = attention_step(q, k_pre, v_pre, len_pre, prompt_len, k_blk, v_blk,
                          q_off, k_suf, v_suf, len_suf)
    attn_r = round_to(attn, dtype)
    B = attn.shape[0]
    src = attn_r.reshape(B, q_len, -1) if hidden is None else np.asarray(hidden, np.float64)
    rows = shifted_rows(src, None if h_prev is None else np.asarray(h_prev, np.float64),
                        int(c["shift"]))
    bt = np.asarray(block_tokens)
    active = bt[:, q_off:q_off + q_len] == mask_id
    conf, tok, gap = lmhead_stage(rows, w_lm, active)
    new, committed, n_comm, n_left = threshold_commit(bt, conf, tok, q_off, q_len,
                                                      mask_id, tau)
    # Decision margins: logit gap and |conf - tau| per active row; the
    # relative confidence gap between the two best candidates where the
    # fallback fires.
    cand_gap = np.full(B, np.inf)
    for b in range(B):
        cs = sorted(conf[b][active[b]], reverse=True)
        if len(cs) >= 2 and cs[0] < tau:
            cand_gap[b] = (cs[0] - cs[1]) / cs[0]
    return dict(attn=attn, attn_rounded=attn_r, rows=rows, active=active,
                conf=conf, tok=tok, logit_gap=gap, block_tokens=new,
                committed=committed, n_committed=n_comm, n_masked_left=n_left,
                tau=tau, cand_gap=cand_gap)


# ---------------------------------------------- factor / budget selection
# (technical review section 5.1 eq. (9); section 6 eq. (13), Algorithm 3)

def heterogeneous_budget_ok(eps) -> bool:
    """Eq. (9): sum_j eps_j + max_j eps_j < 1."""
    eps = [float(e) for e in eps]
    return sum(eps) + max(eps) < 1.0


def factor_select(masked_positions, conf_of, f: float):
    """Algorithm 3 with eq. (13): sort the masked positions by decreasing
    confidence (ties: lower position first); keep the largest n with
    (n + 1) (1 - c_(n)) < f; if no n qualifies, the first position alone."""
    order = sorted(masked_positions, key=lambda p: (-conf_of(p), p))
    best = 0
    for n in range(1, len(order) + 1):
        if (n + 1) * (1.0 - conf_of(order[n - 1])) < f:
            best = n
    if best == 0:
        return order[:1]
    return order[:best]


def budget_select(masked_positions, conf_of):
    """Selection by the heterogeneous error budget of eq. (9): sort the masked
    positions by decreasing confidence (ties: lower position first), with
    eps_j = 1 - c_j; keep the largest n whose first n positions satisfy
    sum eps + max eps < 1; if no n qualifies, the first position alone."""
    order = sorted(masked_positions, key=lambda p: (-conf_of(p), p))
    best = 0
    for n in range(1, len(order) + 1):
        if heterogeneous_budget_ok([1.0 - conf_of(q) for q in order[:n]]):
            best = n
    if best == 0:
        return order[:1]
    return order[:best]
