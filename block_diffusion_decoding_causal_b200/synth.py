"""Seeded synthetic inputs for one denoising step of the active block.

This module only draws random tensors with the shapes and distributions of the
workloads the Fast-dLLM pages evaluate (Qwen2.5-1.5B/7B and LLaDA-8B head and
vocabulary shapes, block size 32, sub-block 8).  It holds none of the method's
arithmetic: no attention, no softmax, no commit rule.  Both the CUDA path
(tests, bench) and the CPU oracle read the tensors it makes.

Every tensor is drawn from its own stream: a ``torch.Generator`` seeded from a
SHA-256 of ``(seed, tensor name, chunk)``, so a tensor's values do not depend
on which other tensors were drawn or in which order.  Large matrices are drawn
in fixed 4096-row chunks so the values do not depend on memory limits either.

Distributions (from the workload descriptions): Q, K, V and the LM-head input
rows ~ N(0, 1); W_lm ~ N(0, 1/H) times a logit scale; committed block
positions hold tokens uniform in [0, V) minus the mask id; still-masked
positions hold the mask id.  Floating tensors are drawn in fp32 and rounded to
the storage dtype by torch (round to nearest even for bf16).
"""
from __future__ import annotations

import dataclasses
import hashlib
from typing import Dict, Optional

import torch

_CHUNK_ROWS = 4096

# Mask-token ids.  LLaDA-8B uses 126336; the Qwen2.5-based v2 models append a
# dedicated mask token after the chat special tokens (id 151665).  The tiny
# case uses the last vocabulary entry.
QWEN_MASK_ID = 151665
LLADA_MASK_ID = 126336

CONFIGS: Dict[str, dict] = {
    # batch 1, prefix 64, block 8 with 4 of 8 masked, 4/4 heads, d 32, fp32
    "tiny": dict(batch=1, n_q_heads=4, n_kv_heads=4, head_dim=32, block_size=8,
                 q_len=8, q_off=0, prefix=(64, 64), cap_prefix=64, suffix=0,
                 cap_suffix=0, hidden=128, vocab=512, mask_id=511, shift=0,
                 tau=0.9, w_scale=6.0, dtype="f32", masked=(4, 4)),
    # Qwen2.5-1.5B shapes: batch 1, 12/2 heads, prefix 512, sub-block 8 of 32
    "qwen1.5b": dict(batch=1, n_q_heads=12, n_kv_heads=2, head_dim=128,
                     block_size=32, q_len=8, q_off=None, prefix=(512, 512),
                     cap_prefix=512, suffix=0, cap_suffix=0, hidden=1536,
                     vocab=151936, mask_id=QWEN_MASK_ID, shift=1, tau=0.9,
                     w_scale=8.0, dtype="bf16", masked=(8, 8)),
    # Qwen2.5-7B shapes: batch 4, 28/4 heads, prefix U[1024, 2048]
    "qwen7b": dict(batch=4, n_q_heads=28, n_kv_heads=4, head_dim=128,
                   block_size=32, q_len=8, q_off=None, prefix=(1024, 2048),
                   cap_prefix=2048, suffix=0, cap_suffix=0, hidden=3584,
                   vocab=152064, mask_id=QWEN_MASK_ID, shift=1, tau=0.9,
                   w_scale=8.0, dtype="bf16", masked=(4, 8)),
    # LLaDA-8B-like DualCache: prompt 512 + 8 finished blocks, suffix 736
    "llada": dict(batch=1, n_q_heads=32, n_kv_heads=32, head_dim=128,
                  block_size=32, q_len=32, q_off=0, prefix=(768, 768),
                  cap_prefix=768, suffix=736, cap_suffix=736, hidden=4096,
                  vocab=126464, mask_id=LLADA_MASK_ID, shift=0, tau=0.9,
                  w_scale=8.0, dtype="bf16", masked=(32, 32)),
}


def sweep_config(batch: int, prefix: int, w_scale: float = 8.0) -> dict:
    """Long-context sweep point at Qwen2.5-7B shapes (batch x prefix x scale)."""
    c = dict(CONFIGS["qwen7b"])
    c.update(batch=batch, prefix=(prefix, prefix), cap_prefix=prefix,
             w_scale=float(w_scale))
    return c


@dataclasses.dataclass
class Case:
    """One synthetic step input.  Tensors live on the CPU; bf16 or fp32."""
    name: str
    seed: int
    cfg: dict                      # geometry + tau + mask id + dtype
    q: torch.Tensor                # [B, q_len, Hq, d]
    k_pre: torch.Tensor            # [B, Hkv, cap_prefix, d]
    v_pre: torch.Tensor
    len_pre: torch.Tensor          # [B] int32
    prompt_len: torch.Tensor       # [B] int32, prompt part of the prefix
    k_blk: torch.Tensor            # [B, Hkv, D, d]
    v_blk: torch.Tensor
    k_suf: Optional[torch.Tensor]  # [B, Hkv, cap_suffix, d] (DualCache only)
    v_suf: Optional[torch.Tensor]
    len_suf: Optional[torch.Tensor]
    hidden: Optional[torch.Tensor]  # [B, q_len, H] LM-head input rows, or None
    h_prev: Optional[torch.Tensor]  # [B, H] hidden state before the unit
    w_lm: Optional[torch.Tensor]   # [V, H] (None when not drawn)
    block_tokens: torch.Tensor     # [B, D] int32


def _stream(seed: int, *key) -> torch.Generator:
    h = hashlib.sha256(repr((int(seed),) + tuple(key)).encode()).digest()
    g = torch.Generator(device="cpu")
    g.manual_seed(int.from_bytes(h[:8], "little") & ((1 << 63) - 1))
    return g


def _normal(seed: int, name: str, shape, dtype: torch.dtype, scale: float = 1.0,
            extra=()) -> torch.Tensor:
    """N(0, scale^2) in fp32, rounded to ``dtype``; drawn in 4096-row chunks."""
    shape = tuple(int(s) for s in shape)
    rows = shape[0]
    inner = shape[1:]
    out = torch.empty(shape, dtype=dtype)
    for c0 in range(0, rows, _CHUNK_ROWS):
        c1 = min(rows, c0 + _CHUNK_ROWS)
        g = _stream(seed, name, c0 // _CHUNK_ROWS, *extra)
        x = torch.randn((c1 - c0,) + inner, generator=g, dtype=torch.float32)
        if scale != 1.0:
            x.mul_(scale)
        out[c0:c1] = x.to(dtype)
    return out


def _ints(seed: int, name: str, n: int, lo: int, hi: int) -> torch.Tensor:
    """n integers uniform in [lo, hi] (inclusive)."""
    g = _stream(seed, name)
    return torch.randint(lo, hi + 1, (n,), generator=g, dtype=torch.int64)


def torch_dtype(dtype: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[dtype]


def make_case(name: str, seed: int, cfg: Optional[dict] = None,
              attn_as_hidden: bool = False, draw_w: bool = True, **overrides) -> Case:
    """Draw one step input.

    ``name`` picks a row of ``CONFIGS`` (or pass ``cfg`` explicitly); keyword
    overrides replace config entries (e.g. ``tau=0.7``, ``batch=2``).  With
    ``attn_as_hidden`` the LM-head rows are the attention output itself (no
    separate hidden input), the literal single-layer chaining.  With
    ``draw_w=False`` the LM-head weight is not drawn (``w_lm`` is None), for
    callers that already hold the case's weight.
    """
    c = dict(CONFIGS[name] if cfg is None else cfg)
    c.update(overrides)
    B, Hq, Hkv, d = c["batch"], c["n_q_heads"], c["n_kv_heads"], c["head_dim"]
    D, q_len, H, V = c["block_size"], c["q_len"], c["hidden"], c["vocab"]
    dt = torch_dtype(c["dtype"])
    if c.get("q_off") is None:
        n_units = D // q_len
        c["q_off"] = int(_ints(seed, "q_off", 1, 0, n_units - 1)[0]) * q_len
    q_off = c["q_off"]
    assert 0 <= q_off and q_off + q_len <= D

    lo, hi = c["prefix"]
    len_pre = _ints(seed, "len_pre", B, lo, hi).to(torch.int32)
    if c.get("len_pre") is not None:          # explicit per-sequence lengths
        len_pre = torch.tensor(c["len_pre"], dtype=torch.int32)
    # Prompt part of the prefix: the rest is whole finished blocks.
    n_done = (len_pre // (4 * D)).to(torch.int32)
    prompt_len = (len_pre - n_done * D).to(torch.int32)
    cap_p = max(int(c["cap_prefix"]), int(len_pre.max()))
    c["cap_prefix"] = cap_p

    q = _normal(seed, "q", (B, q_len, Hq, d), dt)
    k_pre = _normal(seed, "k_pre", (B * Hkv * cap_p, d), dt).view(B, Hkv, cap_p, d)
    v_pre = _normal(seed, "v_pre", (B * Hkv * cap_p, d), dt).view(B, Hkv, cap_p, d)
    k_blk = _normal(seed, "k_blk", (B, Hkv, D, d), dt)
    v_blk = _normal(seed, "v_blk", (B, Hkv, D, d), dt)
    k_suf = v_suf = len_suf = None
    if c["cap_suffix"] > 0:
        cs = int(c["cap_suffix"])
        k_suf = _normal(seed, "k_suf", (B * Hkv * cs, d), dt).view(B, Hkv, cs, d)
        v_suf = _normal(seed, "v_suf", (B * Hkv * cs, d), dt).view(B, Hkv, cs, d)
        len_suf = torch.full((B,), int(c["suffix"]), dtype=torch.int32)
    hidden = None if attn_as_hidden else _normal(seed, "hidden", (B, q_len, H), dt)
    h_prev = _normal(seed, "h_prev", (B, H), dt) if c["shift"] else None
    w_lm = (_normal(seed, "w_lm", (V, H), dt, scale=c["w_scale"] / H ** 0.5)
            if draw_w else None)

    # Block tokens: finished positions hold random non-mask tokens; inside the
    # unit a seeded subset is masked; later sub-blocks are still all masked.
    mask_id = int(c["mask_id"])
    assert 0 <= mask_id < V, "mask id must be a vocabulary entry"
    toks = _ints(seed, "tokens", B * D, 0, V - 2).view(B, D)
    toks = torch.where(toks >= mask_id, toks + 1, toks).to(torch.int32)
    toks[:, q_off + q_len:] = mask_id
    mlo, mhi = c["masked"]
    n_masked = _ints(seed, "n_masked", B, mlo, mhi)
    for b in range(B):
        g = _stream(seed, "masked_pos", b)
        pos = torch.randperm(q_len, generator=g)[: int(n_masked[b])]
        toks[b, q_off + pos] = mask_id

    return Case(name=name, seed=seed, cfg=c, q=q, k_pre=k_pre, v_pre=v_pre,
                len_pre=len_pre, prompt_len=prompt_len, k_blk=k_blk,
                v_blk=v_blk, k_suf=k_suf, v_suf=v_suf, len_suf=len_suf,
                hidden=hidden, h_prev=h_prev, w_lm=w_lm, block_tokens=toks)


def redraw_row(case: Case, tensor: str, index: tuple, attempt: int) -> None:
    """Replace one row of ``case.<tensor>`` with a fresh N(0,1) draw.

    ``index`` addresses the row: ``("hidden", (b, i))``, ``("h_prev", (b,))``
    or ``("q", (b, r))`` (all heads of query row r).  Each (index, attempt)
    gets its own stream, so a redraw is reproducible.
    """
    t = getattr(case, tensor)
    row = t[index]
    g = _stream(case.seed, "redraw", tensor, tuple(int(i) for i in index), attempt)
    x = torch.randn(row.shape, generator=g, dtype=torch.float32)
    t[index] = x.to(t.dtype)
