"""CPU oracle for one denoising step of the active block: the Python face of
the plain fp64 C++ program in ``step.cc`` (built into ``liboracle.so``).

TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's
CPU-baseline and reference legs may import this package.  The CUDA library
never calls it and shares no code with it.

This module only marshals arguments (numpy arrays or CPU torch tensors in,
numpy arrays out) and sequences no arithmetic of its own: every step of the
method, its citations and the readings taken where the pages are silent are in
``step.cc``.  ``step_np`` holds an earlier, independent numpy restatement of
the same definitions, kept as a second check.

Stored inputs are passed as they are stored (bf16 bit patterns, fp32 or
fp64) and upcast exactly inside the oracle.
"""
from __future__ import annotations

import contextlib
import ctypes
import os

import numpy as np

from . import build as _build

F32, BF16, F64 = 0, 1, 2
RULE_THRESHOLD, RULE_FACTOR, RULE_BUDGET = 0, 1, 2

_P = ctypes.c_void_p
_I = ctypes.c_int
_L = ctypes.c_int64
_D = ctypes.c_double

_lib = None


class StepCfg(ctypes.Structure):
    """Mirror of ``orc_step_cfg`` in step.cc."""
    _fields_ = [("B", _I), ("q_len", _I), ("Hq", _I), ("Hkv", _I), ("d", _I), ("D", _I),
                ("q_off", _I), ("cap_pre", _L), ("cap_suf", _L), ("H", _L), ("V", _L),
                ("mask_id", _L), ("shift", _I), ("stored", _I), ("w_stored", _I),
                ("threads", _I), ("tau", ctypes.c_float)]


def _declare(L):
    L.orc_version.restype = _I
    L.orc_round.argtypes = [_L, _P, _I, _P]
    L.orc_training_mask.argtypes = [_L, _L, _P]
    L.orc_block_ids.argtypes = [_L, _P, _L, _L, _P]
    L.orc_inference_visibility.argtypes = [_L, _P, _L, _P, _L, _L, _I, _P]
    L.orc_masked_attention.argtypes = [_L, _L, _I, _P, _P, _P, _P, _P]
    L.orc_attention_step.argtypes = ([_I] * 6 + [_L, _L, _I, _I] + [_P] * 10 + [_P, _I])
    L.orc_prefixcache_attention.argtypes = [_I] * 5 + [_L, _I] + [_P] * 7 + [_I]
    L.orc_shifted_rows.argtypes = [_I, _I, _L, _I, _P, _P, _P]
    L.orc_lmhead_confidence.argtypes = [_L, _L, _L, _P, _P, _I, _P, _P, _P, _I]
    L.orc_select.argtypes = [_I, _D, _I, _P, _P, _P]
    L.orc_select.restype = _I
    L.orc_budget_ok.argtypes = [_I, _P]
    L.orc_budget_ok.restype = _I
    L.orc_commit.argtypes = [_I, _I, _I, _I, _L, _I, _D] + [_P] * 7
    L.orc_denoise_step.argtypes = [ctypes.POINTER(StepCfg)] + [_P] * 28
    L.orc_denoise_step.restype = _I
    return L


def load(path: str):
    """Load an oracle library from ``path`` (the tests load mutated builds)."""
    return _declare(ctypes.CDLL(path))


def lib():
    global _lib
    if _lib is None:
        _lib = load(_build.build())
    return _lib


@contextlib.contextmanager
def using(library):
    """Route every call of this module to ``library`` inside the block."""
    global _lib
    saved = lib()
    _lib = library
    try:
        yield
    finally:
        _lib = saved


# ------------------------------------------------------------ marshalling

def _ptr(a):
    return None if a is None else a.ctypes.data_as(_P)


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.int64))


def _stored(x):
    """(contiguous numpy array, stored code) for an input kept as stored:
    torch bf16 -> its bit patterns; fp32 stays fp32; anything else fp64."""
    if x is None:
        return None, None
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), BF16
            x = x.numpy()
    except ImportError:
        pass
    x = np.asarray(x)
    if x.dtype == np.float32:
        return np.ascontiguousarray(x), F32
    return _f64(x), F64


def _same_stored(*xs):
    arrs, codes = zip(*(_stored(x) for x in xs))
    kinds = {c for c in codes if c is not None}
    if len(kinds) > 1:                       # mixed storage: compare in fp64
        arrs = tuple(None if x is None else _f64(_as_f64(x)) for x in xs)
        return arrs, F64
    return arrs, (kinds.pop() if kinds else F64)


def _as_f64(x):
    a, code = _stored(x)
    if code == BF16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


# ----------------------------------------------------------------- rounding

def round_to(x, dtype: str) -> np.ndarray:
    """Round fp64 values to the storage dtype ("f32" or "bf16")."""
    code = {"f32": F32, "bf16": BF16}[dtype]
    x = _f64(x)
    out = np.empty_like(x)
    lib().orc_round(x.size, _ptr(x), code, _ptr(out))
    return out


def round_bf16(x) -> np.ndarray:
    """Round fp64 values to bfloat16 (8 significant bits, ties to even)."""
    return round_to(x, "bf16")


# ------------------------------------------------------------------ masks

def training_mask(L: int, D: int) -> np.ndarray:
    """M_full over [x_t ; x_0] (v2 digest, "Attention Mask Design"), [2L, 2L]."""
    out = np.empty((2 * L, 2 * L), dtype=np.uint8)
    lib().orc_training_mask(L, D, _ptr(out))
    return out.astype(bool)


def block_ids(pos, prompt_len: int, D: int) -> np.ndarray:
    """Block index of absolute positions (prompt = block 0)."""
    pos = _i64(pos)
    out = np.empty_like(pos)
    lib().orc_block_ids(pos.size, _ptr(pos), int(prompt_len), int(D), _ptr(out))
    return out


def inference_visibility(q_pos, k_pos, prompt_len: int, D: int, full: bool) -> np.ndarray:
    """Block-causal (or, with ``full``, full) visibility of keys by queries."""
    q_pos, k_pos = _i64(q_pos).ravel(), _i64(k_pos).ravel()
    out = np.empty((q_pos.size, k_pos.size), dtype=np.uint8)
    lib().orc_inference_visibility(q_pos.size, _ptr(q_pos), k_pos.size, _ptr(k_pos),
                                   int(prompt_len), int(D), int(bool(full)), _ptr(out))
    return out.astype(bool)


# -------------------------------------------------------------- attention

def masked_attention(q, k, v, visible) -> np.ndarray:
    """softmax(q k^T / sqrt(d)) v over an explicit visibility mask."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    vis = np.ascontiguousarray(np.broadcast_to(np.asarray(visible, dtype=bool),
                                               (q.shape[0], k.shape[0]))).astype(np.uint8)
    out = np.empty((q.shape[0], q.shape[1]), dtype=np.float64)
    lib().orc_masked_attention(q.shape[0], k.shape[0], q.shape[1], _ptr(q), _ptr(k),
                               _ptr(v), _ptr(vis), _ptr(out))
    return out


def attention_step(q, k_pre, v_pre, len_pre, prompt_len, k_blk, v_blk, q_off,
                   k_suf=None, v_suf=None, len_suf=None, threads: int = 0) -> np.ndarray:
    """Attention of the active unit's queries, fp64, [B, q_len, Hq, d]."""
    (q, k_pre, v_pre, k_blk, v_blk, k_suf, v_suf), code = _same_stored(
        q, k_pre, v_pre, k_blk, v_blk, k_suf, v_suf)
    B, q_len, Hq, d = q.shape
    Hkv, cap_pre, D = k_pre.shape[1], k_pre.shape[2], k_blk.shape[2]
    cap_suf = 0 if k_suf is None else k_suf.shape[2]
    lp, pl = _i64(len_pre), _i64(prompt_len)
    ls = None if len_suf is None else _i64(len_suf)
    out = np.empty((B, q_len, Hq, d), dtype=np.float64)
    lib().orc_attention_step(B, q_len, Hq, Hkv, d, D, cap_pre, cap_suf, int(q_off), code,
                             _ptr(q), _ptr(k_pre), _ptr(v_pre), _ptr(lp), _ptr(pl),
                             _ptr(k_blk), _ptr(v_blk), _ptr(k_suf), _ptr(v_suf), _ptr(ls),
                             _ptr(out), threads)
    return out


def prefixcache_attention(q, k_pre, v_pre, len_pre, k_fresh, v_fresh,
                          threads: int = 0) -> np.ndarray:
    """PrefixCache attention (technical review, section 3), fp64, [B, n, Hq, d]."""
    (q, k_pre, v_pre, k_fresh, v_fresh), code = _same_stored(q, k_pre, v_pre, k_fresh,
                                                              v_fresh)
    B, n, Hq, d = q.shape
    Hkv, cap_pre = k_pre.shape[1], k_pre.shape[2]
    lp = _i64(len_pre)
    out = np.empty((B, n, Hq, d), dtype=np.float64)
    lib().orc_prefixcache_attention(B, n, Hq, Hkv, d, cap_pre, code, _ptr(q), _ptr(k_pre),
                                    _ptr(v_pre), _ptr(lp), _ptr(k_fresh), _ptr(v_fresh),
                                    _ptr(out), threads)
    return out


# ------------------------------------------------------- LM head + commit

def shifted_rows(src, h_prev, shift: int) -> np.ndarray:
    """LM-head input rows with the token shift (v2 digest, Step 5)."""
    src = _f64(src)
    B, q_len, H = src.shape
    hp = _f64(h_prev) if shift else None
    out = np.empty_like(src)
    lib().orc_shifted_rows(B, q_len, H, int(shift), _ptr(src), _ptr(hp), _ptr(out))
    return out


def lmhead_confidence(rows, w, threads: int = 0):
    """(argmax token, confidence, top-1 minus top-2 logit gap) of each row
    over the full vocabulary; ``w`` [V, H] as stored."""
    rows = _f64(rows)
    R, H = rows.shape
    w_arr, w_code = _stored(w)
    V = w_arr.shape[0]
    tok = np.empty(R, dtype=np.int64)
    conf = np.empty(R, dtype=np.float64)
    gap = np.empty(R, dtype=np.float64)
    lib().orc_lmhead_confidence(R, V, H, _ptr(rows), _ptr(w_arr), w_code, _ptr(tok),
                                _ptr(conf), _ptr(gap), threads)
    return tok, conf, gap


def _select(rule: int, param: float, masked_positions, conf_of):
    M = [int(p) for p in masked_positions]
    if not M:
        return []
    conf = np.zeros(max(M) + 1, dtype=np.float64)
    for p in M:
        conf[p] = float(conf_of(p))
    m = np.asarray(M, dtype=np.int32)
    out = np.empty(len(M), dtype=np.int32)
    n = lib().orc_select(rule, float(param), len(M), _ptr(m), _ptr(conf), _ptr(out))
    return out[:n].tolist()


def threshold_select(masked_positions, conf_of, tau: float):
    """Technical review Algorithm 2 over a list of masked positions."""
    return _select(RULE_THRESHOLD, tau, masked_positions, conf_of)


def factor_select(masked_positions, conf_of, f: float):
    """Technical review eq. (13) with Algorithm 3."""
    return _select(RULE_FACTOR, f, masked_positions, conf_of)


def budget_select(masked_positions, conf_of):
    """Selection by the heterogeneous error budget of eq. (9)."""
    return _select(RULE_BUDGET, 0.0, masked_positions, conf_of)


def budget_ok(eps) -> bool:
    """Eq. (9): sum_j eps_j + max_j eps_j < 1."""
    e = _f64(eps).ravel()
    return bool(lib().orc_budget_ok(e.size, _ptr(e)))


def select_commit(block_tokens, conf, tok, q_off: int, q_len: int, mask_id: int,
                  rule: int = RULE_THRESHOLD, param: float = 0.0):
    """Commit over the active unit of every block with a selection rule
    (RULE_THRESHOLD with tau, RULE_FACTOR with f, RULE_BUDGET).  Returns the new
    block tokens, the committed bitmap, the commit counts and the masked counts
    left in the unit."""
    bt = _i64(block_tokens)
    B, D = bt.shape
    c, t = _f64(conf), _i64(tok)
    new = np.empty_like(bt)
    committed = np.empty((B, D), dtype=np.uint8)
    n_comm = np.empty(B, dtype=np.int64)
    n_left = np.empty(B, dtype=np.int64)
    lib().orc_commit(B, D, int(q_off), int(q_len), int(mask_id), int(rule), float(param),
                     _ptr(bt), _ptr(c), _ptr(t), _ptr(new), _ptr(committed), _ptr(n_comm),
                     _ptr(n_left))
    return new, committed, n_comm, n_left


def threshold_commit(block_tokens, conf, tok, q_off: int, q_len: int, mask_id: int,
                     tau: float):
    """Technical review Algorithm 2 over the active unit of every block."""
    return select_commit(block_tokens, conf, tok, q_off, q_len, mask_id,
                         RULE_THRESHOLD, tau)


def lmhead_stage(rows, w, active):
    """LM-head stage outputs as the library reports them: rows whose target
    position is not masked get conf = -1 and tok = -1."""
    rows = _f64(rows)
    B, q_len, H = rows.shape
    tok, conf, gap = lmhead_confidence(rows.reshape(B * q_len, H), w)
    active = np.asarray(active, dtype=bool)
    return (np.where(active, conf.reshape(B, q_len), -1.0),
            np.where(active, tok.reshape(B, q_len), -1), gap.reshape(B, q_len))


def denoise_step(c: dict, q, k_pre, v_pre, len_pre, prompt_len, k_blk, v_blk,
                 hidden, h_prev, w_lm, block_tokens, k_suf=None, v_suf=None,
                 len_suf=None, threads: int = 0, previous: dict = None,
                 redo_q=None, redo_lm=None) -> dict:
    """One denoising step of the active unit (``orc_denoise_step``).

    Tensors may be numpy arrays or CPU torch tensors, as stored.  With
    ``previous`` (an earlier result on the same case) and the [B, q_len] flags
    ``redo_q`` / ``redo_lm``, only the flagged attention query rows and LM-head
    rows are recomputed; the result equals a full call (every row is
    independent of the others).
    """
    (q, k_pre, v_pre, k_blk, v_blk, k_suf, v_suf, hidden, h_prev), code = _same_stored(
        q, k_pre, v_pre, k_blk, v_blk, k_suf, v_suf, hidden, h_prev)
    w_arr, w_code = _stored(w_lm)
    B, q_len, Hq, d = q.shape
    Hkv, cap_pre, D = k_pre.shape[1], k_pre.shape[2], k_blk.shape[2]
    cap_suf = 0 if k_suf is None else k_suf.shape[2]
    V, H = w_arr.shape
    cfg = StepCfg(B=B, q_len=q_len, Hq=Hq, Hkv=Hkv, d=d, D=D, q_off=int(c["q_off"]),
                  cap_pre=cap_pre, cap_suf=cap_suf, H=H, V=V, mask_id=int(c["mask_id"]),
                  shift=int(c["shift"]), stored=code, w_stored=w_code, threads=threads,
                  tau=float(c["tau"]))
    lp, pl, bt = _i64(len_pre), _i64(prompt_len), _i64(block_tokens)
    ls = None if len_suf is None else _i64(len_suf)
    if previous is not None:
        attn = np.array(previous["attn"], dtype=np.float64, order="C")
        conf = np.array(previous["conf"], dtype=np.float64, order="C")
        tok = np.array(previous["tok"], dtype=np.int64, order="C")
        gap = np.array(previous["logit_gap"], dtype=np.float64, order="C")
        rq = np.ascontiguousarray(np.asarray(redo_q, dtype=np.uint8).reshape(B, q_len))
        rl = np.ascontiguousarray(np.asarray(redo_lm, dtype=np.uint8).reshape(B, q_len))
    else:
        attn = np.empty((B, q_len, Hq, d), dtype=np.float64)
        conf = np.empty((B, q_len), dtype=np.float64)
        tok = np.empty((B, q_len), dtype=np.int64)
        gap = np.empty((B, q_len), dtype=np.float64)
        rq = rl = None
    attn_r = np.empty_like(attn)
    rows = np.empty((B, q_len, H), dtype=np.float64)
    active = np.empty((B, q_len), dtype=np.uint8)
    new = np.empty_like(bt)
    committed = np.empty((B, D), dtype=np.uint8)
    n_comm = np.empty(B, dtype=np.int64)
    n_left = np.empty(B, dtype=np.int64)
    cand_gap = np.empty(B, dtype=np.float64)
    rc = lib().orc_denoise_step(
        ctypes.byref(cfg), _ptr(q), _ptr(k_pre), _ptr(v_pre), _ptr(lp), _ptr(pl),
        _ptr(k_blk), _ptr(v_blk), _ptr(k_suf), _ptr(v_suf), _ptr(ls), _ptr(hidden),
        _ptr(h_prev), _ptr(w_arr), _ptr(bt), _ptr(rq), _ptr(rl), _ptr(attn), _ptr(attn_r),
        _ptr(rows), _ptr(active), _ptr(conf), _ptr(tok), _ptr(gap), _ptr(new),
        _ptr(committed), _ptr(n_comm), _ptr(n_left), _ptr(cand_gap))
    if rc != 0:
        raise ValueError("oracle rejected the step's shapes")
    return dict(attn=attn, attn_rounded=attn_r, rows=rows, active=active.astype(bool),
                conf=conf, tok=tok, logit_gap=gap, block_tokens=new, committed=committed,
                n_committed=n_comm, n_masked_left=n_left, tau=float(np.float32(c["tau"])),
                cand_gap=cand_gap)


def library_path() -> str:
    return os.path.abspath(lib()._name)
