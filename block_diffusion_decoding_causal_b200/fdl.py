"""ctypes binding of libfdl.so: the entry points of include/fdl.h, same names.

Argument marshalling only: tensors are passed as raw device pointers, the
configuration as the C struct, the stream as the CUDA stream handle.  Every
step of the computation runs in the library's CUDA kernels; there is no
Python or CPU fallback, and loading fails loudly if the library is missing.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfdl.so")

F32, BF16 = 0, 1
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_DEVICE_STATUS = (
    0, -1, -2, -3, -4, -5)
DEV_BAD_PREFIX_LEN, DEV_BAD_SUFFIX_LEN, DEV_TIMEOUT = 1, 2, 4
SELECT_THRESHOLD, SELECT_FACTOR, SELECT_BUDGET = 0, 1, 2
W_ROW_MAJOR, W_PACKED = 0, 1

# Every symbol include/fdl.h declares.
SYMBOLS = ["fdl_version", "fdl_last_error", "fdl_workspace_size",
           "fdl_reset_workspace", "fdl_block_attn", "fdl_dualcache_attn",
           "fdl_lmhead_confidence", "fdl_threshold_commit", "fdl_denoise_step",
           "fdl_get_status", "fdl_lmhead_confidence_noalloc", "fdl_select_commit",
           "fdl_unit_status", "fdl_append_block", "fdl_prefixcache_attn",
           "fdl_check_wait_timeout", "fdl_lmhead_pack_weight",
           "fdl_lmhead_noalloc_status", "fdl_lmhead_noalloc_reset",
           "fdl_lmhead_noalloc_check_wait_timeout"]
NOALLOC_MAX_ROWS = 128


class StepCfg(ctypes.Structure):
    """Mirror of ``fdl_step_cfg``."""
    _fields_ = [("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("q_off", ctypes.c_int32),
                ("q_len", ctypes.c_int32), ("cap_prefix", ctypes.c_int32),
                ("cap_suffix", ctypes.c_int32), ("hidden", ctypes.c_int32),
                ("vocab", ctypes.c_int32), ("mask_id", ctypes.c_int32),
                ("shift", ctypes.c_int32), ("tau", ctypes.c_float),
                ("dtype", ctypes.c_int32), ("w_layout", ctypes.c_int32)]


class FdlError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"fdl error {code}: {msg}")
        self.code = code


_lib = None
_P = ctypes.c_void_p


def lib() -> ctypes.CDLL:
    """Load libfdl.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise FdlError(ERR_UNSUPPORTED, f"{LIB_PATH} is missing: run "
                           "python -m block_diffusion_decoding_causal_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        L.fdl_version.restype = ctypes.c_int
        L.fdl_last_error.restype = ctypes.c_char_p
        L.fdl_workspace_size.restype = ctypes.c_size_t
        L.fdl_workspace_size.argtypes = [ctypes.POINTER(StepCfg)]
        L.fdl_reset_workspace.argtypes = [_P, ctypes.c_size_t, _P]
        L.fdl_block_attn.argtypes = [ctypes.POINTER(StepCfg)] + [_P] * 7 + [
            _P, ctypes.c_size_t, _P]
        L.fdl_dualcache_attn.argtypes = [ctypes.POINTER(StepCfg)] + [_P] * 10 + [
            _P, ctypes.c_size_t, _P]
        L.fdl_lmhead_confidence.argtypes = [ctypes.POINTER(StepCfg)] + [_P] * 5 + [
            _P, ctypes.c_size_t, _P]
        L.fdl_threshold_commit.argtypes = [ctypes.POINTER(StepCfg)] + [_P] * 6 + [_P]
        L.fdl_denoise_step.argtypes = [ctypes.POINTER(StepCfg)] + [_P] * 19 + [
            _P, ctypes.c_size_t, _P]
        L.fdl_get_status.argtypes = [_P, _P, ctypes.POINTER(ctypes.c_uint32)]
        L.fdl_lmhead_confidence_noalloc.argtypes = [ctypes.POINTER(StepCfg)] + [_P] * 5 + [_P]
        L.fdl_select_commit.argtypes = [ctypes.POINTER(StepCfg), ctypes.c_int, ctypes.c_float] + [
            _P] * 6 + [_P]
        L.fdl_unit_status.argtypes = [ctypes.POINTER(StepCfg), _P, _P, _P, ctypes.c_ulonglong, _P]
        L.fdl_prefixcache_attn.argtypes = [ctypes.POINTER(StepCfg)] + [_P] * 7 + [
            _P, ctypes.c_size_t, _P]
        L.fdl_check_wait_timeout.argtypes = [_P, ctypes.c_size_t, ctypes.c_longlong, _P]
        L.fdl_lmhead_pack_weight.argtypes = [ctypes.POINTER(StepCfg), _P, _P, _P]
        L.fdl_append_block.argtypes = [ctypes.POINTER(StepCfg)] + [_P] * 5 + [_P, ctypes.c_size_t, _P]
        L.fdl_lmhead_noalloc_status.argtypes = [_P, ctypes.POINTER(ctypes.c_uint32)]
        L.fdl_lmhead_noalloc_reset.argtypes = [_P]
        L.fdl_lmhead_noalloc_check_wait_timeout.argtypes = [ctypes.c_longlong, _P]
        for name in ["fdl_reset_workspace", "fdl_block_attn", "fdl_dualcache_attn",
                     "fdl_lmhead_confidence", "fdl_threshold_commit",
                     "fdl_denoise_step", "fdl_get_status",
                     "fdl_lmhead_confidence_noalloc", "fdl_select_commit",
                     "fdl_unit_status", "fdl_append_block", "fdl_prefixcache_attn",
                     "fdl_check_wait_timeout", "fdl_lmhead_pack_weight",
                     "fdl_lmhead_noalloc_status", "fdl_lmhead_noalloc_reset",
                     "fdl_lmhead_noalloc_check_wait_timeout"]:
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def last_error() -> str:
    return lib().fdl_last_error().decode()


def _check(rc: int) -> None:
    if rc != OK:
        raise FdlError(rc, last_error())


def make_cfg(c: dict) -> StepCfg:
    """Build the C struct from a config dict (keys as in ``synth.CONFIGS``)."""
    return StepCfg(batch=c["batch"], n_q_heads=c["n_q_heads"],
                   n_kv_heads=c["n_kv_heads"], head_dim=c["head_dim"],
                   block_size=c["block_size"], q_off=c["q_off"], q_len=c["q_len"],
                   cap_prefix=c["cap_prefix"], cap_suffix=c.get("cap_suffix", 0),
                   hidden=c["hidden"], vocab=c["vocab"], mask_id=c["mask_id"],
                   shift=c["shift"], tau=c["tau"],
                   dtype=BF16 if c["dtype"] == "bf16" else F32,
                   w_layout=c.get("w_layout", W_ROW_MAJOR))


def ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def stream_ptr(stream: Optional[torch.cuda.Stream] = None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def workspace_size(cfg: StepCfg) -> int:
    n = lib().fdl_workspace_size(ctypes.byref(cfg))
    if n == 0:
        raise FdlError(ERR_INVALID_ARG, last_error())
    return n


def workspace(cfg: StepCfg, device="cuda") -> torch.Tensor:
    """A zero-filled workspace tensor for ``cfg`` (torch blocks are 512-byte
    aligned)."""
    return torch.zeros(workspace_size(cfg), dtype=torch.uint8, device=device)


def block_attn(cfg, q, k_pre, v_pre, len_pre, k_blk, v_blk, out, ws, stream=None):
    _check(lib().fdl_block_attn(ctypes.byref(cfg), ptr(q), ptr(k_pre), ptr(v_pre),
                                ptr(len_pre), ptr(k_blk), ptr(v_blk), ptr(out),
                                ptr(ws), ws.numel(), stream_ptr(stream)))


def dualcache_attn(cfg, q, k_pre, v_pre, len_pre, k_blk, v_blk, k_suf, v_suf,
                   len_suf, out, ws, stream=None):
    _check(lib().fdl_dualcache_attn(ctypes.byref(cfg), ptr(q), ptr(k_pre), ptr(v_pre),
                                    ptr(len_pre), ptr(k_blk), ptr(v_blk), ptr(k_suf),
                                    ptr(v_suf), ptr(len_suf), ptr(out), ptr(ws),
                                    ws.numel(), stream_ptr(stream)))


def prefixcache_attn(cfg, q, k_pre, v_pre, len_pre, k_fresh, v_fresh, out, ws, stream=None):
    _check(lib().fdl_prefixcache_attn(ctypes.byref(cfg), ptr(q), ptr(k_pre), ptr(v_pre),
                                      ptr(len_pre), ptr(k_fresh), ptr(v_fresh), ptr(out),
                                      ptr(ws), ws.numel(), stream_ptr(stream)))


def lmhead_confidence(cfg, rows, w_lm, row_active, conf, tok, ws, stream=None):
    _check(lib().fdl_lmhead_confidence(ctypes.byref(cfg), ptr(rows), ptr(w_lm),
                                       ptr(row_active), ptr(conf), ptr(tok), ptr(ws),
                                       ws.numel(), stream_ptr(stream)))


def lmhead_confidence_noalloc(cfg, rows, w_lm, row_active, conf, tok, stream=None):
    """fdl_lmhead_confidence with the library's built-in scratch instead of a
    caller workspace (at most NOALLOC_MAX_ROWS rows; calls on one device must
    not overlap on the GPU; make the first call on a device before any stream
    capture; device failures are read with ``lmhead_noalloc_status``)."""
    _check(lib().fdl_lmhead_confidence_noalloc(ctypes.byref(cfg), ptr(rows), ptr(w_lm),
                                               ptr(row_active), ptr(conf), ptr(tok),
                                               stream_ptr(stream)))


def threshold_commit(cfg, conf, tok, block_tokens, committed, n_committed,
                     n_masked_left, stream=None):
    _check(lib().fdl_threshold_commit(ctypes.byref(cfg), ptr(conf), ptr(tok),
                                      ptr(block_tokens), ptr(committed),
                                      ptr(n_committed), ptr(n_masked_left),
                                      stream_ptr(stream)))


def select_commit(cfg, policy, param, conf, tok, block_tokens, committed, n_committed,
                  n_masked_left, stream=None):
    _check(lib().fdl_select_commit(ctypes.byref(cfg), int(policy), float(param), ptr(conf),
                                   ptr(tok), ptr(block_tokens), ptr(committed),
                                   ptr(n_committed), ptr(n_masked_left), stream_ptr(stream)))


def unit_status(cfg, n_masked_left, any_masked=None, step_count=None, while_handle=0,
                stream=None):
    _check(lib().fdl_unit_status(ctypes.byref(cfg), ptr(n_masked_left), ptr(any_masked),
                                 ptr(step_count), int(while_handle), stream_ptr(stream)))


def append_block(cfg, k_blk, v_blk, k_pre, v_pre, len_pre, ws, stream=None):
    _check(lib().fdl_append_block(ctypes.byref(cfg), ptr(k_blk), ptr(v_blk), ptr(k_pre),
                                  ptr(v_pre), ptr(len_pre), ptr(ws), ws.numel(),
                                  stream_ptr(stream)))


def denoise_step(cfg, q, k_pre, v_pre, len_pre, k_blk, v_blk, k_suf, v_suf, len_suf,
                 hidden, h_prev, w_lm, block_tokens, attn_out, conf, tok, committed,
                 n_committed, n_masked_left, ws, stream=None):
    _check(lib().fdl_denoise_step(
        ctypes.byref(cfg), ptr(q), ptr(k_pre), ptr(v_pre), ptr(len_pre), ptr(k_blk),
        ptr(v_blk), ptr(k_suf), ptr(v_suf), ptr(len_suf), ptr(hidden), ptr(h_prev),
        ptr(w_lm), ptr(block_tokens), ptr(attn_out), ptr(conf), ptr(tok),
        ptr(committed), ptr(n_committed), ptr(n_masked_left), ptr(ws), ws.numel(),
        stream_ptr(stream)))


def lmhead_pack_weight(cfg, w_lm, w_packed, stream=None):
    _check(lib().fdl_lmhead_pack_weight(ctypes.byref(cfg), ptr(w_lm), ptr(w_packed),
                                        stream_ptr(stream)))


def check_wait_timeout(ws, limit_cycles=1_000_000, stream=None):
    _check(lib().fdl_check_wait_timeout(ptr(ws), ws.numel(), int(limit_cycles),
                                        stream_ptr(stream)))


def get_status(ws, stream=None) -> int:
    """Synchronise, read and clear the device status word (FDL_DEV_* bits)."""
    st = ctypes.c_uint32(0)
    rc = lib().fdl_get_status(ptr(ws), stream_ptr(stream), ctypes.byref(st))
    if rc not in (OK, ERR_DEVICE_STATUS):
        raise FdlError(rc, last_error())
    return int(st.value)


def lmhead_noalloc_status(stream=None) -> int:
    """Synchronise, read and clear the allocation-free LM head's own status
    word (FDL_DEV_* bits)."""
    st = ctypes.c_uint32(0)
    rc = lib().fdl_lmhead_noalloc_status(stream_ptr(stream), ctypes.byref(st))
    if rc not in (OK, ERR_DEVICE_STATUS):
        raise FdlError(rc, last_error())
    return int(st.value)


def lmhead_noalloc_reset(stream=None):
    _check(lib().fdl_lmhead_noalloc_reset(stream_ptr(stream)))


def lmhead_noalloc_check_wait_timeout(limit_cycles=1_000_000, stream=None):
    _check(lib().fdl_lmhead_noalloc_check_wait_timeout(int(limit_cycles), stream_ptr(stream)))
