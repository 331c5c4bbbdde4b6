"""Host-only checks of the C ABI: the library loads without a GPU, exports
every symbol include/fdl.h declares, and rejects bad arguments before any
launch (these calls return before touching CUDA)."""
import ctypes
import os
import re

import pytest

from block_diffusion_decoding_causal_b200 import build, fdl, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return fdl.lib()


def _declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(fdl_[a-z0-9_]+)\s*\(", src))
    return names


def test_library_exports_every_declared_symbol(L):
    declared = _declared_symbols()
    assert declared >= {"fdl_denoise_step", "fdl_block_attn", "fdl_dualcache_attn",
                        "fdl_lmhead_confidence", "fdl_threshold_commit"}
    for name in declared:
        assert hasattr(L, name), name
    assert declared == set(fdl.SYMBOLS) | (declared - set(fdl.SYMBOLS))
    assert set(fdl.SYMBOLS) <= declared


def test_version(L):
    assert L.fdl_version() == 1


def _cfg(**kw):
    c = dict(synth.CONFIGS["qwen7b"], q_off=8)
    c.update(kw)
    return fdl.make_cfg(c)


@pytest.mark.parametrize("bad,msg", [
    (dict(batch=0), "batch"),
    (dict(n_kv_heads=3), "multiple"),
    (dict(head_dim=96), "head_dim"),
    (dict(q_off=28), "unit"),
    (dict(q_len=33), "q_len"),
    (dict(mask_id=152064), "mask_id"),
    (dict(shift=2), "shift"),
    (dict(tau=float("nan")), "tau"),
    (dict(hidden=100), "hidden"),
    (dict(batch=33), "256"),
    (dict(dtype=""), "dtype"),
])
def test_invalid_configs_are_rejected(L, bad, msg):
    c = dict(synth.CONFIGS["qwen7b"], q_off=8)
    c.update(bad)
    cfg = fdl.make_cfg(c) if bad.get("dtype") != "" else _cfg()
    if bad.get("dtype") == "":
        cfg.dtype = 7
    assert L.fdl_workspace_size(ctypes.byref(cfg)) == 0
    assert msg in fdl.last_error()
    rc = L.fdl_block_attn(ctypes.byref(cfg), *([None] * 7), None, 0, None)
    assert rc == fdl.ERR_INVALID_ARG


def test_workspace_size_grows_with_the_problem(L):
    small = L.fdl_workspace_size(ctypes.byref(_cfg(batch=1)))
    big = L.fdl_workspace_size(ctypes.byref(_cfg(batch=16, cap_prefix=8192)))
    assert 0 < small < big
    assert small % 256 == 0 and big % 256 == 0


def _fake(n=1):
    # addresses are never dereferenced: every call below fails its checks first
    return [ctypes.c_void_p(0x10000 * (i + 1)) for i in range(n)]


def test_null_and_misaligned_pointers_are_rejected(L):
    cfg = _cfg()
    p = _fake(7)
    rc = L.fdl_block_attn(ctypes.byref(cfg), None, *p[1:7], None, 0, None)
    assert rc == fdl.ERR_INVALID_ARG and "q is NULL" in fdl.last_error()
    mis = ctypes.c_void_p(0x10008)
    rc = L.fdl_block_attn(ctypes.byref(cfg), mis, *p[1:7], None, 0, None)
    assert rc == fdl.ERR_INVALID_ARG and "aligned" in fdl.last_error()


def test_workspace_checks(L):
    cfg = _cfg()
    need = L.fdl_workspace_size(ctypes.byref(cfg))
    p = _fake(7)
    rc = L.fdl_block_attn(ctypes.byref(cfg), *p, None, need, None)
    assert rc == fdl.ERR_WORKSPACE and "NULL" in fdl.last_error()
    rc = L.fdl_block_attn(ctypes.byref(cfg), *p, ctypes.c_void_p(0x20080), need, None)
    assert rc == fdl.ERR_WORKSPACE and "256" in fdl.last_error()
    rc = L.fdl_block_attn(ctypes.byref(cfg), *p, ctypes.c_void_p(0x20000), need - 256, None)
    assert rc == fdl.ERR_WORKSPACE and "needs" in fdl.last_error()


def test_denoise_step_argument_rules(L):
    cfg = _cfg()
    need = L.fdl_workspace_size(ctypes.byref(cfg))
    p = _fake(20)
    ws = ctypes.c_void_p(0x100000)
    args = list(p[:19])
    # suffix pointers must come together
    a = list(args)          # q, k_pre, v_pre, len_pre, k_blk, v_blk, k_suf(6),
    a[6] = None             # v_suf(7), len_suf(8), hidden(9), h_prev(10), ...
    a[8] = None
    rc = L.fdl_denoise_step(ctypes.byref(cfg), *a, ws, need, None)
    assert rc == fdl.ERR_INVALID_ARG and "all be set" in fdl.last_error()
    # shift needs h_prev
    a = list(args)
    a[6] = a[7] = a[8] = None
    a[10] = None
    rc = L.fdl_denoise_step(ctypes.byref(cfg), *a, ws, need, None)
    assert rc == fdl.ERR_INVALID_ARG and "h_prev" in fdl.last_error()
    # attention output as LM-head input needs hidden == Hq * d
    cfg2 = _cfg(hidden=1024)
    a = list(args)
    a[6] = a[7] = a[8] = None
    a[9] = None
    rc = L.fdl_denoise_step(ctypes.byref(cfg2), *a, ws, need, None)
    assert rc == fdl.ERR_INVALID_ARG and "Hq*d" in fdl.last_error()


def test_last_error_is_cleared_by_success(L):
    L.fdl_workspace_size(ctypes.byref(_cfg(batch=0)))
    assert fdl.last_error() != ""
    assert L.fdl_workspace_size(ctypes.byref(_cfg())) > 0
    assert fdl.last_error() == ""
