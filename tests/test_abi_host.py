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


def _declared_arity():
    """Parameter count of every fdl_* function include/*.h declares."""
    out = {}
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            for name, params in re.findall(r"\b(fdl_[a-z0-9_]+)\s*\(([^)]*)\)\s*;", src):
                params = params.strip()
                out[name] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_argument_counts_match_the_header(L):
    arity = _declared_arity()
    assert set(fdl.SYMBOLS) <= set(arity)
    for name in fdl.SYMBOLS:
        fn = getattr(L, name)
        if fn.argtypes is not None:
            assert len(fn.argtypes) == arity[name], name


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
    (dict(block_size=5000), "block_size"),
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


def test_loop_control_and_append_reject_bad_arguments(L):
    cfg = _cfg()
    nl = ctypes.c_void_p(16)        # never dereferenced: rejected before any launch
    rc = L.fdl_unit_status(ctypes.byref(cfg), None, None, None, 0, None)
    assert rc == fdl.ERR_INVALID_ARG and "n_masked_left" in fdl.last_error()
    rc = L.fdl_unit_status(ctypes.byref(cfg), nl, None, None, 12345, None)
    assert rc == fdl.ERR_INVALID_ARG and "step_count" in fdl.last_error()
    rc = L.fdl_append_block(ctypes.byref(cfg), None, nl, nl, nl, nl, nl, 1 << 30, None)
    assert rc == fdl.ERR_INVALID_ARG
    small = _cfg(cap_prefix=16)
    rc = L.fdl_append_block(ctypes.byref(small), nl, nl, nl, nl, nl, nl, 1 << 30, None)
    assert rc == fdl.ERR_INVALID_ARG and "cap_prefix" in fdl.last_error()
    rc = L.fdl_select_commit(ctypes.byref(cfg), 7, 1.0, nl, nl, nl, nl, nl, nl, None)
    assert rc == fdl.ERR_INVALID_ARG


def test_prefixcache_needs_every_recomputed_row_as_a_query(L):
    c = dict(synth.CONFIGS["llada"], block_size=288, q_len=280, q_off=8, cap_suffix=0)
    cfg = fdl.make_cfg(c)
    rc = L.fdl_prefixcache_attn(ctypes.byref(cfg), *([None] * 7), None, 0, None)
    assert rc == fdl.ERR_INVALID_ARG and "q_off = 0" in fdl.last_error()


def test_wide_attention_shapes_only_on_the_tensor_core_path(L):
    big = dict(synth.CONFIGS["llada"], block_size=768, q_len=768, q_off=0, cap_suffix=0)
    assert L.fdl_workspace_size(ctypes.byref(fdl.make_cfg(big))) > 0
    assert L.fdl_workspace_size(ctypes.byref(fdl.make_cfg(dict(big, dtype="f32")))) == 0
    assert "bf16" in fdl.last_error()
    assert L.fdl_workspace_size(ctypes.byref(fdl.make_cfg(dict(big, head_dim=64)))) == 0
    # the fused step keeps its own limits
    nl = ctypes.c_void_p(16)
    rc = L.fdl_threshold_commit(ctypes.byref(fdl.make_cfg(big)), nl, nl, nl, nl, nl, nl, None)
    assert rc == fdl.ERR_INVALID_ARG and "block_size" in fdl.last_error()


def test_step_rows_beyond_one_lm_pass_are_accepted_up_to_4096(L):
    ok = _cfg(batch=512, q_len=8, q_off=0)
    assert L.fdl_workspace_size(ctypes.byref(ok)) > 0
    too_many = _cfg(batch=513, q_len=8, q_off=0)
    assert L.fdl_workspace_size(ctypes.byref(too_many)) > 0      # attention-level only
    nl = ctypes.c_void_p(16)
    rc = L.fdl_threshold_commit(ctypes.byref(too_many), nl, nl, nl, nl, nl, nl, None)
    assert rc == fdl.ERR_INVALID_ARG and "4096" in fdl.last_error()


def test_rows_past_one_pass_get_a_second_partial_region(L):
    """Past 256 LM-head rows the CTA-pair form runs two passes in one launch,
    each with its own region of per-CTA partials (up to 4 x 148 CTAs x 256
    rows x 16 bytes): crossing from 256 to 264 rows adds at least that much
    workspace, while 8 more rows below one pass add little."""
    region = 4 * 148 * 256 * 16
    size = lambda b: L.fdl_workspace_size(ctypes.byref(_cfg(batch=b, q_len=8, q_off=0)))
    assert size(33) - size(32) >= region
    assert size(32) - size(31) < region // 4


def test_wait_timeout_check_rejects_bad_arguments(L):
    rc = L.fdl_check_wait_timeout(None, 256, 1000000, None)
    assert rc == fdl.ERR_WORKSPACE
    rc = L.fdl_check_wait_timeout(ctypes.c_void_p(256), 256, 10, None)
    assert rc == fdl.ERR_INVALID_ARG and "limit_cycles" in fdl.last_error()


def test_noalloc_helpers_reject_bad_arguments(L):
    assert L.fdl_lmhead_noalloc_status(None, None) == fdl.ERR_INVALID_ARG
    rc = L.fdl_lmhead_noalloc_check_wait_timeout(10, None)
    assert rc == fdl.ERR_INVALID_ARG and "limit_cycles" in fdl.last_error()


def test_noalloc_limits_in_header_match_binding(tmp_path):
    """FDL_NOALLOC_MAX_ROWS and FDL_NOALLOC_SCRATCH_BYTES as the C compiler
    reads them from include/fdl.h (the library static_asserts the latter
    against its own array); the binding's row limit agrees."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "limits.c"
    src.write_text("#include <stdio.h>\n#include \"fdl.h\"\n"
                   "int main(void) { printf(\"%d %d\\n\", FDL_NOALLOC_MAX_ROWS, "
                   "FDL_NOALLOC_SCRATCH_BYTES); return 0; }\n")
    exe = tmp_path / "limits"
    include = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                           "include")
    subprocess.run([cc, "-I", include, str(src), "-o", str(exe)], check=True)
    rows, nbytes = map(int, subprocess.run([str(exe)], check=True, capture_output=True,
                                           text=True).stdout.split())
    assert rows == fdl.NOALLOC_MAX_ROWS
    assert nbytes == 256 + 16 * 296 * rows


def test_weight_layout_rules(L):
    bad = _cfg()
    bad.w_layout = 2
    assert L.fdl_workspace_size(ctypes.byref(bad)) == 0
    assert "w_layout" in fdl.last_error()
    p = _fake(2)
    assert L.fdl_lmhead_pack_weight(None, *p, None) == fdl.ERR_INVALID_ARG
    f32 = _cfg(dtype="f32")
    assert L.fdl_lmhead_pack_weight(ctypes.byref(f32), *p, None) == fdl.ERR_UNSUPPORTED
    assert L.fdl_lmhead_pack_weight(ctypes.byref(_cfg(hidden=96)), *p, None) == \
        fdl.ERR_UNSUPPORTED
    rc = L.fdl_lmhead_pack_weight(ctypes.byref(_cfg()), None, p[1], None)
    assert rc == fdl.ERR_INVALID_ARG and "NULL" in fdl.last_error()
    # a 152064 x 3584 bf16 weight spans 1.09 GB: these two ranges overlap
    rc = L.fdl_lmhead_pack_weight(ctypes.byref(_cfg()), ctypes.c_void_p(0x10000000),
                                  ctypes.c_void_p(0x20000000), None)
    assert rc == fdl.ERR_INVALID_ARG and "overlap" in fdl.last_error()
    # the fp32 LM head has no tiled form
    f32.w_layout = fdl.W_PACKED
    q = _fake(4)
    rc = L.fdl_lmhead_confidence(ctypes.byref(f32), q[0], q[1], None, q[2], q[3], None, 0, None)
    assert rc == fdl.ERR_UNSUPPORTED and "bf16" in fdl.last_error()
    rc = L.fdl_lmhead_confidence_noalloc(ctypes.byref(f32), q[0], q[1], None, q[2], q[3], None)
    assert rc == fdl.ERR_UNSUPPORTED and "bf16" in fdl.last_error()


def test_step_cfg_layout_matches_the_header(tmp_path):
    """The binding's StepCfg has the size and field offsets of fdl_step_cfg
    as the C compiler lays it out from include/fdl.h."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    names = [f[0] for f in fdl.StepCfg._fields_]
    src = tmp_path / "layout.c"
    src.write_text("#include <stddef.h>\n#include <stdio.h>\n#include \"fdl.h\"\n"
                   "int main(void) {\n"
                   "  printf(\"size %zu\\n\", sizeof(fdl_step_cfg));\n"
                   + "".join(f'  printf("{n} %zu\\n", offsetof(fdl_step_cfg, {n}));\n'
                             for n in names)
                   + "  return 0;\n}\n")
    exe = tmp_path / "layout"
    include = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                           "include")
    subprocess.run([cc, "-I", include, str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    c_layout = dict(line.split() for line in out.splitlines())
    assert int(c_layout["size"]) == ctypes.sizeof(fdl.StepCfg)
    for n in names:
        assert int(c_layout[n]) == getattr(fdl.StepCfg, n).offset, n
