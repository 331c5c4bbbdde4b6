"""The allocation-free LM-head entry point: for callers that cannot allocate
device memory (a plugin inside an engine that owns every allocation, a loop
that may not allocate after start-up), its scratch is a fixed array inside
the library.  It must give the same result as the workspace entry point,
allocate nothing, and report device-side failures through its own status
word.  Collected last on purpose, so a run that stops at the first failure
has run every other test already; it also passes alone in a fresh process."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from block_diffusion_decoding_causal_b200 import fdl

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _case(R, V, H, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    rows = torch.randn((R, H), generator=g).to(dtype)
    w = (torch.randn((V, H), generator=g) * (8.0 / H ** 0.5)).to(dtype)
    active = (torch.rand(R, generator=g) < 0.7).to(torch.uint8)
    cfg = fdl.make_cfg(dict(batch=R, n_q_heads=1, n_kv_heads=1, head_dim=32, block_size=1,
                            q_off=0, q_len=1, cap_prefix=0, hidden=H, vocab=V,
                            mask_id=V - 1, shift=0, tau=0.9,
                            dtype="bf16" if dtype == torch.bfloat16 else "f32"))
    return cfg, rows.cuda(), w.cuda(), active.cuda()


def _reference(cfg, rows, w, active, R):
    conf_ref = torch.empty(R, dtype=torch.float32, device="cuda")
    tok_ref = torch.empty(R, dtype=torch.int32, device="cuda")
    ws = fdl.workspace(cfg)
    fdl.lmhead_confidence(cfg, rows, w, active, conf_ref, tok_ref, ws)
    assert fdl.get_status(ws) == 0
    return conf_ref, tok_ref


@pytest.mark.parametrize("R,V,H,dtype", [(32, 152064, 3584, torch.bfloat16),
                                         (128, 20000, 256, torch.bfloat16),
                                         (8, 512, 128, torch.float32)])
def test_noalloc_matches_workspace_entry_point_twice(R, V, H, dtype):
    cfg, rows, w, active = _case(R, V, H, dtype, R + V)
    conf_ref, tok_ref = _reference(cfg, rows, w, active, R)
    for _ in range(2):                       # two calls in a row share the scratch
        conf = torch.full((R,), 7.0, device="cuda")
        tok = torch.full((R,), 7, dtype=torch.int32, device="cuda")
        fdl.lmhead_confidence_noalloc(cfg, rows, w, active, conf, tok)
        torch.cuda.synchronize()
        assert torch.equal(tok, tok_ref)
        rtol = 2e-2 if dtype == torch.bfloat16 else 1e-4
        np.testing.assert_allclose(conf.cpu().numpy(), conf_ref.cpu().numpy(), rtol=rtol)
    assert fdl.lmhead_noalloc_status() == 0


def test_noalloc_allocates_no_device_memory():
    R, V, H = 32, 20000, 512
    cfg, rows, w, active = _case(R, V, H, torch.bfloat16, 5)
    conf = torch.empty(R, device="cuda")
    tok = torch.empty(R, dtype=torch.int32, device="cuda")
    fdl.lmhead_confidence_noalloc(cfg, rows, w, active, conf, tok)   # loads the kernel
    torch.cuda.synchronize()
    torch_before = torch.cuda.memory_allocated()
    free_before = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        fdl.lmhead_confidence_noalloc(cfg, rows, w, active, conf, tok)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == torch_before
    assert torch.cuda.mem_get_info()[0] == free_before
    assert fdl.lmhead_noalloc_status() == 0


def test_noalloc_reports_a_timeout_through_its_own_status_word():
    """A bounded wait run out on purpose against the static scratch's status
    word (no fault): while the bit is set every row reports conf = -1 and
    tok = -1; reading the status returns the bit and clears it; after a reset
    the entry point is correct again."""
    R, V, H = 16, 5000, 256
    cfg, rows, w, active = _case(R, V, H, torch.bfloat16, 9)
    conf_ref, tok_ref = _reference(cfg, rows, w, active, R)
    conf = torch.empty(R, device="cuda")
    tok = torch.empty(R, dtype=torch.int32, device="cuda")
    fdl.lmhead_noalloc_check_wait_timeout(limit_cycles=1_000_000)
    fdl.lmhead_confidence_noalloc(cfg, rows, w, active, conf, tok)
    torch.cuda.synchronize()
    assert (conf.cpu() == -1).all() and (tok.cpu() == -1).all()
    assert fdl.lmhead_noalloc_status() & fdl.DEV_TIMEOUT
    assert fdl.lmhead_noalloc_status() == 0                 # read and cleared
    fdl.lmhead_noalloc_reset()
    fdl.lmhead_confidence_noalloc(cfg, rows, w, active, conf, tok)
    torch.cuda.synchronize()
    assert torch.equal(tok, tok_ref)
    np.testing.assert_allclose(conf.cpu().numpy(), conf_ref.cpu().numpy(), rtol=2e-2)
    assert fdl.lmhead_noalloc_status() == 0


_FRESH = r"""
import numpy as np, torch
from block_diffusion_decoding_causal_b200 import fdl
g = torch.Generator().manual_seed(3)
R, V, H = 24, 30000, 512
rows = torch.randn((R, H), generator=g).to(torch.bfloat16).cuda()
w = (torch.randn((V, H), generator=g) * (8.0 / H ** 0.5)).to(torch.bfloat16).cuda()
cfg = fdl.make_cfg(dict(batch=R, n_q_heads=1, n_kv_heads=1, head_dim=32, block_size=1,
                        q_off=0, q_len=1, cap_prefix=0, hidden=H, vocab=V, mask_id=V - 1,
                        shift=0, tau=0.9, dtype="bf16"))
s = torch.cuda.Stream()
conf = torch.empty(R, device="cuda")
tok = torch.empty(R, dtype=torch.int32, device="cuda")
with torch.cuda.stream(s):
    fdl.lmhead_confidence_noalloc(cfg, rows, w, None, conf, tok, stream=s)
s.synchronize()
ws = fdl.workspace(cfg)
conf_ref = torch.empty(R, device="cuda")
tok_ref = torch.empty(R, dtype=torch.int32, device="cuda")
fdl.lmhead_confidence(cfg, rows, w, None, conf_ref, tok_ref, ws)
torch.cuda.synchronize()
assert torch.equal(tok, tok_ref), "tokens differ"
np.testing.assert_allclose(conf.cpu().numpy(), conf_ref.cpu().numpy(), rtol=2e-2)
assert fdl.lmhead_noalloc_status(stream=s) == 0
print("FRESH_OK")
"""


def test_noalloc_first_call_in_a_fresh_process_on_a_side_stream():
    """The first call on a device queues the zeroing of the scratch's control
    words on the caller's stream; on a non-blocking side stream that must
    still come before the kernel."""
    env = dict(os.environ, PYTHONPATH=ROOT + os.pathsep + os.environ.get("PYTHONPATH", ""))
    r = subprocess.run([sys.executable, "-c", _FRESH], capture_output=True, text=True,
                       timeout=300, env=env, cwd=ROOT)
    assert r.returncode == 0 and "FRESH_OK" in r.stdout, r.stdout + r.stderr


def test_noalloc_rejects_more_rows_than_its_scratch_holds():
    R = fdl.NOALLOC_MAX_ROWS + 1
    cfg, rows, w, _ = _case(R, 1000, 64, torch.bfloat16, 1)
    conf = torch.empty(R, device="cuda")
    tok = torch.empty(R, dtype=torch.int32, device="cuda")
    with pytest.raises(fdl.FdlError) as e:
        fdl.lmhead_confidence_noalloc(cfg, rows, w, None, conf, tok)
    assert e.value.code == fdl.ERR_UNSUPPORTED and str(fdl.NOALLOC_MAX_ROWS) in str(e.value)
