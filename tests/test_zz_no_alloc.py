"""The allocation-free LM-head entry point (for callers that cannot allocate
device memory: its scratch is a fixed array inside the library) must give
the same result as the workspace entry point.  Collected last on purpose, so
a run that stops at the first failure has run every other test already; it
also passes alone in a fresh process."""
import numpy as np
import pytest
import torch

from block_diffusion_decoding_causal_b200 import fdl

pytestmark = pytest.mark.gpu


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


@pytest.mark.parametrize("R,V,H,dtype", [(32, 152064, 3584, torch.bfloat16),
                                         (128, 20000, 256, torch.bfloat16),
                                         (8, 512, 128, torch.float32)])
def test_noalloc_matches_workspace_entry_point_twice(R, V, H, dtype):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    cfg, rows, w, active = _case(R, V, H, dtype, R + V)
    conf_ref = torch.empty(R, dtype=torch.float32, device="cuda")
    tok_ref = torch.empty(R, dtype=torch.int32, device="cuda")
    ws = fdl.workspace(cfg)
    fdl.lmhead_confidence(cfg, rows, w, active, conf_ref, tok_ref, ws)
    for _ in range(2):                       # two calls in a row share the scratch
        conf = torch.full((R,), 7.0, device="cuda")
        tok = torch.full((R,), 7, dtype=torch.int32, device="cuda")
        fdl.lmhead_confidence_noalloc(cfg, rows, w, active, conf, tok)
        torch.cuda.synchronize()
        assert torch.equal(tok, tok_ref)
        rtol = 2e-2 if dtype == torch.bfloat16 else 1e-4
        np.testing.assert_allclose(conf.cpu().numpy(), conf_ref.cpu().numpy(), rtol=rtol)
    assert fdl.get_status(ws) == 0


def test_noalloc_rejects_more_rows_than_its_scratch_holds():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    cfg, rows, w, _ = _case(129, 1000, 64, torch.bfloat16, 1)
    conf = torch.empty(129, device="cuda")
    tok = torch.empty(129, dtype=torch.int32, device="cuda")
    with pytest.raises(fdl.FdlError) as e:
        fdl.lmhead_confidence_noalloc(cfg, rows, w, None, conf, tok)
    assert e.value.code == fdl.ERR_UNSUPPORTED and "128" in str(e.value)
