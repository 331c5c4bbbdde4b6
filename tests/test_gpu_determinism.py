"""Repeatability: the same inputs give bit-identical outputs call after call.

Every reduction on the CUDA path sums in a fixed order: the stream-K split of
the attention and its merge kernel, the in-kernel row merge of the attention
beside the LM head, and the two-level merge of the LM head's per-CTA partials
(teams of CTAs, then the teams, each in index order).  None depends on which
CTA finishes first, so two calls must agree bit for bit, not merely within a
tolerance.  Shapes follow the Qwen2.5-7B workloads (full vocabulary).
"""
import pytest
import torch

from block_diffusion_decoding_causal_b200 import fdl, synth
from oracle import step
from tests import gpu_harness as gh

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


@pytest.mark.parametrize("batch", [1, 4, 16, 32])
def test_lmhead_repeats_bit_for_bit(batch):
    """8, 32, 128 and 256 rows: the one-CTA kernel (both epilogue forms) and
    the CTA-pair kernel, over the tiled weight."""
    c = dict(synth.CONFIGS["qwen7b"], batch=batch, q_off=0)
    cfg = fdl.make_cfg(c)
    V, H, R = c["vocab"], c["hidden"], batch * c["q_len"]
    g = torch.Generator(device="cuda").manual_seed(batch)
    w_rm = (torch.randn((V, H), generator=g, device="cuda") * (8.0 / H ** 0.5)).to(torch.bfloat16)
    w = torch.empty_like(w_rm)
    fdl.lmhead_pack_weight(cfg, w_rm, w)
    del w_rm
    cfg.w_layout = fdl.W_PACKED
    rows = torch.randn((R, H), generator=g, device="cuda").to(torch.bfloat16)
    ws = fdl.workspace(cfg)
    runs = []
    for _ in range(3):
        conf = torch.empty(R, dtype=torch.float32, device="cuda")
        tok = torch.empty(R, dtype=torch.int32, device="cuda")
        fdl.lmhead_confidence(cfg, rows, w, None, conf, tok, ws)
        torch.cuda.synchronize()
        runs.append((conf.cpu(), tok.cpu()))
    for conf, tok in runs[1:]:
        assert torch.equal(tok, runs[0][1])
        assert torch.equal(conf.view(torch.int32), runs[0][0].view(torch.int32))
    assert fdl.get_status(ws) == 0


@pytest.mark.parametrize("batch,prefix", [(16, 8192), (4, 8192), (1, 8192), (4, 2048)])
def test_attention_repeats_bit_for_bit(batch, prefix):
    """The attention entry point alone: stream-K over 296 CTAs, partials
    combined by the merge kernel (narrow form at batch 4 and 16, lanes over
    the partials at batch 1)."""
    c = synth.sweep_config(batch, prefix)
    c["q_off"] = 0
    cfg = fdl.make_cfg(c)
    Hq, Hkv, d, D, q_len = c["n_q_heads"], c["n_kv_heads"], c["head_dim"], c["block_size"], c["q_len"]
    g = torch.Generator(device="cuda").manual_seed(batch * 10 + prefix)
    rn = lambda *s: torch.randn(s, generator=g, device="cuda").to(torch.bfloat16)
    q = rn(batch, q_len, Hq, d)
    kp, vp = rn(batch, Hkv, prefix, d), rn(batch, Hkv, prefix, d)
    kb, vb = rn(batch, Hkv, D, d), rn(batch, Hkv, D, d)
    lens = torch.randint(prefix // 2, prefix + 1, (batch,), generator=g, device="cuda",
                         dtype=torch.int32)
    ws = fdl.workspace(cfg)
    outs = []
    for _ in range(3):
        out = torch.empty_like(q)
        fdl.block_attn(cfg, q, kp, vp, lens, kb, vb, out, ws)
        torch.cuda.synchronize()
        outs.append(out.cpu())
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
    assert fdl.get_status(ws) == 0


def test_fused_step_repeats_bit_for_bit():
    """The fused step at the benchmark shapes (attention beside the LM head,
    rows merged inside the attention kernel, commit in the LM head's final
    merge), from the same block state each time."""
    case = synth.make_case("qwen7b", 11)
    d = gh.device_case(case)
    cfg = fdl.make_cfg(case.cfg)
    ws = fdl.workspace(cfg)
    runs = [gh.run_denoise_step(case, ws=ws, d=d, packed=True) for _ in range(3)]
    for r in runs[1:]:
        for k in ("conf", "attn"):
            assert torch.equal(r[k].view(torch.int16 if r[k].dtype == torch.bfloat16
                                         else torch.int32),
                               runs[0][k].view(torch.int16 if runs[0][k].dtype == torch.bfloat16
                                               else torch.int32)), k
        for k in ("tok", "committed", "n_committed", "n_masked_left", "block_tokens"):
            assert torch.equal(r[k], runs[0][k]), k
        assert r["status"] == 0


@pytest.mark.parametrize("batch,prefix", [(4, 8192), (1, 8192), (4, 2048)])
def test_attention_calls_back_to_back(batch, prefix):
    """Consecutive standalone attention calls on one stream and one
    workspace with no synchronisation between them.  Each launch is a
    programmatic dependent of the previous call's merge kernel: it starts
    during that merge and must wait for it before reading its lengths or
    reusing the workspace's tickets and partial slots.  Three different
    inputs (ragged prefix lengths), each output against the oracle; at
    prefix 8192 batch 1 merges tens of partials per item (the wide merge),
    batch 4 about twenty."""
    outs, cases_ = [], []
    c = dict(synth.sweep_config(batch, prefix), prefix=(prefix // 2, prefix))
    for seed in (21, 22, 23):
        case = synth.make_case("sweep", seed, cfg=c, draw_w=False)
        cases_.append((case, fdl.make_cfg(case.cfg), gh.device_case(case)))
    ws = fdl.workspace(cases_[0][1])  # same geometry; the unit offset differs
    torch.cuda.synchronize()
    for case, cfg, d in cases_:
        out = torch.empty_like(d["q"])
        fdl.block_attn(cfg, d["q"], d["k_pre"], d["v_pre"], d["len_pre"], d["k_blk"],
                       d["v_blk"], out, ws)
        outs.append(out)
    torch.cuda.synchronize()
    assert fdl.get_status(ws) == 0
    for (case, _, _), out in zip(cases_, outs):
        ref = step.attention_step(case.q, case.k_pre, case.v_pre, case.len_pre.numpy(),
                                  case.prompt_len.numpy(), case.k_blk, case.v_blk,
                                  case.cfg["q_off"])
        gh.assert_close_scaled(out.double().cpu().numpy(), ref, 2e-2, "attn")


def test_two_pass_launch_matches_two_single_passes():
    """512 rows (two passes of 256 in one launch of the CTA pairs, the first
    pass's merges on a second ticket set under the second pass's stream)
    return the very same bits as the two halves called one by one: the
    arithmetic of each pass is unchanged by sharing a launch."""
    c = dict(synth.CONFIGS["qwen7b"], batch=64, q_off=0)
    V, H = c["vocab"], c["hidden"]
    g = torch.Generator(device="cuda").manual_seed(512)
    w_rm = (torch.randn((V, H), generator=g, device="cuda") * (8.0 / H ** 0.5)).to(torch.bfloat16)
    cfg = fdl.make_cfg(c)
    w = torch.empty_like(w_rm)
    fdl.lmhead_pack_weight(cfg, w_rm, w)
    del w_rm
    rows = torch.randn((512, H), generator=g, device="cuda").to(torch.bfloat16)
    cfg.w_layout = fdl.W_PACKED
    conf = torch.empty(512, dtype=torch.float32, device="cuda")
    tok = torch.empty(512, dtype=torch.int32, device="cuda")
    ws = fdl.workspace(cfg)
    fdl.lmhead_confidence(cfg, rows, w, None, conf, tok, ws)
    half = fdl.make_cfg(dict(c, batch=32))
    half.w_layout = fdl.W_PACKED
    ws_h = fdl.workspace(half)
    conf_h = torch.empty(512, dtype=torch.float32, device="cuda")
    tok_h = torch.empty(512, dtype=torch.int32, device="cuda")
    for r0 in (0, 256):
        fdl.lmhead_confidence(half, rows[r0:r0 + 256], w, None, conf_h[r0:r0 + 256],
                              tok_h[r0:r0 + 256], ws_h)
    torch.cuda.synchronize()
    assert torch.equal(tok.cpu(), tok_h.cpu())
    assert torch.equal(conf.cpu().view(torch.int32), conf_h.cpu().view(torch.int32))
    assert fdl.get_status(ws) == 0 and fdl.get_status(ws_h) == 0
