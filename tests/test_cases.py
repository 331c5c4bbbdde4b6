"""Host-side checks of the seeded generator and the margin-repaired cases."""
import numpy as np
import torch

from block_diffusion_decoding_causal_b200 import synth
from oracle import cases


def test_generator_is_deterministic_and_stream_separated():
    a = synth.make_case("tiny", 3)
    b = synth.make_case("tiny", 3)
    c = synth.make_case("tiny", 4)
    for name in ["q", "k_pre", "v_pre", "k_blk", "v_blk", "hidden", "w_lm", "block_tokens"]:
        assert torch.equal(getattr(a, name), getattr(b, name))
        assert not torch.equal(getattr(a, name), getattr(c, name))
    # changing one config entry does not move another tensor's values
    d = synth.make_case("tiny", 3, tau=0.5)
    assert torch.equal(a.w_lm, d.w_lm) and torch.equal(a.q, d.q)


def test_generator_shapes_and_block_tokens():
    c = synth.make_case("qwen7b", 1, vocab=4096, hidden=256, n_q_heads=4,
                        n_kv_heads=2, head_dim=64, prefix=(40, 90), cap_prefix=96,
                        mask_id=4000)
    cfg = c.cfg
    B, D, q_off, q_len = cfg["batch"], cfg["block_size"], cfg["q_off"], cfg["q_len"]
    assert c.q.shape == (B, q_len, 4, 64) and c.q.dtype == torch.bfloat16
    assert c.k_pre.shape == (B, 2, 96, 64)
    assert ((c.len_pre >= 40) & (c.len_pre <= 90)).all()
    assert ((c.len_pre - c.prompt_len) % D == 0).all()
    t = c.block_tokens
    mask = cfg["mask_id"]
    assert (t[:, q_off + q_len:] == mask).all()
    assert (t[:, :q_off] != mask).all()
    n_m = (t[:, q_off:q_off + q_len] == mask).sum(1)
    assert ((n_m >= cfg["masked"][0]) & (n_m <= cfg["masked"][1])).all()
    assert (t >= 0).all() and (t < cfg["vocab"]).all()


def test_tiny_parity_case_margins_hold():
    case, res, redrawn = cases.parity_case("tiny", 11)
    act = res["active"]
    assert act.sum() == 4
    tau = res["tau"]
    assert (res["logit_gap"][act] >= cases.GAP).all()
    assert (np.abs(res["conf"][act] - tau) >= cases.CONF_MARGIN).all()
    assert (res["conf"][~act] == -1).all() and (res["tok"][~act] == -1).all()
    # the commit wrote exactly the committed positions and nothing else
    bt0 = case.block_tokens.numpy()
    changed = res["block_tokens"] != bt0
    assert np.array_equal(changed.astype(np.uint8), res["committed"] & changed)
    assert res["n_committed"][0] == res["committed"].sum() >= 1
    again = cases.parity_case("tiny", 11)
    assert np.array_equal(again[1]["block_tokens"], res["block_tokens"]) and again[2] == redrawn


def test_attention_as_hidden_case_repairs_query_rows():
    case, res, _ = cases.parity_case("tiny", 5, attn_as_hidden=True)
    assert case.hidden is None
    assert np.array_equal(res["rows"], res["attn_rounded"].reshape(res["rows"].shape))
