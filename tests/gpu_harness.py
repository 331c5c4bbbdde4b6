"""Shared helpers of the GPU parity tests: move a synthetic case to the
device, run the library through its C ABI, compare with the oracle."""
import numpy as np
import torch

from block_diffusion_decoding_causal_b200 import fdl

RTOL = {"bf16": 2e-2, "f32": 1e-4}


def dev(t):
    return None if t is None else t.cuda().contiguous()


def device_case(case):
    d = {k: dev(getattr(case, k)) for k in
         ["q", "k_pre", "v_pre", "len_pre", "k_blk", "v_blk", "k_suf", "v_suf",
          "len_suf", "hidden", "h_prev", "w_lm", "block_tokens"]}
    return d


def outputs(case):
    c = case.cfg
    B, q_len, D = c["batch"], c["q_len"], c["block_size"]
    dt = case.q.dtype
    return dict(
        attn=torch.empty((B, q_len, c["n_q_heads"], c["head_dim"]), dtype=dt, device="cuda"),
        conf=torch.empty((B, q_len), dtype=torch.float32, device="cuda"),
        tok=torch.empty((B, q_len), dtype=torch.int32, device="cuda"),
        committed=torch.empty((B, D), dtype=torch.uint8, device="cuda"),
        n_committed=torch.empty((B,), dtype=torch.int32, device="cuda"),
        n_masked_left=torch.empty((B,), dtype=torch.int32, device="cuda"))


def run_denoise_step(case, ws=None, d=None, keep_attn=True, packed=False):
    """fdl_denoise_step on a case; returns CPU copies of every output.
    packed: the LM-head weight is first rewritten into the tiled layout."""
    cfg = fdl.make_cfg(case.cfg)
    d = device_case(case) if d is None else d
    o = outputs(case)
    ws = fdl.workspace(cfg) if ws is None else ws
    bt = d["block_tokens"].clone()
    w_lm = d["w_lm"]
    if packed:
        w_lm = torch.empty_like(d["w_lm"])
        fdl.lmhead_pack_weight(cfg, d["w_lm"], w_lm)
        cfg.w_layout = fdl.W_PACKED
    fdl.denoise_step(cfg, d["q"], d["k_pre"], d["v_pre"], d["len_pre"], d["k_blk"],
                     d["v_blk"], d["k_suf"], d["v_suf"], d["len_suf"], d["hidden"],
                     d["h_prev"], w_lm, bt, o["attn"] if keep_attn else None,
                     o["conf"], o["tok"], o["committed"], o["n_committed"],
                     o["n_masked_left"], ws)
    torch.cuda.synchronize()
    res = {k: v.cpu() for k, v in o.items()}
    res["block_tokens"] = bt.cpu()
    res["status"] = fdl.get_status(ws)
    return res


def assert_close_scaled(got, want, rtol, what):
    """|got - want| <= rtol * (|want| + mean|want|), elementwise."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    scale = np.abs(want).mean() if want.size else 0.0
    err = np.abs(got - want)
    bound = rtol * (np.abs(want) + scale)
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} elements outside "
                           f"tolerance; worst err {err.max():.3e}")


def compare_step(case, gpu, ref, check_attn=True):
    dt = case.cfg["dtype"]
    rtol = RTOL[dt]
    if check_attn:
        assert_close_scaled(gpu["attn"].to(torch.float64).numpy(), ref["attn"], rtol,
                            "attention output")
    act = ref["active"]
    assert np.array_equal(gpu["tok"].numpy(), ref["tok"]), "argmax tokens differ"
    gc = gpu["conf"].numpy().astype(np.float64)
    assert np.array_equal(gc[~act], ref["conf"][~act])        # exactly -1
    np.testing.assert_allclose(gc[act], ref["conf"][act], rtol=rtol, atol=0)
    assert np.array_equal(gpu["block_tokens"].numpy(), ref["block_tokens"])
    assert np.array_equal(gpu["committed"].numpy(), ref["committed"])
    assert np.array_equal(gpu["n_committed"].numpy(), ref["n_committed"])
    assert np.array_equal(gpu["n_masked_left"].numpy(), ref["n_masked_left"])
    assert gpu["status"] == 0
