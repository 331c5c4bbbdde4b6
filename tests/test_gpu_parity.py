"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Bit-exact on committed token ids, argmax tokens, bitmaps and counts (inputs
are margin-repaired so no decision sits on a rounding boundary); within
2e-2 (bf16) or 1e-4 (fp32) relative for attention outputs and confidences.
"""
import numpy as np
import pytest
import torch

from block_diffusion_decoding_causal_b200 import fdl, synth
from oracle import cases, step
from tests import gpu_harness as gh
from tests.pack_layout import pack_reference

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


# ------------------------------------------------------------ fused step

@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_tiny_fp32_step(seed):
    case, ref, _ = cases.parity_case("tiny", seed)
    gh.compare_step(case, gh.run_denoise_step(case), ref)


@pytest.mark.parametrize("seed", [0, 1])
def test_tiny_fp32_step_attention_feeds_lm_head(seed):
    case, ref, _ = cases.parity_case("tiny", seed, attn_as_hidden=True)
    gh.compare_step(case, gh.run_denoise_step(case), ref)


@pytest.mark.parametrize("seed", [0, 1])
def test_qwen15b_step(seed):
    case, ref, _ = cases.parity_case("qwen1.5b", seed)
    gh.compare_step(case, gh.run_denoise_step(case), ref)


@pytest.mark.parametrize("tau", [0.7, 0.9])
def test_qwen7b_step(tau):
    case, ref, _ = cases.parity_case("qwen7b", 0, tau=tau)
    gh.compare_step(case, gh.run_denoise_step(case), ref)


def test_qwen7b_step_attention_feeds_lm_head():
    case, ref, _ = cases.parity_case("qwen7b", 3, attn_as_hidden=True)
    gh.compare_step(case, gh.run_denoise_step(case), ref)


def test_llada_dualcache_step():
    case, ref, _ = cases.parity_case("llada", 0)
    gh.compare_step(case, gh.run_denoise_step(case), ref)


# ------------------------------------------------------- ragged / edges

SMALL = dict(batch=3, n_q_heads=14, n_kv_heads=2, head_dim=64, block_size=16,
             q_len=5, q_off=None, prefix=(0, 300), cap_prefix=320, suffix=0,
             cap_suffix=0, hidden=448, vocab=5000, mask_id=4999, shift=1,
             tau=0.8, w_scale=8.0, dtype="bf16", masked=(1, 5))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_ragged_shapes_step(seed):
    """GQA group 7, q_len 5 (ragged row tiles), prefix lengths in [0, 300]
    (empty prefix included), vocab not a multiple of the tile."""
    lens = [0, 157, 300] if seed == 0 else None
    case, ref, _ = cases.parity_case("small", seed, cfg=SMALL, len_pre=lens)
    gh.compare_step(case, gh.run_denoise_step(case), ref)


def test_unit_of_one_position_mha():
    cfg = dict(SMALL, n_q_heads=4, n_kv_heads=4, q_len=1, masked=(1, 1), shift=0,
               head_dim=32, hidden=128, dtype="f32")
    case, ref, _ = cases.parity_case("one", 4, cfg=cfg)
    gh.compare_step(case, gh.run_denoise_step(case), ref)


def test_workspace_reuse_two_calls_in_a_row():
    case, ref, _ = cases.parity_case("qwen1.5b", 5)
    ws = fdl.workspace(fdl.make_cfg(case.cfg))
    d = gh.device_case(case)
    for _ in range(2):
        gh.compare_step(case, gh.run_denoise_step(case, ws=ws, d=d), ref)


def test_bad_prefix_length_sets_status_and_does_not_fault():
    case = synth.make_case("tiny", 0)
    case.len_pre[0] = case.cfg["cap_prefix"] + 5
    res = gh.run_denoise_step(case)
    assert res["status"] & fdl.DEV_BAD_PREFIX_LEN
    # processed as an empty prefix: attention over the block rows alone
    case.len_pre[0] = 0
    ref = cases.run_oracle(case)
    gh.assert_close_scaled(res["attn"].double().numpy(), ref["attn"], 1e-4, "attn")


# ------------------------------------------------- standalone entry points

def test_block_attn_entry_point():
    case = synth.make_case("qwen7b", 7)
    cfg = fdl.make_cfg(case.cfg)
    d = gh.device_case(case)
    out = torch.empty_like(d["q"])
    ws = fdl.workspace(cfg)
    fdl.block_attn(cfg, d["q"], d["k_pre"], d["v_pre"], d["len_pre"], d["k_blk"],
                   d["v_blk"], out, ws)
    ref = cases.run_oracle(case)
    gh.assert_close_scaled(out.double().cpu().numpy(), ref["attn"], 2e-2, "attn")


def test_dualcache_attn_entry_point():
    case = synth.make_case("llada", 2)
    cfg = fdl.make_cfg(case.cfg)
    d = gh.device_case(case)
    out = torch.empty_like(d["q"])
    ws = fdl.workspace(cfg)
    fdl.dualcache_attn(cfg, d["q"], d["k_pre"], d["v_pre"], d["len_pre"], d["k_blk"],
                       d["v_blk"], d["k_suf"], d["v_suf"], d["len_suf"], out, ws)
    ref = cases.run_oracle(case)
    gh.assert_close_scaled(out.double().cpu().numpy(), ref["attn"], 2e-2, "attn")


def test_lmhead_confidence_entry_point_with_row_mask():
    case, ref, _ = cases.parity_case("qwen7b", 1)
    cfg = fdl.make_cfg(case.cfg)
    rows = torch.from_numpy(ref["rows"]).to(case.w_lm.dtype).cuda().contiguous()
    active = torch.from_numpy(ref["active"].astype(np.uint8)).cuda()
    conf = torch.empty(ref["conf"].shape, dtype=torch.float32, device="cuda")
    tok = torch.empty(ref["conf"].shape, dtype=torch.int32, device="cuda")
    fdl.lmhead_confidence(cfg, rows, case.w_lm.cuda(), active, conf, tok,
                          fdl.workspace(cfg))
    act = ref["active"]
    assert np.array_equal(tok.cpu().numpy(), ref["tok"])
    c = conf.cpu().numpy().astype(np.float64)
    assert (c[~act] == -1).all()
    np.testing.assert_allclose(c[act], ref["conf"][act], rtol=2e-2)


def test_threshold_commit_entry_point_hand_cases():
    """Algorithm 2 on hand-made confidences, including the fallback, an exact
    tie, conf == tau and units with nothing masked."""
    B, D, q_off, q_len, mask = 5, 16, 8, 8, 99
    conf = np.array([
        [0.95, 0.91, 0.5, 0.99, 0.1, 0.1, 0.1, 0.1],   # several above tau
        [0.3, 0.8, 0.5, 0.8, 0.1, 0.2, 0.7, 0.6],      # fallback, tie -> lowest
        [0.9, 0.2, 0.3, 0.4, 0.5, 0.6, 0.7, 0.8],      # conf == tau commits
        [0.99] * 8,                                    # nothing masked
        [0.5] * 8,                                     # masked only at the end
    ], dtype=np.float32)
    tok = np.arange(B * q_len, dtype=np.int32).reshape(B, q_len) + 1000
    bt = np.full((B, D), mask, dtype=np.int32)
    bt[:, :q_off] = 7
    bt[3, q_off:] = 5
    bt[4, q_off:q_off + 6] = 6
    cfg = fdl.make_cfg(dict(batch=B, n_q_heads=1, n_kv_heads=1, head_dim=32,
                            block_size=D, q_off=q_off, q_len=q_len, cap_prefix=0,
                            hidden=8, vocab=2000, mask_id=mask, shift=0, tau=0.9,
                            dtype="f32"))
    d_bt = torch.from_numpy(bt).cuda()
    comm = torch.empty((B, D), dtype=torch.uint8, device="cuda")
    n_c = torch.empty(B, dtype=torch.int32, device="cuda")
    n_l = torch.empty(B, dtype=torch.int32, device="cuda")
    fdl.threshold_commit(cfg, torch.from_numpy(conf).cuda(), torch.from_numpy(tok).cuda(),
                         d_bt, comm, n_c, n_l)
    want = step.threshold_commit(bt, conf.astype(np.float64), tok, q_off, q_len, mask,
                                 float(np.float32(0.9)))
    assert np.array_equal(d_bt.cpu().numpy(), want[0])
    assert np.array_equal(comm.cpu().numpy(), want[1])
    assert np.array_equal(n_c.cpu().numpy(), want[2])
    assert np.array_equal(n_l.cpu().numpy(), want[3])
    assert want[2].tolist() == [3, 1, 1, 0, 1]


# ------------------------------------------------ full-size sweep points

@pytest.mark.parametrize("batch,prefix", [(16, 8192), (1, 8192)])
def test_sweep_full_size(batch, prefix):
    """Long-context sweep shapes at full size (prefix 8192, batch 16 = 128
    LM-head rows): every output against the oracle."""
    cfg = synth.sweep_config(batch, prefix, 8.0)
    case, ref, _ = cases.parity_case("sweep", 0, cfg=cfg)
    gpu = gh.run_denoise_step(case)
    gh.compare_step(case, gpu, ref, check_attn=True)


def _assert_regime(ref, regime):
    """The commit regime a case claims to exercise, read from the oracle.
    "fallback": no candidate reaches tau, so each unit with candidates
    commits exactly its single most confident position (Algorithm 2's
    fallback); "parallel": at least one unit commits several positions in
    this one step."""
    act, tau = ref["active"], ref["tau"]
    has_cand = act.any(axis=1)
    if regime == "fallback":
        assert (ref["conf"][act] < tau).all()
        assert (ref["n_committed"][has_cand] == 1).all()
    elif regime == "parallel":
        assert ref["n_committed"].max() > 1
    else:
        raise ValueError(regime)


@pytest.mark.parametrize("batch,prefix,scale,tau,regime", [
    (4, 2048, 4.0, 0.9, "fallback"),      # mostly below tau: the fallback decides
    (1, 2048, 4.0, 0.9, "fallback"),
    (4, 8192, 12.0, 0.9, "parallel"),     # mostly above tau: several commit at once
    (16, 2048, 12.0, 0.9, "parallel"),
    (4, 2048, 8.0, 0.7, "parallel"),      # the 7B workload's lower threshold
    (16, 8192, 4.0, 0.9, None),
])
def test_sweep_points_and_their_commit_regimes(batch, prefix, scale, tau, regime):
    """Long-context sweep points at full size over batch, prefix and logit
    scale (the confidence regime), each checked against the oracle and for
    the regime it is meant to exercise."""
    cfg = synth.sweep_config(batch, prefix, scale)
    cfg["tau"] = tau
    case, ref, _ = cases.parity_case("sweep", 0, cfg=cfg)
    if regime is not None:
        _assert_regime(ref, regime)
    gh.compare_step(case, gh.run_denoise_step(case), ref, check_attn=True)


@pytest.mark.parametrize("seed,regime", [(1, None), (2, "parallel")])
def test_llada_dualcache_step_more_seeds(seed, regime):
    case, ref, _ = cases.parity_case("llada", seed)
    if regime is not None:
        _assert_regime(ref, regime)
    gh.compare_step(case, gh.run_denoise_step(case), ref)


# ---------------------------------------------- LM head shapes and tails

@pytest.mark.parametrize("R,V,H", [(1, 5000, 64), (32, 5000, 448), (33, 33000, 128),
                                   (128, 20000, 256), (256, 7001, 64), (8, 151936, 1536),
                                   (256, 152064, 256), (200, 152064, 128),
                                   (256, 152885, 256), (144, 21000, 128)])
def test_lmhead_shapes_against_oracle(R, V, H):
    """Every N padding (32..256), partial vocab tiles (5000 / 148 CTAs = 48
    rows each), ragged vocab ends and several K depths.  From 129 rows the
    CTA pairs: at the 7B vocabulary 1040 rows per CTA, eight full tiles and
    a 16-row short tile folded into the first one (operands swapped); at
    V = 152885 the last pair's odd CTA holds 5 rows (its short-tile and most
    of its tile rows masked); at V = 21000, 144 rows per CTA, one full tile
    and the folded one.  Tokens must match wherever the oracle's top-2 logit
    gap exceeds 1e-3 (fp32 accumulation error is ~1e-5 at these sizes);
    confidences within 1e-3 relative."""
    g = torch.Generator().manual_seed(R * 7 + V + H)
    rows = torch.randn((R, H), generator=g).to(torch.bfloat16)
    w = (torch.randn((V, H), generator=g) * (8.0 / H ** 0.5)).to(torch.bfloat16)
    cfg = fdl.make_cfg(dict(batch=R, n_q_heads=1, n_kv_heads=1, head_dim=32,
                            block_size=1, q_off=0, q_len=1, cap_prefix=0, hidden=H,
                            vocab=V, mask_id=V - 1, shift=0, tau=0.9, dtype="bf16"))
    conf = torch.empty(R, dtype=torch.float32, device="cuda")
    tok = torch.empty(R, dtype=torch.int32, device="cuda")
    ws = fdl.workspace(cfg)
    for _ in range(2):                       # the second call reuses the workspace
        fdl.lmhead_confidence(cfg, rows.cuda(), w.cuda(), None, conf, tok, ws)
        torch.cuda.synchronize()
        t_ref, c_ref, gap = step.lmhead_confidence(rows.double().numpy(), w.float().numpy())
        t_gpu = tok.cpu().numpy()
        sure = gap > 1e-3
        assert np.array_equal(t_gpu[sure], t_ref[sure])
        np.testing.assert_allclose(conf.cpu().numpy().astype(np.float64), c_ref, rtol=1e-3)
    assert fdl.get_status(ws) == 0


# ------------------------------------------- attention split bookkeeping

EDGE = dict(batch=1, n_q_heads=1, n_kv_heads=1, head_dim=128, block_size=32,
            q_len=1, q_off=0, prefix=(0, 0), cap_prefix=64, suffix=0, cap_suffix=0,
            hidden=128, vocab=1000, mask_id=999, shift=0, tau=0.9, w_scale=8.0,
            dtype="bf16", masked=(1, 1))


@pytest.mark.parametrize("over", [
    dict(),                                                    # one chunk in total
    dict(n_q_heads=8, q_len=8, prefix=(8192, 8192), cap_prefix=8192),  # 1 item, ~129 CTAs
    dict(batch=3, n_q_heads=4, n_kv_heads=2, q_len=8, prefix=(1, 5000), cap_prefix=5000),
    dict(batch=2, n_q_heads=32, n_kv_heads=1, q_len=32, prefix=(100, 700), cap_prefix=700),
    dict(batch=2, n_q_heads=6, n_kv_heads=3, q_len=3, prefix=(60, 70), cap_prefix=80,
         suffix=130, cap_suffix=130),                          # DualCache, short
])
@pytest.mark.parametrize("path", ["entry", "step"])
def test_attention_split_extremes(over, path):
    """Stream-K partition edges: fewer chunks than CTAs, one item spread over
    most CTAs, row tiles of 128 (group 32 x 4 positions), DualCache.  "entry":
    the attention entry points (two CTAs per SM, merge kernel); "step": the
    fused step, where the attention runs beside the LM head (one CTA per SM,
    partials merged inside the kernel); only its attention output is checked
    here."""
    cfg = dict(EDGE, **over)
    case = synth.make_case("edge", 3, cfg=cfg)
    c = fdl.make_cfg(case.cfg)
    d = gh.device_case(case)
    out = torch.empty_like(d["q"])
    ws = fdl.workspace(c)
    for _ in range(2):
        if path == "step":
            gh.run_denoise_step(case, ws=ws, d=d)
            res = gh.run_denoise_step(case, ws=ws, d=d)
            ref = cases.run_oracle(case)
            gh.assert_close_scaled(res["attn"].double().numpy(), ref["attn"], 2e-2, "attn")
            assert res["status"] == 0
            continue
        if case.k_suf is None:
            fdl.block_attn(c, d["q"], d["k_pre"], d["v_pre"], d["len_pre"], d["k_blk"],
                           d["v_blk"], out, ws)
        else:
            fdl.dualcache_attn(c, d["q"], d["k_pre"], d["v_pre"], d["len_pre"], d["k_blk"],
                               d["v_blk"], d["k_suf"], d["v_suf"], d["len_suf"], out, ws)
        ref = cases.run_oracle(case)
        gh.assert_close_scaled(out.double().cpu().numpy(), ref["attn"], 2e-2, "attn")
    assert fdl.get_status(ws) == 0


# ------------------------------------------- factor / budget selection

def _ranked_margin_ok(conf_row, masked, policy, f):
    cs = sorted((float(conf_row[i]) for i in masked), reverse=True)
    run = 0.0
    for n, c in enumerate(cs, start=1):
        e = 1.0 - c
        run += e
        v = (n + 1) * e - f if policy == fdl.SELECT_FACTOR else run + e - 1.0
        if abs(v) < 1e-4:
            return False
    return True


@pytest.mark.parametrize("policy,f", [(1, 1.0), (1, 0.5), (1, 2.5), (2, 0.0)])
def test_select_commit_factor_and_budget(policy, f):
    """Algorithm 3 / eq. 13 and eq. 9 against the oracle on random units
    (decisions kept 1e-4 away from their boundaries), including an exact
    confidence tie and units with nothing or one thing masked."""
    rng = np.random.default_rng(policy * 10 + int(f * 10))
    B, D, q_off, q_len, mask = 16, 32, 8, 16, 77
    conf = np.zeros((B, q_len), dtype=np.float32)
    bt = np.zeros((B, D), dtype=np.int32)
    for b in range(B):
        while True:
            row = rng.uniform(0.3, 1.0, q_len).astype(np.float32) ** rng.uniform(0.2, 3)
            row = row.astype(np.float32)
            if b == 0:
                row[1] = row[5]                      # exact tie
            masked = np.flatnonzero(rng.random(q_len) < rng.uniform(0, 1))
            if b == 1:
                masked = np.array([], dtype=int)
            if b == 2:
                masked = np.array([3])
            if _ranked_margin_ok(row, masked, policy, f):
                break
        conf[b] = row
        bt[b] = rng.integers(0, 70, D)
        bt[b, q_off + masked] = mask
    tok = rng.integers(100, 200, (B, q_len)).astype(np.int32)
    cfg = fdl.make_cfg(dict(batch=B, n_q_heads=1, n_kv_heads=1, head_dim=32,
                            block_size=D, q_off=q_off, q_len=q_len, cap_prefix=0,
                            hidden=8, vocab=1000, mask_id=mask, shift=0, tau=0.9, dtype="f32"))
    d_bt = torch.from_numpy(bt).cuda()
    comm = torch.empty((B, D), dtype=torch.uint8, device="cuda")
    n_c = torch.empty(B, dtype=torch.int32, device="cuda")
    n_l = torch.empty(B, dtype=torch.int32, device="cuda")
    fdl.select_commit(cfg, policy, f, torch.from_numpy(conf).cuda(), torch.from_numpy(tok).cuda(),
                      d_bt, comm, n_c, n_l)
    rule = step.RULE_FACTOR if policy == fdl.SELECT_FACTOR else step.RULE_BUDGET
    want = step.select_commit(bt, conf.astype(np.float64), tok, q_off, q_len, mask, rule, f)
    assert np.array_equal(d_bt.cpu().numpy(), want[0])
    assert np.array_equal(comm.cpu().numpy(), want[1])
    assert np.array_equal(n_c.cpu().numpy(), want[2])
    assert np.array_equal(n_l.cpu().numpy(), want[3])
    assert want[2][1] == 0 and want[2][2] == 1


# ------------------------------------------------ PrefixCache (queries = block + suffix)

@pytest.mark.parametrize("B,Hq,Hkv,n,lens", [
    (1, 32, 32, 288, [768]),          # LLaDA-like: block 32 + suffix 256 recomputed
    (2, 28, 4, 100, [0, 1500]),       # GQA 7, ragged: empty prefix, 100 rows (2 chunks)
    (3, 8, 8, 200, [64, 65, 300]),    # MHA, prefixes on and off the 64-key chunk grid
    (1, 32, 32, 768, [768]),          # LLaDA bench shape: 192 items, one CTA each
    (2, 8, 8, 256, [512, 512]),       # equal lengths, 32 items over the stream-K grid
    (4, 40, 40, 128, [300, 0, 64, 1000]),  # 160 ragged items, one CTA each: merges
])
def test_prefixcache_attn_against_oracle(B, Hq, Hkv, n, lens):
    """PrefixCache attention: the recomputed rows (several 64-key chunks and
    several 128-row query tiles) over [prefix | their own fresh K/V]."""
    d = 128
    cap = max(max(lens), 1)
    g = torch.Generator().manual_seed(B * 100 + n)
    rn = lambda *s: torch.randn(s, generator=g).to(torch.bfloat16)
    q, kp, vp, kn, vn = rn(B, n, Hq, d), rn(B, Hkv, cap, d), rn(B, Hkv, cap, d), \
        rn(B, Hkv, n, d), rn(B, Hkv, n, d)
    len_pre = torch.tensor(lens, dtype=torch.int32)
    cfg = fdl.make_cfg(dict(batch=B, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, block_size=n,
                            q_off=0, q_len=n, cap_prefix=cap, hidden=128, vocab=1000,
                            mask_id=999, shift=0, tau=0.9, dtype="bf16"))
    ws = fdl.workspace(cfg)
    out = torch.empty((B, n, Hq, d), dtype=torch.bfloat16, device="cuda")
    dv = [t.cuda() for t in (q, kp, vp, len_pre, kn, vn)]
    f64 = lambda t: t.double().numpy()
    ref = step.prefixcache_attention(f64(q), f64(kp), f64(vp), lens, f64(kn), f64(vn))
    for _ in range(2):                        # the second call reuses the workspace
        fdl.prefixcache_attn(cfg, *dv, out, ws)
        torch.cuda.synchronize()
        gh.assert_close_scaled(out.double().cpu().numpy(), ref, 2e-2, "prefixcache attn")
    assert fdl.get_status(ws) == 0


# ---------------------------------------- more LM-head rows than one pass holds

@pytest.mark.parametrize("V", [20000, 59200])
def test_lmhead_more_rows_than_one_pass(V):
    """batch * q_len = 600 rows: passes of 256, 256 and 88 rows over the
    weight (the first two in one launch of the CTA pairs), against the
    oracle (tokens where the top-2 gap exceeds 1e-3).  V = 20000: one full
    tile per CTA plus the folded short tile; V = 59200: three (an odd group
    count, so the second pass starts on the other TMEM buffer)."""
    B, q_len, H = 75, 8, 256
    g = torch.Generator().manual_seed(600 + V)
    rows = torch.randn((B * q_len, H), generator=g).to(torch.bfloat16)
    w = (torch.randn((V, H), generator=g) * (8.0 / H ** 0.5)).to(torch.bfloat16)
    active = (torch.rand(B * q_len, generator=g) < 0.8).to(torch.uint8)
    cfg = fdl.make_cfg(dict(batch=B, n_q_heads=1, n_kv_heads=1, head_dim=32, block_size=q_len,
                            q_off=0, q_len=q_len, cap_prefix=0, hidden=H, vocab=V,
                            mask_id=V - 1, shift=0, tau=0.9, dtype="bf16"))
    conf = torch.empty(B * q_len, dtype=torch.float32, device="cuda")
    tok = torch.empty(B * q_len, dtype=torch.int32, device="cuda")
    ws = fdl.workspace(cfg)
    fdl.lmhead_confidence(cfg, rows.cuda(), w.cuda(), active.cuda(), conf, tok, ws)
    torch.cuda.synchronize()
    t_ref, c_ref, gap = step.lmhead_confidence(rows.double().numpy(), w.float().numpy())
    act = active.numpy().astype(bool)
    t_gpu, c_gpu = tok.cpu().numpy(), conf.cpu().numpy().astype(np.float64)
    sure = (gap > 1e-3) & act
    assert np.array_equal(t_gpu[sure], t_ref[sure])
    np.testing.assert_allclose(c_gpu[act], c_ref[act], rtol=1e-3)
    assert (c_gpu[~act] == -1).all() and (t_gpu[~act] == -1).all()
    assert fdl.get_status(ws) == 0


LARGE_BATCH = dict(batch=40, n_q_heads=8, n_kv_heads=2, head_dim=128, block_size=32,
                   q_len=8, q_off=None, prefix=(100, 400), cap_prefix=400, suffix=0,
                   cap_suffix=0, hidden=256, vocab=5000, mask_id=4999, shift=1, tau=0.8,
                   w_scale=8.0, dtype="bf16", masked=(1, 8))


@pytest.mark.parametrize("vocab", [5000, 59200])
def test_fused_step_two_lm_passes_in_one_launch(vocab):
    """400 LM-head rows (passes of 256 and 144, both on CTA pairs, in one
    launch): the first pass commits its 32 sequences from the epilogue warps
    while the second pass streams, the second its 18 after the main loop;
    bit-exact commits against the oracle.  vocab 59200: three tiles per CTA
    and the folded short tile in each pass."""
    cfg = dict(LARGE_BATCH, batch=50, vocab=vocab, mask_id=vocab - 1)
    case, ref, _ = cases.parity_case("large_batch", 0, cfg=cfg)
    gh.compare_step(case, gh.run_denoise_step(case), ref)
    gh.compare_step(case, gh.run_denoise_step(case, packed=True), ref)


@pytest.mark.parametrize("shift", [1, 0])
def test_fused_step_with_two_lm_passes(shift):
    """A fused step with 320 LM-head rows (passes of 256 and 64 rows, each
    committing its own sequences) against the oracle, bit-exact commits,
    with and without the token-shift gather before the LM head."""
    case, ref, _ = cases.parity_case("large_batch", 0, cfg=dict(LARGE_BATCH, shift=shift))
    gh.compare_step(case, gh.run_denoise_step(case), ref)


# ----------------------------------------------- tiled LM-head weight layout

@pytest.mark.parametrize("V,H", [(5000, 448), (7001, 64), (1, 128)])
def test_pack_weight_matches_the_stated_layout(V, H):
    g = torch.Generator().manual_seed(V + H)
    w = torch.randn((V, H), generator=g).to(torch.bfloat16)
    cfg = fdl.make_cfg(dict(batch=1, n_q_heads=1, n_kv_heads=1, head_dim=32, block_size=1,
                            q_off=0, q_len=1, cap_prefix=0, hidden=H, vocab=V,
                            mask_id=0, shift=0, tau=0.9, dtype="bf16"))
    packed = torch.empty((V, H), dtype=torch.bfloat16, device="cuda")
    fdl.lmhead_pack_weight(cfg, w.cuda(), packed)
    torch.cuda.synchronize()
    want = pack_reference(w.view(torch.int16).numpy(), V, H)
    assert np.array_equal(packed.cpu().view(torch.int16).numpy(), want)


@pytest.mark.parametrize("R,V,H", [(32, 152064, 3584), (40, 5000, 448), (600, 20000, 256),
                                   (256, 7001, 64)])
@pytest.mark.parametrize("entry", ["lmhead", "noalloc"])
def test_packed_weight_gives_identical_results(R, V, H, entry):
    """The LM head over the tiled weight returns the very same bits as over
    the row-major one (same MMAs, same order), and matches the oracle."""
    if entry == "noalloc" and R > 128:
        pytest.skip("the allocation-free entry takes at most 128 rows")
    g = torch.Generator().manual_seed(R + V + H)
    rows = torch.randn((R, H), generator=g).to(torch.bfloat16)
    w = (torch.randn((V, H), generator=g) * (8.0 / H ** 0.5)).to(torch.bfloat16)
    cfg = fdl.make_cfg(dict(batch=R, n_q_heads=1, n_kv_heads=1, head_dim=32, block_size=1,
                            q_off=0, q_len=1, cap_prefix=0, hidden=H, vocab=V,
                            mask_id=V - 1, shift=0, tau=0.9, dtype="bf16"))
    w_d = w.cuda()
    w_p = torch.empty_like(w_d)
    fdl.lmhead_pack_weight(cfg, w_d, w_p)
    ws = fdl.workspace(cfg)
    got = {}
    for layout, wt in [(fdl.W_ROW_MAJOR, w_d), (fdl.W_PACKED, w_p)]:
        cfg.w_layout = layout
        conf = torch.empty(R, dtype=torch.float32, device="cuda")
        tok = torch.empty(R, dtype=torch.int32, device="cuda")
        if entry == "lmhead":
            fdl.lmhead_confidence(cfg, rows.cuda(), wt, None, conf, tok, ws)
        else:
            fdl.lmhead_confidence_noalloc(cfg, rows.cuda(), wt, None, conf, tok)
        torch.cuda.synchronize()
        got[layout] = (conf.cpu().numpy(), tok.cpu().numpy())
    assert np.array_equal(got[0][0].view(np.int32), got[1][0].view(np.int32))
    assert np.array_equal(got[0][1], got[1][1])
    t_ref, c_ref, gap = step.lmhead_confidence(rows.double().numpy(), w.float().numpy())
    sure = gap > 1e-3
    assert np.array_equal(got[1][1][sure], t_ref[sure])
    np.testing.assert_allclose(got[1][0].astype(np.float64), c_ref, rtol=1e-3)
    assert fdl.get_status(ws) == 0


@pytest.mark.parametrize("name,cfg", [("qwen7b", None), ("large_batch", LARGE_BATCH)])
def test_fused_step_over_the_packed_weight(name, cfg):
    """The fused step (LM head beside the attention, or in two passes) over
    the tiled weight: bit-exact commits against the oracle, as row-major."""
    case, ref, _ = cases.parity_case(name, 1, cfg=cfg) if cfg else cases.parity_case(name, 1)
    gh.compare_step(case, gh.run_denoise_step(case, packed=True), ref)


# ------------------------------------------------------ failure detection

def test_bounded_wait_times_out_into_the_status_word():
    """A wait that nothing satisfies runs out after its bound: the timeout
    bit lands in the workspace status word, the context stays usable, and
    the next step through the same workspace is correct."""
    cfg = fdl.make_cfg(synth.CONFIGS["tiny"] | dict(q_off=0))
    ws = fdl.workspace(cfg)
    fdl.check_wait_timeout(ws, limit_cycles=1_000_000)
    assert fdl.get_status(ws) == fdl.DEV_TIMEOUT
    assert fdl.get_status(ws) == 0                     # read and cleared
    case, ref, _ = cases.parity_case("tiny", 0)
    gh.compare_step(case, gh.run_denoise_step(case, ws=ws), ref)
