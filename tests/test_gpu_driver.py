"""GPU tests of the block decode loop: the block-cache append and the
sub-block WHILE loop (host-driven and as one CUDA graph), against the
oracle's commit rule iterated on the same confidences."""
import numpy as np
import pytest
import torch

from block_diffusion_decoding_causal_b200 import driver, fdl, synth
from oracle import cases, step

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _cfg(**kw):
    c = dict(batch=3, n_q_heads=2, n_kv_heads=2, head_dim=64, block_size=32, q_off=0,
             q_len=8, cap_prefix=0, cap_suffix=0, hidden=64, vocab=1000, mask_id=999,
             shift=0, tau=0.8, dtype="bf16")
    c.update(kw)
    return c


def test_append_block_extends_the_prefix_cache_on_device():
    c = _cfg(batch=3, n_kv_heads=2, head_dim=64, block_size=8, cap_prefix=40)
    cfg = fdl.make_cfg(c)
    g = torch.Generator().manual_seed(0)
    kp = torch.randn((3, 2, 40, 64), generator=g).to(torch.bfloat16)
    vp = torch.randn((3, 2, 40, 64), generator=g).to(torch.bfloat16)
    kb = torch.randn((3, 2, 8, 64), generator=g).to(torch.bfloat16)
    vb = torch.randn((3, 2, 8, 64), generator=g).to(torch.bfloat16)
    lens = torch.tensor([0, 10, 35], dtype=torch.int32)       # the last one overflows
    d = [t.cuda() for t in (kp, vp, kb, vb, lens)]
    ws = fdl.workspace(cfg)
    fdl.append_block(cfg, d[2], d[3], d[0], d[1], d[4], ws)
    torch.cuda.synchronize()
    kp2, vp2, lens2 = d[0].cpu(), d[1].cpu(), d[4].cpu()
    assert lens2.tolist() == [8, 18, 35]
    for b, L0 in [(0, 0), (1, 10)]:
        assert torch.equal(kp2[b, :, L0:L0 + 8], kb[b]) and torch.equal(vp2[b, :, L0:L0 + 8], vb[b])
        assert torch.equal(kp2[b, :, :L0], kp[b, :, :L0])
        assert torch.equal(kp2[b, :, L0 + 8:], kp[b, :, L0 + 8:])
    assert torch.equal(kp2[2], kp[2]) and torch.equal(vp2[2], vp[2])
    assert fdl.get_status(ws) & fdl.DEV_BAD_PREFIX_LEN


def _oracle_unit_loop(bt, conf, tok, q_off, q_len, mask_id, tau):
    """Iterate Algorithm 2 on fixed confidences until the unit is decoded;
    returns the final tokens and the number of steps."""
    n = 0
    while (bt[:, q_off:q_off + q_len] == mask_id).any() and n < q_len:
        bt = step.threshold_commit(bt, conf, tok, q_off, q_len, mask_id, tau)[0]
        n += 1
    return bt, n


def _commit_loop_setup(seed):
    rng = np.random.default_rng(seed)
    c = _cfg(batch=3, block_size=32, q_len=8, tau=0.8)
    B, D, q_len, mask = 3, 32, 8, 999
    units = D // q_len
    conf = []
    for u in range(units):
        # distinct confidences, at least 0.01 apart, some above tau
        base = rng.permutation(np.arange(30, 100)).astype(np.float32)[: B * q_len] / 100.0
        conf.append(base.reshape(B, q_len).astype(np.float32))
    tok = [rng.integers(0, 900, (B, q_len)).astype(np.int32) for _ in range(units)]
    bt = np.full((B, D), mask, dtype=np.int32)
    return c, conf, tok, bt


@pytest.mark.parametrize("use_graph", [False, True])
def test_block_loop_commits_every_position(use_graph):
    c, conf, tok, bt0 = _commit_loop_setup(7)
    B, D, q_len, mask, tau = 3, 32, 8, 999, 0.8
    units = D // q_len
    cfgs = [fdl.make_cfg(dict(c, q_off=u * q_len)) for u in range(units)]
    d_conf = [torch.from_numpy(x).cuda() for x in conf]
    d_tok = [torch.from_numpy(x).cuda() for x in tok]
    d_bt = torch.from_numpy(bt0.copy()).cuda()
    comm = torch.empty((B, D), dtype=torch.uint8, device="cuda")
    n_c = torch.empty(B, dtype=torch.int32, device="cuda")
    n_l = torch.empty(B, dtype=torch.int32, device="cuda")
    any_m = torch.zeros(1, dtype=torch.int32, device="cuda")
    steps = torch.zeros(units, dtype=torch.int32, device="cuda")

    def one_step(u, s):
        fdl.threshold_commit(cfgs[u], d_conf[u], d_tok[u], d_bt, comm, n_c, n_l, stream=s)

    if use_graph:
        g = driver.BlockGraph(cfgs, one_step, n_l, steps)
        g.launch()
        torch.cuda.synchronize()
        got_steps = steps.cpu().tolist()
    else:
        got_steps = []
        driver.run_host_loop(cfgs, one_step, n_l, any_m, got_steps)
    want = bt0.copy()
    want_steps = []
    for u in range(units):
        want, n = _oracle_unit_loop(want, conf[u].astype(np.float64), tok[u], u * q_len, q_len,
                                    mask, float(np.float32(tau)))
        want_steps.append(n)
    assert np.array_equal(d_bt.cpu().numpy(), want)
    assert got_steps == want_steps
    assert not (want == mask).any()


def test_block_graph_with_fused_step_and_append():
    """A whole block of a small bf16 model shape decoded by one graph launch:
    per sub-block a WHILE loop of fdl_denoise_step, then the block append;
    every committed token equals the oracle's iterated step."""
    c = dict(synth.CONFIGS["qwen1.5b"], vocab=3000, mask_id=2999, hidden=256, n_q_heads=4,
             n_kv_heads=2, head_dim=64, prefix=(100, 100), cap_prefix=160, block_size=16,
             q_len=4, q_off=0, masked=(4, 4), shift=0)
    units = c["block_size"] // c["q_len"]
    ok_case = None
    for seed in range(40):
        case = synth.make_case("loop", seed, cfg=dict(c))
        res = cases.run_oracle(case)
        confs = res["conf"][0]
        srt = np.sort(confs)[::-1]
        if (res["logit_gap"].min() > 0.05 and np.abs(confs - res["tau"]).min() > 5e-3
                and (res["tok"] != c["mask_id"]).all()
                and (np.diff(srt) < -2e-3 * srt[:-1]).all()):
            ok_case = case
            break
    assert ok_case is not None
    case = ok_case
    cfgs = [fdl.make_cfg(dict(case.cfg, q_off=u * c["q_len"])) for u in range(units)]
    dcase = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in vars(case).items()}
    B, D = case.cfg["batch"], case.cfg["block_size"]
    bt = torch.full((B, D), case.cfg["mask_id"], dtype=torch.int32, device="cuda")
    o = dict(attn=torch.empty_like(dcase["q"]),
             conf=torch.empty((B, c["q_len"]), dtype=torch.float32, device="cuda"),
             tok=torch.empty((B, c["q_len"]), dtype=torch.int32, device="cuda"),
             comm=torch.empty((B, D), dtype=torch.uint8, device="cuda"),
             n_c=torch.empty(B, dtype=torch.int32, device="cuda"),
             n_l=torch.empty(B, dtype=torch.int32, device="cuda"))
    steps = torch.zeros(units, dtype=torch.int32, device="cuda")
    ws = fdl.workspace(cfgs[0])
    len0 = int(case.len_pre[0])

    def one_step(u, s):
        fdl.denoise_step(cfgs[u], dcase["q"], dcase["k_pre"], dcase["v_pre"], dcase["len_pre"],
                         dcase["k_blk"], dcase["v_blk"], None, None, None, dcase["hidden"], None,
                         dcase["w_lm"], bt, o["attn"], o["conf"], o["tok"], o["comm"], o["n_c"],
                         o["n_l"], ws, stream=s)

    def append(s):
        fdl.append_block(cfgs[0], dcase["k_blk"], dcase["v_blk"], dcase["k_pre"], dcase["v_pre"],
                         dcase["len_pre"], ws, stream=s)

    g = driver.BlockGraph(cfgs, one_step, o["n_l"], steps, append=append)
    g.launch()
    torch.cuda.synchronize()
    # the oracle: the same step inputs every iteration, so the same conf/tok
    # per sub-block; iterate the commit rule.
    want = np.full((B, D), case.cfg["mask_id"], dtype=np.int64)
    want_steps = []
    for u in range(units):
        want, n = _oracle_unit_loop(want, res["conf"], res["tok"], u * c["q_len"], c["q_len"],
                                    case.cfg["mask_id"], res["tau"])
        want_steps.append(n)
    assert np.array_equal(bt.cpu().numpy(), want)
    assert steps.cpu().tolist() == want_steps
    assert int(dcase["len_pre"][0]) == len0 + D
    assert torch.equal(dcase["k_pre"][0, :, len0:len0 + D].cpu(), case.k_blk[0])
    assert fdl.get_status(ws) == 0


def test_block_graph_on_the_tensor_core_step_matches_the_host_loop():
    """The bf16 / head-dim-128 fused step (LM head first, attention beside it
    through programmatic launches, token-shift gather before them) captured
    in the WHILE-node graph: same tokens, step counts and appended cache as
    the host-driven loop."""
    c = dict(synth.CONFIGS["qwen7b"], batch=2, prefix=(300, 500), cap_prefix=600, q_off=0,
             vocab=8000, mask_id=7999, hidden=512, masked=(8, 8), tau=0.9)
    for seed in range(20):          # a case whose argmax is never the mask token
        case = synth.make_case("graph_tc", seed, cfg=dict(c))
        if (cases.run_oracle(case)["tok"] != c["mask_id"]).all():
            break
    B, D, q_len = c["batch"], c["block_size"], c["q_len"]
    units = D // q_len
    cfgs = [fdl.make_cfg(dict(case.cfg, q_off=u * q_len)) for u in range(units)]
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in vars(case).items()}

    def run(use_graph):
        kp, vp, lens = d["k_pre"].clone(), d["v_pre"].clone(), d["len_pre"].clone()
        bt = torch.full((B, D), c["mask_id"], dtype=torch.int32, device="cuda")
        o = dict(attn=torch.empty_like(d["q"]),
                 conf=torch.empty((B, q_len), dtype=torch.float32, device="cuda"),
                 tok=torch.empty((B, q_len), dtype=torch.int32, device="cuda"),
                 comm=torch.empty((B, D), dtype=torch.uint8, device="cuda"),
                 n_c=torch.empty(B, dtype=torch.int32, device="cuda"),
                 n_l=torch.empty(B, dtype=torch.int32, device="cuda"))
        steps = torch.zeros(units, dtype=torch.int32, device="cuda")
        ws = fdl.workspace(cfgs[0])

        def one_step(u, s):
            fdl.denoise_step(cfgs[u], d["q"], kp, vp, lens, d["k_blk"], d["v_blk"], None, None,
                             None, d["hidden"], d["h_prev"], d["w_lm"], bt, o["attn"], o["conf"],
                             o["tok"], o["comm"], o["n_c"], o["n_l"], ws, stream=s)

        def append(s):
            fdl.append_block(cfgs[0], d["k_blk"], d["v_blk"], kp, vp, lens, ws, stream=s)

        if use_graph:
            g = driver.BlockGraph(cfgs, one_step, o["n_l"], steps, append=append)
            g.launch()
            torch.cuda.synchronize()
            n = steps.cpu().tolist()
        else:
            n = []
            driver.run_host_loop(cfgs, one_step, o["n_l"],
                                 torch.zeros(1, dtype=torch.int32, device="cuda"), n)
            append(torch.cuda.current_stream())
            torch.cuda.synchronize()
        assert fdl.get_status(ws) == 0
        return bt.cpu(), n, lens.cpu(), kp.cpu()

    bt_h, n_h, len_h, kp_h = run(False)
    bt_g, n_g, len_g, kp_g = run(True)
    assert not (bt_h == c["mask_id"]).any()
    assert torch.equal(bt_g, bt_h) and n_g == n_h
    assert torch.equal(len_g, len_h) and torch.equal(len_h, case.len_pre + D)
    assert torch.equal(kp_g, kp_h)
