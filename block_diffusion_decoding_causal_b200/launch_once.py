"""Run one entry point a few times on a benchmark-shaped workload.

A profiling harness: hardware-counter tools capture one launch of one kernel,
so this runs ``--kernel`` (lmhead, attn, dualcache or step) ``--launches``
times on synthetic inputs drawn on the device, synchronises and exits.

    python -m block_diffusion_decoding_causal_b200.launch_once --kernel lmhead
"""
from __future__ import annotations

import argparse

import torch

from block_diffusion_decoding_causal_b200 import fdl, synth


def main() -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--kernel", default="lmhead",
                    choices=["lmhead", "attn", "dualcache", "step", "prefixcache"])
    ap.add_argument("--rows", type=int, default=768,
                    help="prefixcache: recomputed rows (block + suffix)")
    ap.add_argument("--workload", default="qwen7b")
    ap.add_argument("--batch", type=int, default=None)
    ap.add_argument("--prefix", type=int, default=None)
    ap.add_argument("--launches", type=int, default=3)
    ap.add_argument("--packed", action="store_true",
                    help="lmhead / step: the LM-head weight in the tiled layout")
    args = ap.parse_args()

    c = dict(synth.CONFIGS[args.workload])
    if args.batch is not None:
        c["batch"] = args.batch
    if args.prefix is not None:
        c.update(prefix=(args.prefix, args.prefix), cap_prefix=args.prefix)
    c["q_off"] = c["q_off"] or 0
    if args.kernel == "prefixcache":
        # the recomputed rows take the block's place: queries = keys = rows
        c.update(block_size=args.rows, q_len=args.rows, q_off=0, cap_suffix=0, suffix=0)
    B, q_len, H, V = c["batch"], c["q_len"], c["hidden"], c["vocab"]
    Hq, Hkv, d, D = c["n_q_heads"], c["n_kv_heads"], c["head_dim"], c["block_size"]
    dt = synth.torch_dtype(c["dtype"])
    g = torch.Generator(device="cuda").manual_seed(1)
    rn = lambda *s: torch.randn(s, generator=g, device="cuda").to(dt)
    cfg = fdl.make_cfg(c)
    ws = fdl.workspace(cfg)
    conf = torch.empty((B, q_len), dtype=torch.float32, device="cuda")
    tok = torch.empty((B, q_len), dtype=torch.int32, device="cuda")
    cap_p, cap_s = c["cap_prefix"], c.get("cap_suffix", 0)
    lo, hi = c["prefix"]
    len_pre = torch.randint(lo, hi + 1, (B,), generator=g, device="cuda", dtype=torch.int32)
    q = rn(B, q_len, Hq, d)
    out = torch.empty_like(q)
    if args.kernel in ("attn", "dualcache", "step", "prefixcache"):
        kp, vp = rn(B, Hkv, cap_p, d), rn(B, Hkv, cap_p, d)
        kb, vb = rn(B, Hkv, D, d), rn(B, Hkv, D, d)
        if cap_s:
            ks, vs = rn(B, Hkv, cap_s, d), rn(B, Hkv, cap_s, d)
            len_suf = torch.full((B,), c["suffix"], dtype=torch.int32, device="cuda")
    if args.kernel in ("lmhead", "step"):
        w = (torch.randn((V, H), generator=g, device="cuda") * (c["w_scale"] / H ** 0.5)).to(dt)
        rows = rn(B * q_len, H)
        if args.packed:
            w_rm, w = w, torch.empty_like(w)
            fdl.lmhead_pack_weight(cfg, w_rm, w)
            del w_rm
            cfg.w_layout = fdl.W_PACKED
    for _ in range(args.launches):
        if args.kernel == "lmhead":
            fdl.lmhead_confidence(cfg, rows, w, None, conf, tok, ws)
        elif args.kernel == "prefixcache":
            fdl.prefixcache_attn(cfg, q, kp, vp, len_pre, kb, vb, out, ws)
        elif args.kernel == "attn":
            fdl.block_attn(cfg, q, kp, vp, len_pre, kb, vb, out, ws)
        elif args.kernel == "dualcache":
            fdl.dualcache_attn(cfg, q, kp, vp, len_pre, kb, vb, ks, vs, len_suf, out, ws)
        else:
            bt = torch.full((B, D), c["mask_id"], dtype=torch.int32, device="cuda")
            comm = torch.empty((B, D), dtype=torch.uint8, device="cuda")
            n_c = torch.empty(B, dtype=torch.int32, device="cuda")
            n_l = torch.empty(B, dtype=torch.int32, device="cuda")
            h_prev = rn(B, H) if c["shift"] else None
            fdl.denoise_step(cfg, q, kp, vp, len_pre, kb, vb, None, None, None,
                             rows.view(B, q_len, H), h_prev, w, bt, out, conf, tok, comm,
                             n_c, n_l, ws)
    torch.cuda.synchronize()
    status = fdl.get_status(ws)
    print(f"{args.kernel}: {args.launches} launches, status {status}")
    return 0 if status == 0 else 1


if __name__ == "__main__":
    raise SystemExit(main())
