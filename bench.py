"""Benchmark: one denoising step of the active block on B200.

Workload: Qwen2.5-7B shapes in bf16 (batch 4, 28 query / 4 KV heads, head dim
128, hidden 3584, vocab 152064, per-sequence prefix lengths U[1024, 2048],
block 32 with the sub-block of 8 active, tau 0.9), synthetic seeded inputs.

``python bench.py --gpus N --steps K --warmup W`` prints one JSON line.  A
step is one fdl_denoise_step (attention -> token-shift gather -> fused LM
head / confidence / commit).  With N > 1 (torchrun) every rank runs its own
batch of 4 sequences (weak scaling, no collective on the data path); the time
is the max over ranks.  ``--impl reference`` times the CPU oracle instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORKLOAD = "qwen7b"
METRIC = "denoise-step latency (us) & positions/s at Qwen2.5-7B shapes; % HBM roofline"
UNIT = "positions/s"


def roofline_seconds(bytes_moved: float, flops: float, hbm_bps: float,
                     flops_per_s: float) -> float:
    """Lower bound on a kernel's time: the slower of moving its bytes at the
    memory bandwidth and doing its FLOPs at the arithmetic peak."""
    return max(bytes_moved / hbm_bps, flops / flops_per_s)


def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=float(p["hbm_gbs"]), bf16_tflops=float(p["bf16_tflops"]),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, source="fallback")


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during a region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax = float(parts[2])
                except ValueError:
                    continue
                for name, val in zip(names, parts[5:9]):
                    if val.lower().startswith("active"):
                        reasons.add(name)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------- CPU oracle

def host_cores() -> int:
    """Host threads this process may run on (the oracle uses one per core)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_baseline(case, min_seconds: float = 10.0, max_steps: int = 50) -> dict:
    """Time the CPU oracle (the plain fp64 C++ program, as it stands) on this
    workload: whole steps on every host core, repeated until ``min_seconds``
    have passed, then one whole step on a single thread."""
    from oracle import cases
    threads = host_cores()
    n, t0 = 0, time.perf_counter()
    while True:
        cases.run_oracle(case, threads=threads)
        n += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or n >= max_steps:
            break
    c = case.cfg
    per_step = c["batch"] * c["q_len"]
    t1 = time.perf_counter()
    cases.run_oracle(case, threads=1)
    el1 = time.perf_counter() - t1
    return {"value": n * per_step / el, "unit": UNIT, "cores": int(threads),
            "kind": "oracle",
            "sample": f"{n} whole oracle step(s) of the benchmark workload "
                      f"({c['batch']} x {c['q_len']} positions each), {el:.1f} s, "
                      f"plain fp64 C++ (no BLAS) on {threads} threads",
            "seconds": el, "steps": n,
            "single_thread": {"value": per_step / el1, "unit": UNIT, "seconds": el1,
                              "sample": "one whole oracle step on one thread"}}


# ------------------------------------------------------------ timing helpers

def rounds_us(timed, fn, k: int, reps: int, world: int) -> list:
    """Per-launch microseconds of ``reps`` timed regions of ``k`` launches
    each (every region the max over ranks)."""
    return [max_over_ranks(timed(fn, k), world) / k * 1e6 for _ in range(reps)]


def graph_rounds_us(torch, stream, fn, k: int, reps: int, world: int) -> list:
    """Per-launch microseconds of ``reps`` replays of one CUDA graph that holds
    ``k`` launches of ``fn`` (captured on ``stream``): the device time of
    back-to-back launches without the host's per-call work between them, as
    a serving loop that captures its step sees it."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(k):
            fn(i)
    out = []
    with torch.cuda.stream(stream):
        g.replay()
        stream.synchronize()
        for _ in range(reps):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            g.replay()
            e1.record(stream)
            stream.synchronize()
            out.append(max_over_ranks(e0.elapsed_time(e1) * 1e3 / k, world))
    del g
    return out


def spread(us: list) -> dict:
    """Median and range of repeated timings."""
    return {"median": statistics.median(us), "min": min(us), "max": max(us),
            "rounds": len(us)}


def kv_copies_for(torch, bytes_per_copy: int, lo: int = 2, hi: int = 64) -> int:
    """How many copies of a KV input to rotate over so that the bytes read in
    one pass over all copies exceed twice the L2 (the reads then come from
    HBM)."""
    l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
    need = -(-2 * l2 // max(1, bytes_per_copy))
    return int(min(hi, max(lo, need)))


# ------------------------------------------------------------------- main

def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=1002)
    ap.add_argument("--kv-copies", type=int, default=16)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the sweep, the other workloads and the block-decode grid")
    return ap.parse_args()


def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch
        import torch.distributed as dist
        dist.barrier(device_ids=[torch.cuda.current_device()])


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """The slowest rank's time: every rank's number, max-reduced."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(seed: int, rank: int) -> int:
    """Each rank decodes its own batch of sequences (weak scaling)."""
    return seed + 7919 * rank


def run_reference(args):
    """Reference arm: the CPU oracle, timed on the host cores."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from block_diffusion_decoding_causal_b200 import synth
    from oracle import cases
    case = synth.make_case(WORKLOAD, args.seed)
    c = case.cfg
    threads = host_cores()
    for _ in range(args.warmup):
        cases.run_oracle(case, threads=threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        cases.run_oracle(case, threads=threads)
    el = time.perf_counter() - t0
    pos = args.steps * c["batch"] * c["q_len"]
    value = pos / el
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _config(c, args),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": int(threads),
                         "kind": "oracle",
                         "sample": f"{args.steps} whole oracle steps of the workload, "
                                   f"plain fp64 C++ (no BLAS) on {threads} threads"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _config(c, args):
    return {"workload": "Qwen2.5-7B-shape denoise step (bf16, batch 4, 28/4 heads, "
                        "d 128, H 3584, V 152064, prefix U[1024,2048], block 32, "
                        "sub-block 8, tau 0.9)",
            "batch": c["batch"], "q_len": c["q_len"], "block_size": c["block_size"],
            "n_q_heads": c["n_q_heads"], "n_kv_heads": c["n_kv_heads"],
            "head_dim": c["head_dim"], "hidden": c["hidden"], "vocab": c["vocab"],
            "prefix": list(c["prefix"]), "tau": c["tau"], "seed": args.seed,
            "parallelism": f"replicas x{int(os.environ.get('WORLD_SIZE', '1'))}",
            "lm_weight_layout": "tiled (fdl_lmhead_pack_weight, once before timing)",
            "l2": "inputs larger than L2: the 1.09 GB LM-head weight streams every "
                  f"step; KV caches rotate over {args.kv_copies} copies"}


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)

    import torch
    from block_diffusion_decoding_causal_b200 import fdl, synth

    world, rank, local = dist_setup()
    peaks = measured_peaks()
    case = synth.make_case(WORKLOAD, rank_seed(args.seed, rank))
    c = case.cfg
    # The LM-head weight is rewritten once, at load time, into the tiled
    # layout the LM head streams fastest (bit-identical results).
    c_run = dict(c, w_layout=fdl.W_PACKED)
    cfg = fdl.make_cfg(c_run)
    B, q_len, H, V = c["batch"], c["q_len"], c["hidden"], c["vocab"]
    stream = torch.cuda.Stream()
    dev = lambda t: None if t is None else t.cuda().contiguous()
    n_copies = max(1, args.kv_copies)
    with torch.cuda.stream(stream):
        w_row_major = dev(case.w_lm)
        w = torch.empty_like(w_row_major)
        fdl.lmhead_pack_weight(cfg, w_row_major, w, stream)
        del w_row_major
        sets = []
        for i in range(n_copies):
            sets.append(dict(q=dev(case.q), k_pre=dev(case.k_pre), v_pre=dev(case.v_pre),
                             len_pre=dev(case.len_pre), k_blk=dev(case.k_blk),
                             v_blk=dev(case.v_blk), hidden=dev(case.hidden),
                             h_prev=dev(case.h_prev), bt=dev(case.block_tokens)))
        # Per-step inputs of each set live in one device buffer (views), so a
        # step's upload is one copy; likewise the step's outputs.
        for x in sets:
            x["_buf"], views = _pack(torch, {k: x[k] for k in STEP_INPUTS
                                             if x[k] is not None}, "cuda")
            x.update(views)
        out_buf, out = _pack(torch, dict(
            conf=torch.empty((B, q_len), dtype=torch.float32),
            tok=torch.empty((B, q_len), dtype=torch.int32),
            committed=torch.empty((B, c["block_size"]), dtype=torch.uint8),
            n_c=torch.empty(B, dtype=torch.int32),
            n_l=torch.empty(B, dtype=torch.int32)), "cuda")
        out["attn"] = torch.empty_like(sets[0]["q"])
        ws = fdl.workspace(cfg)
    stream.synchronize()

    def step(s):
        fdl.denoise_step(cfg, s["q"], s["k_pre"], s["v_pre"], s["len_pre"], s["k_blk"],
                         s["v_blk"], None, None, None, s["hidden"], s["h_prev"], w,
                         s["bt"], out["attn"], out["conf"], out["tok"], out["committed"],
                         out["n_c"], out["n_l"], ws, stream)

    def timed(fn, k):
        ev0 = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        ev0.record(stream)
        for i in range(k):
            fn(i)
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        return ev0.elapsed_time(ev1) / 1e3

    for i in range(args.warmup):
        step(sets[i % n_copies])
    torch.cuda.synchronize()
    assert fdl.get_status(ws, stream) == 0

    with ClockSampler(_gpu_id(torch)) as clocks:
        t_step = timed(lambda i: step(sets[i % n_copies]), args.steps)
        t_step = max_over_ranks(t_step, world)
        # two more rounds of the same K steps, for the spread
        step_rounds = [t_step / args.steps * 1e6] + rounds_us(
            timed, lambda i: step(sets[i % n_copies]), args.steps, 2, world)
    ms_per_step = t_step / args.steps * 1e3
    pos = world * B * q_len * args.steps
    value = pos / t_step
    # The same K steps replayed from one CUDA graph (as a serving loop that
    # captures its step runs them): reported beside the headline, which
    # stays the back-to-back direct calls.
    step_graph = graph_rounds_us(torch, stream, lambda i: step(sets[i % n_copies]),
                                 args.steps, 3, world)

    # Dominant kernel: the fused LM head (weight stream), timed alone on the
    # same stream over K launches.
    rows = sets[0]["hidden"].view(B * q_len, H)
    lm = lambda i: fdl.lmhead_confidence(cfg, rows, w, None, out["conf"], out["tok"],
                                         ws, stream)
    for i in range(3):
        lm(i)
    lm_rounds = rounds_us(timed, lm, args.steps, 3, world)
    t_lm = statistics.median(lm_rounds) * 1e-6
    attn = lambda i: fdl.block_attn(cfg, sets[i % n_copies]["q"], sets[i % n_copies]["k_pre"],
                                    sets[i % n_copies]["v_pre"], sets[i % n_copies]["len_pre"],
                                    sets[i % n_copies]["k_blk"], sets[i % n_copies]["v_blk"],
                                    out["attn"], ws, stream)
    for i in range(3):
        attn(i)
    attn_rounds = rounds_us(timed, attn, args.steps, 3, world)
    t_attn = statistics.median(attn_rounds) * 1e-6
    attn_graph = graph_rounds_us(torch, stream, attn, args.steps, 3, world)
    pc = prefixcache_leg(torch, fdl, stream, timed, world, args.steps, peaks)
    try:
        blk = block_decode_leg(torch, fdl, c_run, sets[0], w, stream, world)
    except Exception as e:  # reported in the JSON line; the headline legs stand
        blk = {"error": f"{type(e).__name__}: {e}"}
    # Every rank takes part in these reductions, whatever its leg did.
    for k in ("graph_us_per_block", "host_loop_us_per_block", "graph_us_per_step"):
        blk[k] = max_over_ranks(float(blk.get(k, float("nan"))), world)
    if "graph_us_per_block" in blk and blk["graph_us_per_block"] == blk["graph_us_per_block"]:
        blk["positions_per_s_graph"] = c["batch"] * c["block_size"] / (
            blk["graph_us_per_block"] * 1e-6)
    lm_big = large_batch_lm_leg(torch, fdl, synth, stream, timed, world, args.steps, peaks)
    sweep = others = grid = None
    if not args.no_sweep:
        sweep = sweep_leg(torch, fdl, synth, stream, timed, world, args.steps, peaks, w,
                          rank_seed(args.seed, rank))
        others = configs_leg(torch, fdl, synth, stream, timed, world, args.steps, peaks,
                             rank_seed(args.seed, rank))
        grid = block_decode_grid(torch, fdl, c_run, sets[0], w, stream, world)

    # End to end through the public API: per step, pinned host inputs copied
    # in, the step, and its results copied out and read on the host.
    host_in = sets[0]["_buf"].cpu().pin_memory()       # one packed upload per step
    n_sets = n_copies
    e2e_out = [_pack(torch, dict(
        conf=torch.empty((B, q_len), dtype=torch.float32),
        tok=torch.empty((B, q_len), dtype=torch.int32),
        committed=torch.empty((B, c["block_size"]), dtype=torch.uint8),
        n_c=torch.empty(B, dtype=torch.int32),
        n_l=torch.empty(B, dtype=torch.int32)), "cuda") for _ in range(n_sets)]
    host_outs = [torch.empty_like(ob, device="cpu").pin_memory() for ob, _ in e2e_out]
    host_bts = [torch.empty_like(sets[0]["bt"], device="cpu").pin_memory()
                for _ in range(n_sets)]
    host_n_l_np = [_views(torch, h, e2e_out[0][0], e2e_out[0][1])["n_l"].numpy()
                   for h in host_outs]
    h2d = host_in.numel()
    d2h = host_outs[0].numel() + host_bts[0].numel() * host_bts[0].element_size()

    # As a serving loop runs it.  Each input set has its own device inputs
    # and outputs and pinned host outputs.  The step is replayed from one CUDA
    # graph per set (captured from the same fdl_denoise_step call).  Step
    # i+1's inputs cross PCIe on a copy stream while step i runs (a set is
    # refilled only after its previous step and result copy finished), and
    # step i's results go back to the host on a third stream while step i+1
    # computes.  Every step uploads its inputs and the host reads every
    # step's result.  Pipelined (the headline): the host reads step i-1's
    # result while step i runs.  Serial (reported beside it): the host reads
    # step i's result before step i+1 is launched.
    copy_stream = torch.cuda.Stream()
    d2h_stream = torch.cuda.Stream()
    copied = [torch.cuda.Event() for _ in range(n_sets)]
    computed = [torch.cuda.Event() for _ in range(n_sets)]
    done = [torch.cuda.Event() for _ in range(n_sets)]

    def step_into(x, o):
        fdl.denoise_step(cfg, x["q"], x["k_pre"], x["v_pre"], x["len_pre"], x["k_blk"],
                         x["v_blk"], None, None, None, x["hidden"], x["h_prev"], w,
                         x["bt"], None, o["conf"], o["tok"], o["committed"],
                         o["n_c"], o["n_l"], ws, stream)

    graphs = []
    for j in range(n_sets):
        gph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gph, stream=stream):
            step_into(sets[j], e2e_out[j][1])
        graphs.append(gph)
    stream.synchronize()

    def upload(i):
        j = i % n_sets
        copy_stream.wait_event(done[j])
        with torch.cuda.stream(copy_stream):
            sets[j]["_buf"].copy_(host_in, non_blocking=True)
        copied[j].record(copy_stream)

    def e2e_run(k, start, pipelined):
        for j in range(n_sets):
            done[j].record(stream)
        copy_stream.wait_event(start)        # the first upload is inside the timing
        upload(0)
        seen = 0
        for i in range(k):
            j = i % n_sets
            stream.wait_event(copied[j])
            with torch.cuda.stream(stream):
                graphs[j].replay()           # the step
            computed[j].record(stream)
            d2h_stream.wait_event(computed[j])
            with torch.cuda.stream(d2h_stream):  # its results to the host
                host_outs[j].copy_(e2e_out[j][0], non_blocking=True)
                host_bts[j].copy_(sets[j]["bt"], non_blocking=True)
            done[j].record(d2h_stream)
            if i + 1 < k and n_sets > 1:
                upload(i + 1)                # crosses PCIe while step i runs
            if pipelined:
                if i >= 1:
                    jp = (i - 1) % n_sets
                    done[jp].synchronize()   # step i-1's results are on the host
                    seen += int(host_n_l_np[jp].sum())
            else:
                done[j].synchronize()
                seen += int(host_n_l_np[j].sum())   # the host reads the result
                if n_sets == 1 and i + 1 < k:
                    upload(i + 1)
        jl = (k - 1) % n_sets
        if pipelined:
            done[jl].synchronize()
            seen += int(host_n_l_np[jl].sum())
        stream.wait_event(done[jl])          # the timing ends after the last read-back
        return seen

    def timed_e2e(k, pipelined):
        ev0 = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        ev0.record(stream)
        e2e_run(k, ev0, pipelined)
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        return ev0.elapsed_time(ev1) / 1e3
    timed_e2e(3, True)                        # warm-up
    t_e2e = max_over_ranks(timed_e2e(args.steps, True), world)
    t_e2e_serial = max_over_ranks(timed_e2e(args.steps, False), world)
    e2e_value = pos / t_e2e
    assert fdl.get_status(ws, stream) == 0
    del graphs

    # Tokens committed by one step from the workload's initial block state.
    with torch.cuda.stream(stream):
        sets[0]["bt"].copy_(case.block_tokens)
    step(sets[0])
    torch.cuda.synchronize()
    committed = float(out["n_c"].float().sum().item())
    clk = clocks.summary()
    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return 0

    lm_bytes = V * H * 2 + B * q_len * H * 2 + B * q_len * 8
    lm_gbs = lm_bytes / t_lm / 1e9
    # Algorithmic bytes of the attention (K and V of every visible key, Q in,
    # O out) and of the whole step (attention + LM head + the token shift).
    d, Hq, Hkv, D = c["head_dim"], c["n_q_heads"], c["n_kv_heads"], c["block_size"]
    keys = int(case.len_pre.sum()) + B * D
    attn_bytes = keys * Hkv * 2 * d * 2 + 2 * B * q_len * Hq * d * 2
    step_bytes = attn_bytes + lm_bytes + (B * q_len * H * 2 * 2 if c["shift"] else 0)
    traffic = _profiled_traffic("lmhead", "lmhead_tc_qwen7b.md")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "step_latency_us": ms_per_step * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) Q/K/V/hidden, W_lm ~ N(0,1/H) x 8)",
        "config": _config(c, args),
        "roofline": {"bound": "hbm", "kernel": "fused LM head + confidence",
                     "achieved": lm_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": lm_gbs / peaks["hbm_gbs"],
                     "peak_source": f"{peaks['source']} hbm_gbs (burst copy)",
                     "traffic": traffic, "bytes_per_launch": lm_bytes,
                     "us_per_launch": t_lm * 1e6, "us_rounds": spread(lm_rounds)},
        "step_us_rounds": spread(step_rounds),
        "attention": {"us_per_launch": t_attn * 1e6, "bytes_per_launch": attn_bytes,
                      "achieved_gbs": attn_bytes / t_attn / 1e9,
                      "frac_hbm": attn_bytes / t_attn / 1e9 / peaks["hbm_gbs"],
                      "us_rounds": spread(attn_rounds),
                      "graph": {"us": spread(attn_graph),
                                "frac_hbm": attn_bytes / statistics.median(attn_graph) / 1e3
                                / peaks["hbm_gbs"]}},
        "step_roofline": {"bytes": step_bytes, "achieved_gbs": step_bytes / (t_step / args.steps) / 1e9,
                          "frac": step_bytes / (t_step / args.steps) / 1e9 / peaks["hbm_gbs"]},
        "step_graph": {"us": spread(step_graph),
                       "positions_per_s": world * B * q_len / statistics.median(step_graph) * 1e6,
                       "frac_hbm": step_bytes / statistics.median(step_graph) / 1e3
                       / peaks["hbm_gbs"]},
        "prefixcache": pc,
        "block_decode": blk,
        "lmhead_large_batch": lm_big,
        "sweep": sweep,
        "other_workloads": others,
        "block_decode_grid": grid,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": t_e2e / args.steps * 1e3,
                "upload": "double-buffered: step i+1's inputs copied on a second stream "
                          "during step i",
                "readback": "every step's results copied to pinned host memory on a third "
                            "stream and read on the host; the host reads step i-1's while "
                            "step i runs",
                "launch": "the step and its result copies replayed from one CUDA graph "
                          "per input set, captured from fdl_denoise_step",
                "serial": {"value": pos / t_e2e_serial,
                           "ms_per_step": t_e2e_serial / args.steps * 1e3,
                           "readback": "step i's results read on the host before step "
                                       "i+1 is launched"}},
        "gpu_launches": _launches_per_step(c) * args.steps,
        "committed_per_step": committed,
        "clocks": clk,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_baseline(case)
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


STEP_INPUTS = ("q", "k_blk", "v_blk", "hidden", "h_prev", "len_pre", "bt")


def _pack(torch, tensors: dict, device):
    """One byte buffer holding every tensor (256-byte aligned offsets) and
    views of it with the tensors' dtypes and shapes, filled with their
    values."""
    offs, total = {}, 0
    for k, t in tensors.items():
        offs[k] = total
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    buf = torch.empty(total, dtype=torch.uint8, device=device)
    views = {}
    for k, t in tensors.items():
        n = t.numel() * t.element_size()
        v = buf[offs[k]:offs[k] + n].view(t.dtype).view(t.shape)
        v.copy_(t)
        views[k] = v
    return buf, views


def _views(torch, buf, like_buf, like_views: dict) -> dict:
    """Views of `buf` at the offsets `like_views` have in `like_buf`."""
    base = like_buf.data_ptr()
    out = {}
    for k, v in like_views.items():
        if v.data_ptr() < base or v.data_ptr() >= base + like_buf.numel():
            continue
        o = v.data_ptr() - base
        n = v.numel() * v.element_size()
        out[k] = buf[o:o + n].view(v.dtype).view(v.shape)
    return out


def block_decode_leg(torch, fdl, c, x, w, stream, world, blocks: int = 5) -> dict:
    """One whole block (4 sub-blocks of 8) decoded by repeated fused steps
    until no position is masked, then appended to the prefix cache: as one
    CUDA graph with a device-side WHILE loop per sub-block, and driven from
    the host (one synchronisation per step).  The step inputs stay fixed
    (no model between steps), so the confidences repeat and each sub-block
    takes 1 + (positions left below tau) steps."""
    from block_diffusion_decoding_causal_b200 import driver
    B, D, q_len = c["batch"], c["block_size"], c["q_len"]
    units = D // q_len
    cap = x["k_pre"].shape[2] + 2 * D
    cfgs = [fdl.make_cfg(dict(c, q_off=u * q_len, cap_prefix=cap)) for u in range(units)]
    Hkv, d = c["n_kv_heads"], c["head_dim"]
    with torch.cuda.stream(stream):
        k_pre = torch.zeros((B, Hkv, cap, d), dtype=torch.bfloat16, device="cuda")
        v_pre = torch.zeros_like(k_pre)
        cap0 = x["k_pre"].shape[2]
        k_pre[:, :, :cap0].copy_(x["k_pre"])
        v_pre[:, :, :cap0].copy_(x["v_pre"])
        len0 = x["len_pre"].clone()
        lens = len0.clone()
        bt0 = torch.full((B, D), c["mask_id"], dtype=torch.int32, device="cuda")
        bt = bt0.clone()
        o = dict(attn=torch.empty_like(x["q"]),
                 conf=torch.empty((B, q_len), dtype=torch.float32, device="cuda"),
                 tok=torch.empty((B, q_len), dtype=torch.int32, device="cuda"),
                 comm=torch.empty((B, D), dtype=torch.uint8, device="cuda"),
                 n_c=torch.empty(B, dtype=torch.int32, device="cuda"),
                 n_l=torch.empty(B, dtype=torch.int32, device="cuda"),
                 any=torch.zeros(1, dtype=torch.int32, device="cuda"),
                 steps=torch.zeros(units, dtype=torch.int32, device="cuda"))
        ws = fdl.workspace(cfgs[0])
    stream.synchronize()

    def step(u, s):
        fdl.denoise_step(cfgs[u], x["q"], k_pre, v_pre, lens, x["k_blk"], x["v_blk"], None, None,
                         None, x["hidden"], x["h_prev"], w, bt, o["attn"], o["conf"], o["tok"],
                         o["comm"], o["n_c"], o["n_l"], ws, stream=s)

    def append(s):
        fdl.append_block(cfgs[0], x["k_blk"], x["v_blk"], k_pre, v_pre, lens, ws, stream=s)

    def reset():
        with torch.cuda.stream(stream):
            bt.copy_(bt0)
            lens.copy_(len0)
            o["steps"].zero_()

    g = driver.BlockGraph(cfgs, step, o["n_l"], o["steps"], append=append)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    for _ in range(2):
        reset()
        g.launch(stream)
    stream.synchronize()
    ev[0].record(stream)
    for _ in range(blocks):
        reset()
        g.launch(stream)
    ev[1].record(stream)
    stream.synchronize()
    steps_graph = o["steps"].cpu().tolist()
    ok = bool((bt != c["mask_id"]).all())
    ev[2].record(stream)
    steps_host = []
    for _ in range(blocks):
        reset()
        steps_host = []
        driver.run_host_loop(cfgs, step, o["n_l"], o["any"], steps_host, stream=stream)
        append(stream)
    ev[3].record(stream)
    stream.synchronize()
    t_graph = ev[0].elapsed_time(ev[1]) / blocks  # this rank's; reduced by the caller
    t_host = ev[2].elapsed_time(ev[3]) / blocks
    n_steps = sum(steps_graph)
    assert fdl.get_status(ws, stream) == 0
    return {"workload": f"one block of {D} positions, {units} sub-blocks of {q_len}, batch {B}",
            "steps_per_block": n_steps, "steps_per_sub_block": steps_graph,
            "host_loop_steps": steps_host, "block_decoded": ok,
            "graph_us_per_block": t_graph * 1e3, "host_loop_us_per_block": t_host * 1e3,
            "graph_us_per_step": t_graph * 1e3 / max(n_steps, 1),
            "positions_per_s_graph": B * D / (t_graph * 1e-3)}


def block_decode_grid(torch, fdl, c, x, w8, stream, world, blocks: int = 3) -> list:
    """The block decode at tau {0.7, 0.9, 1.0} x logit scale {4, 8, 12}:
    steps per block, committed tokens per step per sequence (D / steps, the
    pages' tokens-per-step figure) and the block time from the graph and from
    the host loop.  tau = 1.0 disables parallel decoding (one token per
    step unless an fp32 confidence rounds up to exactly 1)."""
    out = []
    D = c["block_size"]
    for sc in SWEEP_SCALE:
        w = _scaled_weight(torch, w8, sc)
        for tau in (0.7, 0.9, 1.0):
            try:
                r = block_decode_leg(torch, fdl, dict(c, tau=tau), x, w, stream, world,
                                     blocks=blocks)
            except Exception as e:  # reported; every rank still reduces below
                r = {"error": f"{type(e).__name__}: {e}"}
            for k in ("graph_us_per_block", "host_loop_us_per_block"):
                r[k] = max_over_ranks(float(r.get(k, float("nan"))), world)
            n = r.get("steps_per_block", 0)
            out.append({"tau": tau, "scale": sc, "steps_per_block": n,
                        "steps_per_sub_block": r.get("steps_per_sub_block"),
                        "tokens_per_step_per_sequence": D / n if n else None,
                        "graph_us_per_block": r["graph_us_per_block"],
                        "host_loop_us_per_block": r["host_loop_us_per_block"],
                        "block_decoded": r.get("block_decoded"),
                        **({"error": r["error"]} if "error" in r else {})})
        del w
    return out


PREFIXCACHE = dict(batch=1, n_q_heads=32, n_kv_heads=32, head_dim=128, prefix=768, rows=768)


def prefixcache_leg(torch, fdl, stream, timed, world, steps, peaks) -> dict:
    """PrefixCache attention at LLaDA-8B shapes: prompt 512 + 8 finished
    blocks cached (768 rows), answer length 1024 at block 9, so the active
    block and the masked suffix are 32 + 736 = 768 recomputed rows.  Eight
    input sets rotate (about 300 MB, more than L2)."""
    c = PREFIXCACHE
    B, Hq, Hkv, d, Lp, n = (c[k] for k in ("batch", "n_q_heads", "n_kv_heads", "head_dim",
                                           "prefix", "rows"))
    cfg = fdl.make_cfg(dict(batch=B, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, block_size=n,
                            q_off=0, q_len=n, cap_prefix=Lp, hidden=128, vocab=1000,
                            mask_id=999, shift=0, tau=0.9, dtype="bf16"))
    g = torch.Generator(device="cuda").manual_seed(7)
    rn = lambda *sh: torch.randn(sh, generator=g, device="cuda").to(torch.bfloat16)
    with torch.cuda.stream(stream):
        sets = [dict(q=rn(B, n, Hq, d), kp=rn(B, Hkv, Lp, d), vp=rn(B, Hkv, Lp, d),
                     kn=rn(B, Hkv, n, d), vn=rn(B, Hkv, n, d)) for _ in range(8)]
        lens = torch.full((B,), Lp, dtype=torch.int32, device="cuda")
        out = torch.empty((B, n, Hq, d), dtype=torch.bfloat16, device="cuda")
        ws = fdl.workspace(cfg)
    stream.synchronize()

    def run(i):
        x = sets[i % 8]
        fdl.prefixcache_attn(cfg, x["q"], x["kp"], x["vp"], lens, x["kn"], x["vn"], out, ws,
                             stream)
    for i in range(3):
        run(i)
    t = max_over_ranks(timed(run, steps), world) / steps
    t_graph = statistics.median(graph_rounds_us(torch, stream, run, steps, 3, world)) * 1e-6
    flops = 4.0 * B * Hq * n * (Lp + n) * d
    bytes_ = B * Hkv * (Lp + n) * d * 2 * 2 + 2 * B * n * Hq * d * 2
    bound = "tensor" if flops / (peaks["bf16_tflops"] * 1e12) > bytes_ / (peaks["hbm_gbs"] * 1e9) \
        else "hbm"
    return {"workload": "LLaDA-8B shapes, 32/32 heads, d 128, 768 cached + 768 recomputed rows",
            "us_per_launch": t * 1e6, "flops": flops, "bytes": bytes_, "bound": bound,
            "tflops": flops / t / 1e12, "frac_tensor": flops / t / 1e12 / peaks["bf16_tflops"],
            "gbs": bytes_ / t / 1e9, "frac_hbm": bytes_ / t / 1e9 / peaks["hbm_gbs"],
            "graph": {"us_per_launch": t_graph * 1e6,
                      "frac_tensor": flops / t_graph / 1e12 / peaks["bf16_tflops"]}}


def large_batch_lm_leg(torch, fdl, synth, stream, timed, world, steps, peaks) -> dict:
    """The LM head past the ridge: Qwen2.5-7B vocabulary, 64 sequences x 8
    positions = 512 rows, two passes of 256 rows over the weight."""
    c = dict(synth.CONFIGS["qwen7b"], batch=64, q_off=0, w_layout=fdl.W_PACKED)
    cfg = fdl.make_cfg(c)
    R, H, V = c["batch"] * c["q_len"], c["hidden"], c["vocab"]
    g = torch.Generator(device="cuda").manual_seed(11)
    with torch.cuda.stream(stream):
        w_row_major = (torch.randn((V, H), generator=g, device="cuda")
                       * (8.0 / H ** 0.5)).to(torch.bfloat16)
        w = torch.empty_like(w_row_major)
        fdl.lmhead_pack_weight(cfg, w_row_major, w, stream)
        del w_row_major
        rows = torch.randn((R, H), generator=g, device="cuda").to(torch.bfloat16)
        conf = torch.empty(R, dtype=torch.float32, device="cuda")
        tok = torch.empty(R, dtype=torch.int32, device="cuda")
        ws = fdl.workspace(cfg)
    stream.synchronize()
    run = lambda i: fdl.lmhead_confidence(cfg, rows, w, None, conf, tok, ws, stream)
    for i in range(3):
        run(i)
    t = max_over_ranks(timed(run, steps), world) / steps
    flops = 2.0 * V * H * R
    del w
    return {"workload": "Qwen2.5-7B vocabulary, 512 rows (64 x 8), 2 passes",
            "us_per_launch": t * 1e6, "flops": flops, "bound": "tensor",
            "tflops": flops / t / 1e12, "frac_tensor": flops / t / 1e12 / peaks["bf16_tflops"]}


SWEEP_BATCH = (1, 4, 16)
SWEEP_PREFIX = (2048, 8192)
SWEEP_SCALE = (4.0, 8.0, 12.0)


def _scaled_weight(torch, w8, scale: float):
    """The Qwen2.5-7B LM-head weight at another logit scale: the scale-8
    draw times scale / 8, rounded to bf16 (layout-independent, so it applies
    to the tiled copy as is)."""
    if scale == 8.0:
        return w8
    out = torch.empty_like(w8)
    step_rows = 8192
    for r0 in range(0, w8.shape[0], step_rows):
        out[r0:r0 + step_rows] = (w8[r0:r0 + step_rows].float() * (scale / 8.0)).to(w8.dtype)
    return out


def _attn_bytes(c, len_pre, len_suf=None) -> int:
    """Algorithmic bytes of the attention: K and V of every visible key once
    (prefix + block + suffix, per KV head), Q in and O out."""
    B, q_len, D = c["batch"], c["q_len"], c["block_size"]
    keys = int(len_pre.sum()) + B * D + (0 if len_suf is None else int(len_suf.sum()))
    return (keys * c["n_kv_heads"] * 2 * c["head_dim"] * 2
            + 2 * B * q_len * c["n_q_heads"] * c["head_dim"] * 2)


def _lm_bytes_flops(c) -> tuple:
    R, H, V = c["batch"] * c["q_len"], c["hidden"], c["vocab"]
    return V * H * 2 + R * H * 2 + R * 8, 2.0 * V * H * R


def _device_inputs(torch, case, stream, copies: int):
    """The case's step inputs on the device, with ``copies`` distinct copies
    of the KV caches (the attention reads rotate over them)."""
    dev = lambda t: None if t is None else t.cuda().contiguous()
    with torch.cuda.stream(stream):
        base = dict(q=dev(case.q), len_pre=dev(case.len_pre), k_blk=dev(case.k_blk),
                    v_blk=dev(case.v_blk), hidden=dev(case.hidden), h_prev=dev(case.h_prev),
                    len_suf=dev(case.len_suf), bt0=dev(case.block_tokens))
        kv = []
        first = dict(k_pre=dev(case.k_pre), v_pre=dev(case.v_pre), k_suf=dev(case.k_suf),
                     v_suf=dev(case.v_suf))
        for i in range(copies):
            kv.append(first if i == 0 else
                      {k: None if v is None else v.clone() for k, v in first.items()})
        base["bt"] = base["bt0"].clone()
    return base, kv


def _step_outputs(torch, c):
    B, q_len, D = c["batch"], c["q_len"], c["block_size"]
    return dict(conf=torch.empty((B, q_len), dtype=torch.float32, device="cuda"),
                tok=torch.empty((B, q_len), dtype=torch.int32, device="cuda"),
                comm=torch.empty((B, D), dtype=torch.uint8, device="cuda"),
                n_c=torch.empty(B, dtype=torch.int32, device="cuda"),
                n_l=torch.empty(B, dtype=torch.int32, device="cuda"))


def sweep_leg(torch, fdl, synth, stream, timed, world, steps, peaks, w8, seed,
              reps: int = 3) -> dict:
    """Long-context sweep at Qwen2.5-7B shapes: batch {1, 4, 16} x prefix
    {2048, 8192} x logit scale {4, 8, 12}.  Per (batch, prefix): the
    attention entry point alone (algorithmic bytes, GB/s, fraction of the
    measured HBM bandwidth); per batch: the LM head alone against its roofline
    (the slower of its weight bytes at HBM bandwidth and its FLOPs at the
    tensor peak); per point: the fused step and the tokens one step commits
    from the case's block state.  KV caches rotate over enough copies to
    exceed twice the L2; every timing is ``reps`` rounds of ``steps``
    launches (median and range)."""
    hbm = peaks["hbm_gbs"] * 1e9
    tens = peaks["bf16_tflops"] * 1e12
    weights = {sc: _scaled_weight(torch, w8, sc) for sc in SWEEP_SCALE}
    lm_by_batch, points = {}, []
    for B in SWEEP_BATCH:
        for P in SWEEP_PREFIX:
            case = synth.make_case("sweep", seed, cfg=synth.sweep_config(B, P, 8.0),
                                   draw_w=False)
            c = dict(case.cfg, w_layout=fdl.W_PACKED)
            cfg = fdl.make_cfg(c)
            Hkv, d = c["n_kv_heads"], c["head_dim"]
            n_kv = kv_copies_for(torch, B * Hkv * P * d * 2 * 2)
            x, kv = _device_inputs(torch, case, stream, n_kv)
            o = _step_outputs(torch, c)
            with torch.cuda.stream(stream):
                attn_out = torch.empty_like(x["q"])
                ws = fdl.workspace(cfg)
            stream.synchronize()

            def attn(i):
                y = kv[i % n_kv]
                fdl.block_attn(cfg, x["q"], y["k_pre"], y["v_pre"], x["len_pre"], x["k_blk"],
                               x["v_blk"], attn_out, ws, stream)
            for i in range(3):
                attn(i)
            a_us = rounds_us(timed, attn, steps, reps, world)
            a_graph = graph_rounds_us(torch, stream, attn, steps, reps, world)
            a_bytes = _attn_bytes(c, case.len_pre)
            lm_bytes, lm_flops = _lm_bytes_flops(c)
            if B not in lm_by_batch:
                rows = x["hidden"].view(B * c["q_len"], c["hidden"])
                lm = lambda i: fdl.lmhead_confidence(cfg, rows, w8, None, o["conf"], o["tok"],
                                                     ws, stream)
                for i in range(3):
                    lm(i)
                l_us = rounds_us(timed, lm, steps, reps, world)
                t_roof = roofline_seconds(lm_bytes, lm_flops, hbm, tens)
                lm_by_batch[B] = {"rows": B * c["q_len"], "us": spread(l_us),
                                  "roofline_us": t_roof * 1e6,
                                  "frac": t_roof * 1e6 / statistics.median(l_us),
                                  "bound": "hbm" if lm_bytes / hbm >= lm_flops / tens
                                  else "tensor"}
            for sc in SWEEP_SCALE:
                w = weights[sc]

                def step(i):
                    y = kv[i % n_kv]
                    fdl.denoise_step(cfg, x["q"], y["k_pre"], y["v_pre"], x["len_pre"],
                                     x["k_blk"], x["v_blk"], None, None, None, x["hidden"],
                                     x["h_prev"], w, x["bt"], None, o["conf"], o["tok"],
                                     o["comm"], o["n_c"], o["n_l"], ws, stream)
                # tokens one step commits from the case's block state
                with torch.cuda.stream(stream):
                    x["bt"].copy_(x["bt0"])
                step(0)
                stream.synchronize()
                n_c = o["n_c"].cpu()
                masked = int((case.block_tokens[:, c["q_off"]:c["q_off"] + c["q_len"]]
                              == c["mask_id"]).sum())
                for i in range(3):
                    step(i)
                with ClockSampler(_gpu_id(torch)) as clk:
                    s_us = rounds_us(timed, step, steps, reps, world)
                s_bytes = a_bytes + lm_bytes + (2 * B * c["q_len"] * c["hidden"] * 2)
                points.append({
                    "batch": B, "prefix": P, "scale": sc,
                    "attention": {"us": spread(a_us), "bytes": a_bytes,
                                  "gbs": a_bytes / statistics.median(a_us) / 1e3,
                                  "frac_hbm": a_bytes / statistics.median(a_us) / 1e3
                                  / peaks["hbm_gbs"],
                                  "graph": {"us": spread(a_graph),
                                            "frac_hbm": a_bytes / statistics.median(a_graph)
                                            / 1e3 / peaks["hbm_gbs"]}},
                    "lm_head_frac": lm_by_batch[B]["frac"],
                    "step": {"us": spread(s_us),
                             "positions_per_s": B * c["q_len"] / statistics.median(s_us) * 1e6,
                             "frac_hbm": s_bytes / statistics.median(s_us) / 1e3
                             / peaks["hbm_gbs"],
                             "clocks": clk.summary()},
                    "masked_in_unit": masked,
                    "committed_per_step": int(n_c.sum()),
                    "committed_per_sequence": (n_c.float().mean().item()),
                    "kv_copies": n_kv})
            assert fdl.get_status(ws, stream) == 0
            del kv, x, o, attn_out, ws
            torch.cuda.empty_cache()
    del weights
    return {"workload": "Qwen2.5-7B shapes (28/4 heads, d 128, H 3584, V 152064), "
                        "block 32 / sub-block 8, tau 0.9, tiled LM-head weight",
            "peak_hbm_gbs": peaks["hbm_gbs"], "peak_tflops": peaks["bf16_tflops"],
            "lm_head": {str(b): v for b, v in lm_by_batch.items()},
            "points": points}


def configs_leg(torch, fdl, synth, stream, timed, world, steps, peaks, seed,
                reps: int = 3) -> dict:
    """The other single-GPU workloads: Qwen2.5-1.5B shapes (batch 1, prefix
    512) and LLaDA-8B-like DualCache (prefix 768 + block 32 + suffix 736,
    all 32 block positions queried): the fused step, the LM head and the
    attention entry point alone, each against the measured HBM bandwidth."""
    hbm = peaks["hbm_gbs"] * 1e9
    tens = peaks["bf16_tflops"] * 1e12
    res = {}
    for name in ("qwen1.5b", "llada"):
        case = synth.make_case(name, seed)
        c = dict(case.cfg, w_layout=fdl.W_PACKED)
        cfg = fdl.make_cfg(c)
        B, Hkv, d = c["batch"], c["n_kv_heads"], c["head_dim"]
        per_copy = B * Hkv * (c["cap_prefix"] + c["cap_suffix"]) * d * 2 * 2
        n_kv = kv_copies_for(torch, per_copy)
        x, kv = _device_inputs(torch, case, stream, n_kv)
        o = _step_outputs(torch, c)
        with torch.cuda.stream(stream):
            w_rm = case.w_lm.cuda()
            w = torch.empty_like(w_rm)
            fdl.lmhead_pack_weight(cfg, w_rm, w, stream)
            del w_rm
            attn_out = torch.empty_like(x["q"])
            ws = fdl.workspace(cfg)
        stream.synchronize()
        dual = case.k_suf is not None

        def step(i):
            y = kv[i % n_kv]
            fdl.denoise_step(cfg, x["q"], y["k_pre"], y["v_pre"], x["len_pre"], x["k_blk"],
                             x["v_blk"], y["k_suf"], y["v_suf"], x["len_suf"], x["hidden"],
                             x["h_prev"], w, x["bt"], None, o["conf"], o["tok"], o["comm"],
                             o["n_c"], o["n_l"], ws, stream)

        def attn(i):
            y = kv[i % n_kv]
            if dual:
                fdl.dualcache_attn(cfg, x["q"], y["k_pre"], y["v_pre"], x["len_pre"],
                                   x["k_blk"], x["v_blk"], y["k_suf"], y["v_suf"],
                                   x["len_suf"], attn_out, ws, stream)
            else:
                fdl.block_attn(cfg, x["q"], y["k_pre"], y["v_pre"], x["len_pre"], x["k_blk"],
                               x["v_blk"], attn_out, ws, stream)
        rows = x["hidden"].view(B * c["q_len"], c["hidden"])
        lm = lambda i: fdl.lmhead_confidence(cfg, rows, w, None, o["conf"], o["tok"], ws,
                                             stream)
        out = {}
        for key, fn in (("step", step), ("lm_head", lm), ("attention", attn)):
            for i in range(3):
                fn(i)
            out[key] = rounds_us(timed, fn, steps, reps, world)
        attn_graph = graph_rounds_us(torch, stream, attn, steps, reps, world)
        with torch.cuda.stream(stream):
            x["bt"].copy_(x["bt0"])
        step(0)
        stream.synchronize()
        committed = int(o["n_c"].sum().item())
        assert fdl.get_status(ws, stream) == 0
        a_bytes = _attn_bytes(c, case.len_pre, case.len_suf)
        lm_bytes, lm_flops = _lm_bytes_flops(c)
        shift_bytes = 2 * B * c["q_len"] * c["hidden"] * 2 if c["shift"] else 0
        s_bytes = a_bytes + lm_bytes + shift_bytes
        t_step = statistics.median(out["step"])
        t_lm = statistics.median(out["lm_head"])
        t_attn = statistics.median(out["attention"])
        lm_roof = roofline_seconds(lm_bytes, lm_flops, hbm, tens) * 1e6
        res[name] = {
            "workload": ("Qwen2.5-1.5B shapes: batch 1, 12/2 heads, d 128, H 1536, "
                         "V 151936, prefix 512, block 32 / sub-block 8, tau 0.9"
                         if name == "qwen1.5b" else
                         "LLaDA-8B-like DualCache: batch 1, 32/32 heads, d 128, H 4096, "
                         "V 126464, prefix 768 + block 32 + suffix 736, tau 0.9"),
            "step": {"us": spread(out["step"]), "bytes": s_bytes,
                     "positions_per_s": B * c["q_len"] / t_step * 1e6,
                     "frac_hbm": s_bytes / t_step / 1e3 / peaks["hbm_gbs"]},
            "lm_head": {"us": spread(out["lm_head"]), "bytes": lm_bytes,
                        "roofline_us": lm_roof, "frac": lm_roof / t_lm},
            "attention": {"us": spread(out["attention"]), "bytes": a_bytes,
                          "gbs": a_bytes / t_attn / 1e3,
                          "frac_hbm": a_bytes / t_attn / 1e3 / peaks["hbm_gbs"],
                          "graph": {"us": spread(attn_graph),
                                    "frac_hbm": a_bytes / statistics.median(attn_graph) / 1e3
                                    / peaks["hbm_gbs"]}},
            "committed_first_step": committed, "kv_copies": n_kv}
        del kv, x, o, w, attn_out, ws
        torch.cuda.empty_cache()
    return res


def _gpu_id(torch) -> str:
    """nvidia-smi identifier (UUID) of the current CUDA device."""
    try:
        u = str(torch.cuda.get_device_properties(torch.cuda.current_device()).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(torch.cuda.current_device())


def _launches_per_step(c) -> int:
    """Kernels one fdl_denoise_step launches at these shapes.  bf16, head
    dim 128, hidden rows given and at most 64 LM-head rows: the token-shift
    gather (if shifting), the fused LM head + commit, and the attention beside
    it; otherwise attention, its partial merge, the gather (if shifting) and
    the LM head."""
    beside = (c["dtype"] == "bf16" and c["head_dim"] == 128
              and c["batch"] * c["q_len"] <= 64)
    return (2 if beside else 3) + (1 if c["shift"] else 0)


KERNEL_SOURCES = {
    "lmhead": ["lmhead_tc.cu", "lm_merge.cuh", "fdl_common.cuh", "sm100.cuh"],
    "attn": ["attn_tc.cu", "fdl_common.cuh", "sm100.cuh"],
}


def kernel_source_sha(kernel: str) -> str:
    """SHA-256 over the CUDA sources a kernel is built from."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "block_diffusion_decoding_causal_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def _profiled_traffic(kernel: str, summary: str, units_here: float = None):
    """DRAM bytes per launch from a committed ncu summary under profiles/, or
    None when the summary is missing or the kernel's sources changed since the
    counters were taken.  A summary captured on a smaller case states its
    units; the bytes are scaled to this launch's units."""
    path = os.path.join(ROOT, "profiles", summary)
    if not os.path.exists(path):
        return None
    fields = {}
    with open(path) as f:
        for line in f:
            if ":" in line and not line.startswith("|"):
                k, v = line.split(":", 1)
                fields[k.strip().lstrip("- ")] = v.strip().strip("`")
    if fields.get("kernel_source_sha256") != kernel_source_sha(kernel):
        return None
    try:
        b = float(fields["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None
    if units_here is not None and "units_per_launch" in fields:
        b *= units_here / float(fields["units_per_launch"])
    return b


if __name__ == "__main__":
    sys.exit(main())
