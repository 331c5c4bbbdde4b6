"""World-size-2 host logic of the benchmark on CPU (gloo): each rank gets its
own batch of sequences, and the reported time is the max over ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    from block_diffusion_decoding_causal_b200 import synth
    seed = bench.rank_seed(1002, rank)
    case = synth.make_case("tiny", seed)
    mine = float(10 + rank)                       # rank 1 is the slow one
    got = bench.max_over_ranks(mine, world, device="cpu")
    q_sum = float(case.q.double().sum())
    gathered = [None] * world
    dist.all_gather_object(gathered, (seed, q_sum))
    out[rank] = (got, gathered)
    dist.destroy_process_group()


def test_two_ranks_shard_by_sequence_and_take_the_max():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    for rank in range(world):
        got, gathered = out[rank]
        assert got == 11.0
        seeds = [g[0] for g in gathered]
        sums = [g[1] for g in gathered]
        assert len(set(seeds)) == world and sums[0] != sums[1]
