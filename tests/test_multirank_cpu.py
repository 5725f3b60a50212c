"""The multi-GPU plumbing of bench.py on two CPU ranks (gloo): every rank gets a disjoint share of
the decode sequences (together they cover the job), prefill ranks get distinct seeds, and the job's
time is the largest elapsed time over the ranks."""
import os
import socket
import sys

import torch.multiprocessing as tmp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch
    import torch.distributed as dist
    import bench
    from long_context_sparse_mean_b200 import workloads as W

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        seqs = bench.rank_sequences(rank, world, 5)
        gathered = [None] * world
        dist.all_gather_object(gathered, seqs)
        wl = bench.rank_workload(W.WORKLOADS[3], rank)
        seeds = [None] * world
        dist.all_gather_object(seeds, wl.seed)
        t = bench.max_over_ranks(10.0 + 7.0 * rank, dist, "cpu")
        out[rank] = (gathered, seeds, t)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_time():
    world = 2
    port = _free_port()
    mgr = tmp.get_context("spawn").Manager()  # no fork of this (threaded) test process
    out = mgr.dict()
    tmp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    for rank in range(world):
        gathered, seeds, t = out[rank]
        flat = [s for part in gathered for s in part]
        assert sorted(flat) == list(range(world * 5)), "shares overlap or leave a gap"
        assert len(set(seeds)) == world, "prefill ranks share a seed"
        assert t == 17.0, "the job time is the max over ranks"
