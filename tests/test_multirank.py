"""Host-side logic of the multi-GPU (weak-scaling, data-parallel) bench path,
run as two gloo ranks on the CPU: each rank decodes its own batch, times are
the slowest rank's and bytes add up; no collective touches the data path."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from mla_decode_attention_15_b200 import workloads


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, _ = bench.dist_env()
        assert (w, r) == (world, rank)
        # different ranks, different per-rank times and byte counts
        times, total = bench.aggregate_over_ranks([1.0 + rank, 10.0 - rank], 100.0 * (rank + 1),
                                                  torch.device("cpu"))
        seed = bench.rank_seed(1003, rank)
        seeds = [None] * world
        dist.all_gather_object(seeds, seed)
        lens = workloads.build(2, 1, 16, ("uniform", 64, 256), seed=seed)["cache_seqlens"].tolist()
        q.put((rank, times, total, seeds, lens))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_aggregate_max_time_and_sum_bytes():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    for rank, times, total, seeds, _ in out:
        assert times == [2.0, 10.0]          # max over ranks of each entry
        assert total == 300.0                # sum of 100 and 200
        assert seeds == [1003, 1003 + 7919]  # rank 0 decodes the named workload itself
    assert out[0][4] != out[1][4]            # each rank draws its own batch


def test_single_process_aggregation_is_identity():
    times, total = bench.aggregate_over_ranks([3.0, 4.0], 123.0, torch.device("cpu"))
    assert times == [3.0, 4.0] and total == 123.0
