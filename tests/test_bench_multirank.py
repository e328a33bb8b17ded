"""The benchmark's multi-rank host logic on CPU with the gloo backend
(world size 2): rows are sharded by rank (each rank draws its own batch), the
job time is the maximum of the ranks' times, and the throughput counts every
rank's tokens.  The GPU steps themselves need no exchange."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from moe_expert_routing_token_b200 import inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 * (rank + 1)
        dist.barrier()
        ms = bench.job_elapsed_ms(local_ms, world, torch.device("cpu"))
        seed = bench.rank_seed("sigmoid", 64, rank)
        first = inputs.make("sigmoid", 64, seed=seed)["logits"][0, :4].float().tolist()
        out[rank] = (ms, bench.job_tokens_per_s(64, 5, world, ms), seed, first)
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_sharded_rows():
    world = 2
    with mp.get_context("spawn").Manager() as mgr:  # no fork of a threaded test process
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 20.0          # max over ranks, on every rank
    assert res[0][1] == res[1][1] == 64 * 5 * 2 / 0.020
    assert res[0][2] != res[1][2]                  # distinct batches per rank
    assert res[0][3] != res[1][3]


def test_single_rank_needs_no_process_group():
    assert bench.job_elapsed_ms(3.5, 1, torch.device("cpu")) == 3.5
    assert bench.job_tokens_per_s(100, 10, 1, 1000.0) == 1000.0
