"""The N > 1 host path of bench.py, as two gloo ranks on the CPU.

Each rank processes its own sequences (weak scaling, no data-path collective);
the step time is the max over ranks and the throughput counts every rank's
tokens. These checks run the same helpers bench.py uses under torchrun.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    from dsa_inputs import CONFIGS, gen_inputs
    try:
        ms = 10.0 + 5.0 * rank                       # a slower rank 1
        ms_max = bench.dist_max(ms, world)
        bench.barrier(world)
        seed = bench.rank_seed("tiny", rank)
        inp = gen_inputs(CONFIGS["tiny"], "cpu", seed=seed)
        digest = float(inp["q"].float().sum())
        seeds = [None] * world
        dist.all_gather_object(seeds, (seed, digest))
        value = bench.aggregate_tokens_per_s(CONFIGS["tiny"].tokens, world, ms_max)
        q.put((rank, ms_max, seeds, value))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling_host_logic():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms_max, seeds, value in results:
        assert ms_max == 15.0                         # max over ranks, not the local time
        assert seeds[0][0] != seeds[1][0]             # every rank has its own sequences
        assert seeds[0][1] != seeds[1][1]
        assert value == pytest.approx(256 * 2 / 15e-3)  # all ranks' tokens / slowest time
