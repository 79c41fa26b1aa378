"""Multi-rank plumbing of bench.py on CPU: two gloo ranks.

Each rank decodes its own sequences, so the only cross-rank operations are
the timing barrier and the reduction of (elapsed, bytes): the job's time is
the slowest rank's, its bytes the sum over ranks.
"""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cpu = torch.device("cpu")
        bench.barrier(world, cpu)
        elapsed = [12.5, 30.25][rank]
        nbytes = [1e9, 3e9][rank]
        results[rank] = bench.reduce_timing(elapsed, nbytes, world, cpu)
        # each rank draws its own sequences: seed + rank gives other lengths
        import synth
        w = synth.WORKLOADS["llama7b"]
        results[10 + rank] = tuple(synth.draw_lengths(w, 0 + rank)[:4])
        bench.barrier(world, cpu)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_max_time_and_sum_bytes():
    world = 2
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert results[0] == (30.25, 4e9) and results[1] == (30.25, 4e9)
    assert results[10] != results[11]


def test_single_rank_needs_no_collective():
    import bench
    assert bench.reduce_timing(3.0, 5.0, 1, torch.device("cpu")) == (3.0, 5.0)
