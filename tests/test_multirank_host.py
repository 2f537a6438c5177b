"""The multi-rank host logic of bench.py on CPU: two gloo ranks. Step times
are combined as the max over ranks, and a decision that gates collectives
(whether to run the host-buffer measurement) is taken the same way on every
rank. The reference arm does its work on rank 0 only."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


PORT = _free_port()


def _worker(rank, world, port, queue):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(10.0 + rank, dist, device="cpu")
        only_rank0 = bench.all_ranks(rank == 0, dist, device="cpu")
        everyone = bench.all_ranks(True, dist, device="cpu")
        queue.put((rank, ms, only_rank0, everyone))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_time_and_decisions():
    world = 2
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, PORT, queue))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(queue.get(timeout=10) for _ in range(world))
    assert [r[1] for r in res] == [11.0, 11.0]          # max over ranks on every rank
    assert [r[2] for r in res] == [False, False]        # one rank said no: all skip
    assert [r[3] for r in res] == [True, True]



def test_single_process_helpers_without_a_group():
    assert bench.max_over_ranks(3.5, None) == 3.5
    assert bench.all_ranks(True, None) is True
    assert bench.all_ranks(0, None) is False


def test_reference_arm_is_rank0_only():
    class Args:
        workload = "tiny"
        steps = 1
        warmup = 0
    assert bench.main_reference(Args(), world=2, rank=1) is None   # no work, no output
