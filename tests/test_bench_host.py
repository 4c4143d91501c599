"""Host-side logic of bench.py that needs no GPU: the choice of pinned host
buffers for the end-to-end leg, and its agreement across ranks (two gloo ranks
whose free memory differs must take the same, more restrictive choice, or
their collectives would diverge); and the skipping of a grid whose inputs do
not fit in device memory, which all ranks must do together when any one of
them runs short."""

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def test_host_buffer_choice():
    assert bench.host_buffer_choice(10, 20, None) == 0
    assert bench.host_buffer_choice(10, 20, 30) == 0
    assert bench.host_buffer_choice(10, 20, 29) == 1
    assert bench.host_buffer_choice(10, 20, 20) == 1
    assert bench.host_buffer_choice(10, 20, 19) == 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, budgets, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = bench.host_buffer_choice(10, 20, budgets[rank])
        out[rank] = int(bench.max_over_ranks(float(mine), world))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("budgets,expect", [((40, 25), 1), ((25, 15), 2), ((40, 40), 0)])
def test_ranks_agree_on_the_most_restrictive_choice(budgets, expect):
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, budgets, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert out[0] == out[1] == expect


def _workloads_rank(rank, world, port, oom_ranks, out):
    """run_workloads with the grid's inputs failing to allocate on some ranks:
    every rank must skip the grid (and run no timed step), whichever rank ran
    short."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import argparse

        import torch

        def fake_problem(*args, **kwargs):
            if rank in oom_ranks:
                raise torch.cuda.OutOfMemoryError("CUDA out of memory. Tried to allocate 69.00 GiB")
            return object()

        def no_timed_steps(*args, **kwargs):
            raise AssertionError("a skipped grid must not be timed")

        bench.Problem = fake_problem
        bench.time_steps = no_timed_steps
        bench.run_step = no_timed_steps
        args = argparse.Namespace(scaling="weak", steps=1, warmup=3)
        res = bench.run_workloads(["4k"], args, world, rank, torch.device("cpu"), {})
        out[rank] = res["4k"].get("unavailable", "")
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("oom_ranks", [(1,), (0,), (0, 1)])
def test_ranks_skip_a_grid_together_when_any_runs_out_of_memory(oom_ranks):
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_workloads_rank, args=(r, 2, port, oom_ranks, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r in range(2):
        assert out[r].startswith("device memory"), out[r]
        assert ("another rank" in out[r]) == (r not in oom_ranks)
