"""Host-side logic of bench.py that needs no GPU: the choice of pinned host
buffers for the end-to-end leg, and its agreement across ranks (two gloo ranks
whose free memory differs must take the same, more restrictive choice, or
their collectives would diverge)."""

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
