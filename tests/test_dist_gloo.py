"""The multi-rank path on CPU: two gloo ranks (spawned processes) run the
plumbing bench.py uses on N GPUs (lora_gemm_b200.dist) and check what it
promises: the max and sum over ranks, the whole-job rate, and that the ranks'
slices of the Philox stream are disjoint, block-aligned and together equal
one process's stream over the concatenated batches (checked with the
oracle's generator)."""

import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, latent_numel, seed):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    import torch
    import torch.distributed as tdist

    from lora_gemm_b200 import dist
    from oracle import noise

    r, w, local = dist.init(world, backend="gloo", timeout_s=60)
    try:
        assert (r, w, local) == (rank, world, rank)
        assert dist.max_over_ranks(rank + 0.5, w) == world - 0.5
        assert dist.sum_over_ranks(1.0, w) == world
        # every rank's units over the slowest rank's time
        assert dist.whole_job_rate(1000, w, 5, 250.0) == world * 1000 * 5 / 0.25

        off = dist.noise_offset(r, latent_numel)
        assert off % 4 == 0
        offs = [torch.zeros(1, dtype=torch.int64) for _ in range(w)]
        tdist.all_gather(offs, torch.tensor([off], dtype=torch.int64))
        offs = [int(t.item()) for t in offs]
        assert offs == sorted(offs) and offs[0] == 0
        for a, b in zip(offs, offs[1:]):
            assert b - a >= latent_numel and b - a - latent_numel < 4  # disjoint, padded to a block

        mine = noise.normal(seed, off, latent_numel)
        whole = noise.normal(seed, 0, offs[-1] + latent_numel)
        assert np.array_equal(mine, whole[off:off + latent_numel])
        dist.barrier(w)
    finally:
        dist.destroy(w)


@pytest.mark.parametrize("latent_numel", [55296, 1001])
def test_two_gloo_ranks(latent_numel):
    mp.spawn(_rank_main, args=(2, _free_port(), latent_numel, 7), nprocs=2, join=True)
