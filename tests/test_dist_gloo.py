"""The multi-rank path on CPU: two gloo ranks (spawned processes) run the
plumbing bench.py uses on N GPUs (lora_gemm_b200.dist) and check what it
promises: the max and sum over ranks, the whole-job rate, and that the ranks'
slices of the Philox stream are disjoint, block-aligned and together equal
one process's stream over the concatenated batches (checked with the
oracle's generator); and, for one clip split by latent frames over 2 and 3
ranks, that the ranks' re-noised latents and Euler chains (each rank running
the oracle on its own frames with its own noise offset) put side by side
equal one process's bit for bit."""

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


def _clip_rank_main(rank, world, port, shape, seed):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    import torch
    import torch.distributed as tdist

    from lora_gemm_b200 import dist
    from oracle import flow, noise

    F, C, H, W = shape
    r, w, _ = dist.init(world, backend="gloo", timeout_s=60)
    try:
        (t0, t1), (e0, e1) = dist.clip_shard(F, C, H, W, r, w)
        f0, f1 = dist.frame_shard(F, r, w)
        assert (t0, t1) == (f0 * H * W, f1 * H * W) and e0 % 4 == 0
        # The clip's inputs, identical on every rank (seeded); each rank keeps its frames.
        g = np.random.default_rng(seed)
        up = g.standard_normal(F * C * H * W).astype(np.float32)
        vs = [g.standard_normal(F * C * H * W).astype(np.float32) for _ in range(3)]
        sched = flow.SCHEDULE
        z = flow.renoise(up[e0:e1], noise.normal(seed, e0, e1 - e0), sched[0]).astype(np.float32)
        for k in range(3):
            z = flow.euler_step(z, vs[k][e0:e1], sched[k], sched[k + 1]).astype(np.float32)
        # Gather the ranks' slices (padded to the largest) and compare with one process.
        n_max = max(b - a for _, (a, b) in (dist.clip_shard(F, C, H, W, q, w) for q in range(w)))
        mine = torch.zeros(n_max, dtype=torch.float32)
        mine[:e1 - e0] = torch.from_numpy(z)
        parts = [torch.zeros(n_max, dtype=torch.float32) for _ in range(w)]
        tdist.all_gather(parts, mine)
        pieces = []
        for q in range(w):
            _, (a, b) = dist.clip_shard(F, C, H, W, q, w)
            pieces.append(parts[q][:b - a].numpy())
        got = np.concatenate(pieces)
        whole = flow.renoise(up, noise.normal(seed, 0, up.size), sched[0]).astype(np.float32)
        for k in range(3):
            whole = flow.euler_step(whole, vs[k], sched[k], sched[k + 1]).astype(np.float32)
        assert got.shape == whole.shape
        assert np.array_equal(got.view(np.uint32), whole.view(np.uint32))
        dist.barrier(w)
    finally:
        dist.destroy(w)


@pytest.mark.parametrize("world,shape", [(2, (5, 24, 6, 10)), (3, (4, 24, 3, 5))])
def test_one_clip_split_by_frames(world, shape):
    mp.spawn(_clip_rank_main, args=(world, _free_port(), shape, 11), nprocs=world, join=True)


def test_frame_shard_partitions_the_clip():
    from lora_gemm_b200 import dist

    for frames in (0, 1, 5, 37):
        for world in (1, 2, 3, 4, 8):
            ranges = [dist.frame_shard(frames, r, world) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == frames
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)
    (t0, t1), (e0, e1) = dist.clip_shard(37, 24, 90, 160, 1, 8)
    assert (t0, t1) == (5 * 14400, 10 * 14400) and (e0, e1) == (5 * 24 * 14400, 10 * 24 * 14400)
    with pytest.raises(ValueError):
        dist.clip_shard(4, 3, 3, 3, 0, 2)
