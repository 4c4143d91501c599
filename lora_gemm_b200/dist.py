"""Multi-process plumbing for the refiner hot path: one process per GPU.

The path has no exchange step, and it splits two ways with no collective on
the data path:

* replicas (weak scaling): each rank refines its own batch (its own latent
  and activations) and draws its noise from its own slice of the Philox
  stream (noise_offset), so N ranks together compute exactly what one
  process would compute over the concatenation of their batches;
* one clip split by latent frames (strong scaling): rank r takes frames
  [f0, f1) of the clip (frame_shard), i.e. tokens [f0 H W, f1 H W) and the
  latent elements [f0 C H W, f1 C H W) of the flat [F, C, H, W] latent
  (clip_shard); the Philox counter of an element is its global index, so
  the ranks' re-noised latents, put side by side, equal one process's bit
  for bit.

The only collectives are the barrier that brackets a timed region and the
max-over-ranks of its duration.

Works with the NCCL backend (one GPU per rank) and with gloo on CPU, which is
how the multi-rank logic is tested without GPUs.
"""

import datetime
import os

import torch


def env_ranks():
    """(rank, world, local_rank) from the torchrun environment (1 process if unset)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(n_ranks, backend="nccl", timeout_s=600):
    """Join the process group of `n_ranks` processes; returns (rank, world, local).

    With backend "nccl" each rank binds GPU `local`; with one rank no process
    group is created.  The timeout bounds every collective, so a rank that never
    arrives ends the others with an error instead of a hang."""
    rank, world, local = env_ranks()
    if world != n_ranks:
        raise SystemExit(f"{n_ranks} ranks requested but WORLD_SIZE={world}")
    if world > 1:
        import torch.distributed as dist

        kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, **kw)
    elif backend == "nccl":
        torch.cuda.set_device(0)
    return rank, world, local


def _reduce_device():
    import torch.distributed as dist

    return torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu")


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(value, world):
    """The largest `value` over all ranks (every rank gets it)."""
    if world == 1:
        return value
    import torch.distributed as dist

    t = torch.tensor([value], dtype=torch.float64, device=_reduce_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value, world):
    if world == 1:
        return value
    import torch.distributed as dist

    t = torch.tensor([value], dtype=torch.float64, device=_reduce_device())
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def noise_offset(rank, latent_numel):
    """Element offset of rank `rank`'s latent in the shared Philox stream.

    Rank r's batch is elements [r * stride, r * stride + latent_numel) of one
    stream, with stride = latent_numel rounded up to a Philox block (4), the
    granularity at which a re-noise may start."""
    stride = (latent_numel + 3) // 4 * 4
    return rank * stride


def frame_shard(frames, rank, world):
    """Frames [f0, f1) of rank `rank` when one clip's `frames` latent frames are
    split over `world` ranks: contiguous ranges, the first (frames mod world)
    ranks taking one frame more.  A rank may get no frame (f0 == f1) when there
    are more ranks than frames."""
    if world < 1 or not 0 <= rank < world or frames < 0:
        raise ValueError("need 0 <= rank < world and frames >= 0")
    base, extra = divmod(frames, world)
    f0 = rank * base + min(rank, extra)
    return f0, f0 + base + (1 if rank < extra else 0)


def clip_shard(frames, channels, height, width, rank, world):
    """Rank `rank`'s part of one clip split by latent frames:
    ((token0, token1), (elem0, elem1)) -- its tokens (one per latent cell,
    frame-major) and its range of the flat [F, C, H, W] latent.  elem0 is the
    noise offset of its re-noise: the Philox block of an element is its global
    index / 4, and elem0 is a multiple of 4 because C H W is."""
    if (channels * height * width) % 4:
        raise ValueError("C H W must be a multiple of 4 (one Philox block)")
    f0, f1 = frame_shard(frames, rank, world)
    cells = height * width
    return (f0 * cells, f1 * cells), (f0 * channels * cells, f1 * channels * cells)


def whole_job_rate(units_per_rank, world, steps, max_ms):
    """Units per second over all ranks: every rank's units divided by the
    slowest rank's time."""
    return world * units_per_rank * steps / (max_ms * 1e-3)


def destroy(world):
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
