"""Multi-process plumbing for the refiner hot path: one process per GPU.

The path has no exchange step.  Each rank refines its own batch (its own
latent and activations) and draws its noise from its own slice of the Philox
stream, so N ranks together compute exactly what one process would compute
over the concatenation of their batches: weak scaling with no collective on
the data path.  The only collectives are the barrier that brackets a timed
region and the max-over-ranks of its duration.

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


def whole_job_rate(units_per_rank, world, steps, max_ms):
    """Units per second over all ranks: every rank's units divided by the
    slowest rank's time."""
    return world * units_per_rank * steps / (max_ms * 1e-3)


def destroy(world):
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
