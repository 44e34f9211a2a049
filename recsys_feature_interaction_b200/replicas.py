"""Data-parallel replicas of the Wukong stack forward, one process per GPU.

Examples are independent and the weights are read-only, so the forward shards by
example with no collective on the data path: rank r runs the full stack on its own
contiguous block of examples. The only communication is host-side bookkeeping --
a barrier around the timed region and the maximum of the ranks' times -- done with
torch.distributed (NCCL on GPUs, gloo in CPU tests).
"""
import datetime
import os


def rank_info():
    """(rank, world_size, local_rank) from the launcher's environment (defaults: 0, 1, 0)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def example_range(rank, world, per_rank):
    """Weak scaling: rank r owns examples [r * per_rank, (r + 1) * per_rank)."""
    if not (0 <= rank < world) or per_rank < 0:
        raise ValueError("bad rank / world / per_rank")
    return rank * per_rank, (rank + 1) * per_rank


def split_range(rank, world, total):
    """Strong scaling: contiguous, balanced blocks of `total` examples (the first
    total % world ranks take one more)."""
    if not (0 <= rank < world) or total < 0:
        raise ValueError("bad rank / world / total")
    base, extra = divmod(total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def init(backend, device=None, timeout_s=300):
    """Initialises the default process group when more than one rank runs; returns
    (rank, world). A short timeout makes ranks that wait on a missing peer fail
    instead of hanging."""
    import torch.distributed as dist

    rank, world, _ = rank_info()
    if world > 1 and not dist.is_initialized():
        kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
        if device is not None:
            kw["device_id"] = device
        dist.init_process_group(backend, **kw)
    return rank, world


def barrier():
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def max_over_ranks(value, device=None):
    """The maximum of a float over all ranks (every rank gets it)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def finish():
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        if dist.get_world_size() > 1:
            dist.barrier()
        dist.destroy_process_group()
