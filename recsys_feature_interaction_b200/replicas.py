"""Data-parallel replicas of the Wukong stack, one process per GPU.

Forward: examples are independent and the weights are read-only, so the forward shards by
example with no collective on the data path: rank r runs the full stack on its own
contiguous block of examples. The only communication is host-side bookkeeping -- a
barrier around the timed region and the maximum of the ranks' times -- done with
torch.distributed (NCCL on GPUs, gloo in CPU tests).

Training step: each rank differentiates its own examples, and the one exchange is the
average of the parameter gradients over the ranks. GradBuckets keeps each layer's
gradients in one flat fp32 buffer (the views the backward writes), and
average_gradients all-reduces layer l's buffer on a side stream as soon as the backward
has recorded layer l's event, so the reduction of the upper layers overlaps the backward
of the lower ones.
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


class GradBuckets:
    """Per-layer flat fp32 gradient buffers for wk_stack_backward. Layer l's Y, W_j, b_j,
    fmb_gamma, fmb_beta, W_L, out_gamma, out_beta are views into flats[l], each starting on
    a 256-byte boundary; grads[l] is the mapping wk_stack_backward takes."""

    ALIGN = 64  # floats

    def __init__(self, n, d, k, n_l, dims, layers, device=None):
        import torch

        shapes = [("Y", (n, k))] + [("W%d" % j, (dims[j + 1], dims[j])) for j in range(len(dims) - 1)] + \
                 [("b%d" % j, (dims[j + 1],)) for j in range(len(dims) - 1)] + \
                 [("fmb_gamma", (n * k,)), ("fmb_beta", (n * k,)), ("W_L", (n_l, n)), ("out_gamma", (d,)),
                  ("out_beta", (d,))]
        offs, total = [], 0
        for _, sh in shapes:
            size = 1
            for v in sh:
                size *= v
            offs.append(total)
            total += -(-size // self.ALIGN) * self.ALIGN
        self.numel = total
        self.flats, self.grads = [], []
        for _ in range(layers):
            flat = torch.zeros(total, dtype=torch.float32, device=device)
            views = {}
            for (name, sh), o in zip(shapes, offs):
                size = 1
                for v in sh:
                    size *= v
                views[name] = flat[o:o + size].view(*sh)
            m = len(dims) - 1
            g = {"Y": views["Y"], "W": [views["W%d" % j] for j in range(m)], "b": [views["b%d" % j] for j in range(m)],
                 "fmb_gamma": views["fmb_gamma"], "fmb_beta": views["fmb_beta"], "W_L": views["W_L"],
                 "out_gamma": views["out_gamma"], "out_beta": views["out_beta"]}
            self.flats.append(flat)
            self.grads.append(g)


def average_gradients(flats, layer_events=None, comm_stream=None):
    """Averages each layer's flat gradient buffer over the ranks, last layer first (the
    order the backward finishes them). With CUDA tensors, each all-reduce runs on
    comm_stream after layer l's event, and the caller's stream is made to wait for all of
    them before this returns; with CPU tensors (gloo) the reductions are synchronous. A
    single rank returns at once."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return
    world = dist.get_world_size()
    on_gpu = flats[0].is_cuda
    main = torch.cuda.current_stream(flats[0].device) if on_gpu else None
    for l in range(len(flats) - 1, -1, -1):
        if on_gpu:
            comm = comm_stream if comm_stream is not None else main
            if layer_events is not None and layer_events[l] is not None:
                comm.wait_event(layer_events[l])
            else:
                comm.wait_stream(main)
            with torch.cuda.stream(comm):
                dist.all_reduce(flats[l], op=dist.ReduceOp.SUM)
                flats[l].div_(world)
        else:
            dist.all_reduce(flats[l], op=dist.ReduceOp.SUM)
            flats[l].div_(world)
    if on_gpu and comm_stream is not None:
        main.wait_stream(comm_stream)
