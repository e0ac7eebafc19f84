"""Data-parallel plumbing for running N replicas of the streamed step (one
process per GPU, torch.distributed for the process group and host-side
exchanges).  Each rank streams its own copy of the frozen stack on its own
micro-batch; the only exchange is the average of the LoRA gradients before the
(identical) AdamW update on every rank, which the library performs inside the
step (stream_stack_reduce_grads; average_ is the same mean written with
torch.distributed, used by the CPU tests).  Timing is the maximum over ranks.
"""
import datetime
import os

import torch
import torch.distributed as dist


def env():
    """(rank, world_size, local_rank) from the launcher's environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend, timeout_s=300, device=None):
    """Initialise the default process group if the job has more than one rank."""
    rank, world, _ = env()
    if world > 1 and not dist.is_initialized():
        kw = dict(timeout=datetime.timedelta(seconds=timeout_s))
        if device is not None:
            kw["device_id"] = device
        dist.init_process_group(backend, **kw)
    return rank, world


def average_(t):
    """In-place mean over ranks (sum then divide, valid for every backend)."""
    if dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
        t.div_(dist.get_world_size())
    return t


def max_over_ranks(x, device):
    """Maximum of a host float over ranks."""
    if not (dist.is_initialized() and dist.get_world_size() > 1):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    if dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def token_seed(base, rank):
    """Each rank draws its own micro-batches."""
    return base + 1000 * rank


def broadcast_bytes(make, src=0):
    """The bytes `make()` returns on rank `src`, delivered to every rank (host channel)."""
    multi = dist.is_initialized() and dist.get_world_size() > 1
    obj = [make() if (not multi or dist.get_rank() == src) else None]
    if multi:
        dist.broadcast_object_list(obj, src=src)
    return obj[0]


def reduce_grads_stack(L, stack):
    """stream_stack_reduce_grads over this job's ranks: every later step of the stack
    averages its LoRA gradients over the ranks itself, layer by layer, overlapping
    the backward, before its optimiser update."""
    rank, world = ((dist.get_rank(), dist.get_world_size()) if dist.is_initialized() else (0, 1))
    stack.reduce_grads(broadcast_bytes(L.lsq_nccl_unique_id), world, rank)


def shard_stack(L, stack, buf_bytes):
    """stream_stack_shard over this job's ranks: rank 0 makes the NCCL id, every
    rank joins with its own rank.  Each layer copy is then split over the ranks
    and reassembled by an all-gather on the GPUs."""
    rank, world = ((dist.get_rank(), dist.get_world_size()) if dist.is_initialized() else (0, 1))
    stack.shard(broadcast_bytes(L.lsq_nccl_unique_id), world, rank, buf_bytes)

