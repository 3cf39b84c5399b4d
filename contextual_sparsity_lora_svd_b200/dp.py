"""Data-parallel plumbing of the sparse LoRA layer step (host side only).

The step shards by tokens: each rank takes a contiguous block of the global
batch's sequences and runs estimate -> select -> sliced forward/backward on it
alone.  Selection is contextual per batch, so each rank selects from its own
context tokens (SparseLoRA article, section 1: the active channels depend on
the input at hand).  The one exchange is a sum of the LoRA gradients over
ranks (each rank's dA/dB are sums over its tokens, so the sum is the gradient
of the global batch), done as a single all-reduce of one flat fp32 buffer;
NCCL over NVLink on GPUs, gloo in the CPU tests.  Frozen weights and their
SVD factors are identical on every rank and never move.
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def shard(batch: int, world: int, rank: int) -> tuple[int, int]:
    """(first sequence, number of sequences) of `rank`'s block of `batch`
    sequences: contiguous blocks whose sizes differ by at most one, the
    larger ones first.  Ranks beyond `batch` get an empty block."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside world {world}")
    if batch < 0:
        raise ValueError(f"negative batch {batch}")
    base, extra = divmod(batch, world)
    count = base + (1 if rank < extra else 0)
    start = rank * base + min(rank, extra)
    return start, count


def init_from_env(backend: str, timeout_s: float = 120.0) -> tuple[int, int]:
    """Join the process group the launcher describes (RANK, WORLD_SIZE,
    MASTER_ADDR, MASTER_PORT) with a bounded timeout, so that ranks waiting on
    a peer that never arrives end with an error instead of hanging.  Returns
    (rank, world); a single process without the variables is rank 0 of 1."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return rank, world


def allreduce_grads(flat: torch.Tensor, group=None) -> None:
    """In-place sum of the flat LoRA gradient buffer over the ranks of `group`
    (no-op for a single process)."""
    if not dist.is_available() or not dist.is_initialized():
        return
    if dist.get_world_size(group) == 1:
        return
    if flat.dim() != 1 or not flat.is_contiguous():
        raise ValueError("the gradient buffer must be one contiguous vector")
    dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)


def max_over_ranks(value: float, device: str | torch.device = "cpu", group=None) -> float:
    """The largest `value` over the ranks (timings are reported as the max)."""
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size(group) == 1:
        return float(value)
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
