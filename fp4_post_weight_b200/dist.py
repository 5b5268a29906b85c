"""Host-side plumbing for several GPUs, one process per GPU.

The quantizer's work is element-parallel: every 16-block is independent and
s2 is frozen per tensor, so ranks never exchange data on the hot path.  Each
rank steps its own set of tensors (weak scaling: a whole model per GPU, seeded
by rank); the only collectives are the timing reduction and barriers, over
whatever process group is initialised (NCCL on GPUs, gloo in CPU tests).
"""
from __future__ import annotations

import os

import torch


def env():
    """(world_size, rank, local_rank) from the launcher's environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def seed_base(rank: int, base: int = 2) -> int:
    """Seed offset of a rank's model: disjoint from every other rank's tensors
    (each model draws at most 1000 per-tensor seeds)."""
    return base + 1000 * int(rank)


def _dist():
    import torch.distributed as dist
    return dist if dist.is_available() and dist.is_initialized() else None


def barrier() -> None:
    d = _dist()
    if d is not None:
        d.barrier()


def max_over_ranks(x: float) -> float:
    """The max of a per-rank number (a device-timed duration) over all ranks."""
    d = _dist()
    if d is None or d.get_world_size() == 1:
        return float(x)
    dev = torch.device("cuda", torch.cuda.current_device()) if d.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    d.all_reduce(t, op=d.ReduceOp.MAX)
    return float(t.item())


def min_over_ranks(x: float) -> float:
    """The min of a per-rank number over all ranks (a size every rank can afford)."""
    d = _dist()
    if d is None or d.get_world_size() == 1:
        return float(x)
    dev = torch.device("cuda", torch.cuda.current_device()) if d.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    d.all_reduce(t, op=d.ReduceOp.MIN)
    return float(t.item())


def shard(sizes, world: int, rank: int):
    """Indices of the tensors rank `rank` owns when one model is split over
    `world` GPUs: greedy by size (largest first onto the least loaded rank),
    deterministic, every tensor owned by exactly one rank."""
    load = [0] * world
    owner = [0] * len(sizes)
    for i in sorted(range(len(sizes)), key=lambda j: (-int(sizes[j]), j)):
        r = min(range(world), key=lambda k: (load[k], k))
        owner[i] = r
        load[r] += int(sizes[i])
    return [i for i in range(len(sizes)) if owner[i] == rank]
