"""Host-side plumbing for several GPUs, one process per GPU.

The quantizer's work is element-parallel: every 16-block is independent and
s2 is frozen per tensor, so ranks never exchange data on the hot path.  Each
rank steps its own set of tensors (weak scaling: a whole model per GPU, seeded
by rank, or one model's tensors split by `shard`); the only collectives are
the timing reduction and barriers, over whatever process group is initialised
(NCCL on GPUs, gloo in CPU tests).  A tensor split by rows (`row_shard`) needs
one 4-byte all-reduce for its s2 (`s2_across_ranks`), once.
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


def row_shard(out: int, world: int, rank: int):
    """Rows [r0, r1) of a tensor with `out` rows that rank `rank` owns when one
    tensor is split by rows over `world` GPUs (contiguous, sizes differing by at
    most one; a rank may own none)."""
    base, extra = divmod(int(out), int(world))
    r0 = rank * base + min(rank, extra)
    return r0, r0 + base + (1 if rank < extra else 0)


def s2_across_ranks(s2: torch.Tensor) -> torch.Tensor:
    """The tensor scale of a tensor split by rows: every rank passes the s2 of
    its own rows (focus_s2 on its shard; 0 for an empty shard) and receives, in
    place, their maximum, which is the s2 of the whole tensor: s2 = fl(A/2688)
    is monotonic in A, so the max of the shards' fl(A_r/2688) is fl(max_r A_r /
    2688).  One 4-byte all-reduce, once (s2 is frozen)."""
    d = _dist()
    if d is not None and d.get_world_size() > 1:
        d.all_reduce(s2, op=d.ReduceOp.MAX)
    return s2


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
