"""The multi-rank host path on CPU: two gloo ranks, no GPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import synth
from fp4_post_weight_b200 import dist as D


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w, r, _ = D.env()
        assert (w, r) == (world, rank)
        D.barrier()
        t = D.max_over_ranks(10.0 + rank * 3.5)
        lo = D.min_over_ranks(10.0 + rank * 3.5)
        assert lo == 10.0                          # the size every rank can afford
        # each rank's model is seeded apart from the others'
        seeds = [D.seed_base(r) + j for j in range(224)]
        g = synth.llama_8b_tensor(0, (16, 64), "cpu", seed_base=D.seed_base(r))
        first = float(g.W.float()[0, 0])
        all_first = [None] * world
        dist.all_gather_object(all_first, first)
        owned = D.shard([o * i for _, (o, i) in synth.LLAMA_8B.tensors()], world, rank)
        all_owned = [None] * world
        dist.all_gather_object(all_owned, owned)
        # one tensor split by rows: each rank's s2 of its rows, then the max over
        # ranks, is the s2 of the whole tensor (the oracle's, on the full tensor)
        import numpy as np
        import oracle
        for out in (37, 1):                          # with one row, rank 1 owns none
            W = synth.llama_1b_tensor(5, (out, 64), "cpu").W
            r0, r1 = D.row_shard(out, world, rank)
            bits = W.view(torch.int16).numpy().view(np.uint16)
            local = oracle.s2(bits[r0:r1]) if r1 > r0 else np.float32(0)
            s2 = D.s2_across_ranks(torch.tensor([float(local)], dtype=torch.float32))
            assert float(s2.item()) == float(oracle.s2(bits)), (out, rank)
        q.put((rank, t, seeds[0], all_first, all_owned))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    res.sort()
    assert all(t == 13.5 for _, t, _, _, _ in res)          # max over ranks
    assert res[0][2] != res[1][2]
    firsts = res[0][3]
    assert firsts[0] != firsts[1]                             # distinct models per rank
    owned = res[0][4]
    n = len(synth.LLAMA_8B.tensors())
    assert sorted(owned[0] + owned[1]) == list(range(n))      # every tensor owned once
    sizes = [o * i for _, (o, i) in synth.LLAMA_8B.tensors()]
    l0, l1 = sum(sizes[i] for i in owned[0]), sum(sizes[i] for i in owned[1])
    assert abs(l0 - l1) <= max(sizes)


def test_single_process_defaults():
    assert D.max_over_ranks(3.0) == 3.0
    assert D.min_over_ranks(3.0) == 3.0
    D.barrier()
    assert D.shard([5, 1, 1], 1, 0) == [0, 1, 2]
    # row shards: contiguous, covering, sizes within one
    for out, world in ((37, 2), (1, 2), (10, 4), (0, 3)):
        spans = [D.row_shard(out, world, r) for r in range(world)]
        assert spans[0][0] == 0 and spans[-1][1] == out
        assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
        sizes = [b - a for a, b in spans]
        assert max(sizes) - min(sizes) <= 1
    s2 = torch.tensor([0.25])
    assert D.s2_across_ranks(s2) is s2 and float(s2) == 0.25
