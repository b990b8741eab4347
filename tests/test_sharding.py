"""Multi-process (gloo, world size 2, CPU) coverage of the data-parallel path: the packed batch is
cut at image boundaries, each rank quantizes its rows (oracle on CPU), and the gathered ids equal
the single-process result; the max-over-ranks timing reduction works."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from multimodal_visual_tokenization_b200 import sharding


def test_partition_rows_cuts_at_boundaries():
    off = [0, 10, 10, 25, 40, 41, 100]
    for world in (1, 2, 3, 4, 8):
        parts = sharding.partition_rows(off, world)
        assert parts[0][0] == 0 and parts[-1][1] == 100
        for (a, b), (c, _) in zip(parts, parts[1:]):
            assert b == c and a <= b
        for a, b in parts:
            assert a in off and b in off
    # balanced: each cut is the boundary nearest the even split
    assert sharding.partition_rows([0, 30, 50, 70, 100], 2) == [(0, 50), (50, 100)]
    with pytest.raises(ValueError):
        sharding.partition_rows([1, 5], 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, x, C, offsets, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        a, b = sharding.partition_rows(offsets, world)[rank]
        ids, _, _, _ = oracle.encode(x[a:b], C, threads=1)
        sizes = [None] * world
        dist.all_gather_object(sizes, (a, b))
        gathered = [None] * world
        dist.all_gather_object(gathered, ids)
        t = sharding.max_over_ranks(float(rank + 1))
        if rank == 0:
            out_q.put((sizes, np.concatenate(gathered), t))
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_quantization_matches_single_process():
    import oracle
    rng = np.random.Generator(np.random.PCG64(5))
    C = rng.standard_normal((2, 32, 16)).astype(np.float32)
    sizes = rng.integers(3, 12, size=9)
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    x = rng.standard_normal((int(offsets[-1]), 16)).astype(np.float32)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, x, C, offsets, q)) for r in range(2)]
    for p in procs:
        p.start()
    ranges, ids, tmax = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    want, _, _, _ = oracle.encode(x, C)
    assert np.array_equal(ids, want)
    assert ranges[0][1] == ranges[1][0] and ranges[0][1] in offsets
    assert tmax == 2.0


def test_max_over_ranks_without_group_is_identity():
    assert sharding.max_over_ranks(3.5) == 3.5
