"""Host logic of the codebook-sharded encode, on CPU: the shard split and the exchange of the
per-rank (distance, id) arrays between two gloo ranks."""
import os
import socket
import types

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from multimodal_visual_tokenization_b200.sharded import ShardedTokenizer, shard_offsets, split_codebook


@pytest.mark.parametrize("K", [1, 5, 33, 255, 256, 257, 1000, 8192, 16384, 65536, 65537])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 7, 8, 16])
def test_split_codebook(K, world):
    if K < world:
        with pytest.raises(ValueError):
            split_codebook(K, world)
        return
    sizes = split_codebook(K, world)
    assert len(sizes) == world and sum(sizes) == K and min(sizes) >= 1
    head = sizes[:-1]
    whole_tiles = all(s % 256 == 0 for s in head) and (not head or max(head) - min(head) <= 256)
    even = max(sizes) - min(sizes) <= 1
    assert whole_tiles or even, sizes
    if -(-K // 256) >= world + 1:       # enough tiles: whole tiles on every rank but the last
        assert whole_tiles and sizes[-1] <= max(sizes), sizes
    offs = shard_offsets(sizes)
    assert offs[0] == 0 and all(b - a == s for a, b, s in zip(offs, offs[1:], sizes))


def test_split_codebook_whole_tiles():
    assert split_codebook(8192, 4) == [2048] * 4
    assert split_codebook(1000, 4) == [256, 256, 256, 232]
    assert split_codebook(300, 2) == [256, 44]
    assert split_codebook(5, 5) == [1] * 5
    assert split_codebook(300, 4) == [75] * 4        # fewer tiles than ranks: even split


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _exchange_worker(rank, world, port, N, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        shard = types.SimpleNamespace(L=2, D=64, cb_dtype=0, codebooks=torch.empty(1))
        tok = ShardedTokenizer([shard], [5] * world, [0] * world, rank=rank)
        sel = torch.full((world, N, 2), -1.0, dtype=torch.float64)
        rng = np.random.Generator(np.random.PCG64(rank))
        sel[rank] = torch.from_numpy(rng.standard_normal((N, 2)))
        tok._exchange(sel)
        out_q.put((rank, sel.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_exchange_gives_every_rank_all_blocks(world):
    N = 37
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    mp.start_processes(_exchange_worker, args=(world, _free_port(), N, q), nprocs=world, join=True,
                       start_method="spawn")
    got = dict(q.get() for _ in range(world))
    want = np.stack([np.random.Generator(np.random.PCG64(r)).standard_normal((N, 2)) for r in range(world)])
    for r in range(world):
        assert np.array_equal(got[r], want), f"rank {r} missing blocks"
