"""bench.py's replica bookkeeping on two gloo ranks (CPU): each rank times a stub step over its
share of a packed batch (cut at image boundaries by sharding.partition_rows); replica_measure must
report the slowest rank's time on every rank and the rows of all ranks per second."""
import os
import socket
import time

import numpy as np
import torch.distributed as dist
import torch.multiprocessing as mp

from multimodal_visual_tokenization_b200 import sharding


class WallTimer:
    """perf_counter stand-in for the CUDA-event timer."""

    def __init__(self, steps):
        self.t = [[0.0, 0.0] for _ in range(steps)]

    def start(self, k):
        self.t[k][0] = time.perf_counter()

    def stop(self, k):
        self.t[k][1] = time.perf_counter()

    def total_ms(self):
        return sum(b - a for a, b in self.t) * 1e3


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, offsets, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        a, b = sharding.partition_rows(offsets, world)[rank]
        rows = b - a
        calls = {"between": 0}

        def step():  # a replica's step: time proportional to its rows, rank 1 slower per row
            time.sleep(rows * (1 + rank) * 2e-5)

        def between():
            calls["between"] += 1

        steps = 4
        ms, value, total = bench.replica_measure(step, steps, WallTimer(steps), rows, between=between)
        out_q.put((rank, (a, b), ms, value, total, calls["between"]))
    finally:
        dist.destroy_process_group()


def test_replica_measure_takes_the_slowest_rank_and_all_rows():
    rng = np.random.Generator(np.random.PCG64(3))
    sizes = rng.integers(20, 200, size=16)
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, offsets, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, (a0, b0), ms0, v0, t0, n0), (r1, (a1, b1), ms1, v1, t1, n1) = res
    assert (a0, b1) == (0, int(offsets[-1])) and b0 == a1 and b0 in offsets   # cut at an image boundary
    assert ms0 == ms1 and v0 == v1 and t0 == t1                                # one answer on every rank
    slow = (b1 - a1) * 2 * 2e-5 * 1e3                                          # rank 1's sleep per step, ms
    assert ms0 >= slow * 0.99 and ms0 < slow + 50.0
    assert abs(v0 - offsets[-1] / (ms0 / 1e3)) <= 1e-9 * v0                   # all ranks' rows per second
    assert n0 == n1 == 4


def test_replica_measure_without_group():
    import bench
    calls = []
    ms, value, total = bench.replica_measure(lambda: calls.append(1), 3, WallTimer(3), 100)
    assert len(calls) == 3 and total >= 0 and abs(ms - total / 3) < 1e-12
    assert value == 100 / (ms / 1e3) if ms > 0 else True
