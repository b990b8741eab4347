"""Codebook-sharded encode (rvq_shard_select / exchange / rvq_shard_apply) against the fp64 oracle
and against the one-GPU encode of the whole codebook set.

`ShardedTokenizer.local` holds every shard in one process on one GPU, which runs the same kernels
as one process per GPU with the exchange reduced to a no-op.  The last test runs two processes
that share cuda:0: each holds one shard, maps the other's through CUDA IPC and exchanges over
gloo, i.e. the multi-process path without NCCL.
"""
import os
import socket

import numpy as np
import pytest

import workloads
from tests import parity

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU hosts, run only with a GPU
    pytest.skip("needs a CUDA device", allow_module_level=True)

import multimodal_visual_tokenization_b200 as mvt  # noqa: E402
from multimodal_visual_tokenization_b200.sharded import ShardedTokenizer, split_codebook  # noqa: E402


def dev(a, dtype):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype == "bf16":
        t = t.to(torch.bfloat16)
    return t.cuda()


def run_sharded(x, C, world, fd="f32", cd="f32", sizes=None):
    Cd = dev(C, cd)
    tok = ShardedTokenizer.local(Cd, world, sizes=sizes)
    ids, res, fb = tok.encode(dev(x, fd), residual=True)
    rec = mvt.Tokenizer(Cd).decode(ids)
    torch.cuda.synchronize()
    return ids.cpu().numpy(), res.cpu().numpy(), rec.cpu().numpy(), fb.cpu().numpy()


def one_gpu_ids(x, C, fd="f32", cd="f32"):
    ids, _, _ = mvt.Tokenizer(dev(C, cd)).encode(dev(x, fd))
    torch.cuda.synchronize()
    return ids.cpu().numpy()


def check(x, C, ids, res, rec, rows=None):
    rows = np.arange(x.shape[0]) if rows is None else rows
    rep = parity.check_ids(x, C, rows, ids)
    rep.update(parity.check_recon(x, C, rows, ids, rec, res))
    parity.check_all_rows(x, ids, C.shape[1], rec, res)
    return rep


CASES = [
    # N, D, L, K, world, f_dtype, cb_dtype
    (1000, 256, 3, 1000, 4, "f32", "f32"),     # ragged last shard (256, 256, 256, 232), ragged N
    (777, 128, 2, 700, 3, "bf16", "f32"),
    (129, 1024, 3, 600, 2, "bf16", "bf16"),    # two row tiles, shards of 512 and 88
    (1, 64, 2, 40, 5, "f32", "f32"),           # one row, shards of 8 codewords
    (300, 512, 4, 2048, 16, "f32", "bf16"),    # the maximum 16 shards
    (4100, 64, 2, 33, 2, "f32", "f32"),
    (500, 192, 3, 3000, 1, "f32", "f32"),      # one shard: the split reduces to the plain encode
]


@pytest.mark.parametrize("N,D,L,K,world,fd,cd", CASES)
def test_sharded_matches_oracle_and_one_gpu(N, D, L, K, world, fd, cd):
    rng = np.random.Generator(np.random.PCG64([N, D, L, K, world]))
    scale = 0.5 ** np.arange(L).astype(np.float32)
    C = rng.standard_normal((L, K, D)).astype(np.float32) * scale[:, None, None]
    x = rng.standard_normal((N, D)).astype(np.float32)
    if cd == "bf16":
        C = workloads.round_bf16(C)
    if fd == "bf16":
        x = workloads.round_bf16(x)
    ids, res, rec, fb = run_sharded(x, C, world, fd, cd)
    check(x, C, ids, res, rec)
    assert np.array_equal(ids, one_gpu_ids(x, C, fd, cd))


@pytest.mark.parametrize("world", [2, 4])
def test_image_workload_sharded(world):
    g = workloads.generate("image")
    x, C = g["x"], g["codebooks"]
    ids, res, rec, fb = run_sharded(x, C, world, "bf16", "f32")
    assert np.array_equal(ids, one_gpu_ids(x, C, "bf16", "f32"))     # every row
    rows = workloads.sample_rows(len(x), 64, seed=7)
    check(x, C, ids, res, rec, rows)
    assert (ids[:, 0] == g["planted"][:, 0]).all()
    print("image sharded", world, "fallbacks", fb.sum(axis=0).tolist())


def test_duplicates_across_shards_go_to_the_lowest_id():
    """Every codeword of shard 0 repeats in shard 1: the two exact distances are bit-identical, so
    each row must take the shard-0 copy (lowest id), also for rows equal to a codeword (d = 0)."""
    rng = np.random.Generator(np.random.PCG64(31))
    base = rng.standard_normal((64, 128)).astype(np.float32)
    C = np.stack([np.concatenate([base, base]), 0.1 * np.concatenate([base, base])])
    pick = rng.integers(0, 64, size=400)
    x = base[pick] + np.where(np.arange(400)[:, None] < 100, 0.0, 0.01) * rng.standard_normal((400, 128))
    x = x.astype(np.float32)
    ids, res, rec, fb = run_sharded(x, C, 2, sizes=[64, 64])
    assert (ids < 64).all(), "equal codewords in two shards must resolve to the lower id"
    assert (ids[:100, 0] == pick[:100]).all()
    check(x, C, ids, res, rec)


def test_near_ties_take_the_exact_shard_scan():
    """Groups of 16 codewords 1e-7..1e-4 apart (relative) spread over two shards overflow the
    candidate lists: the rows fail the certificate and get the exact scan of each shard."""
    rng = np.random.Generator(np.random.PCG64(39))
    D, G, copies, N = 256, 32, 16, 400
    base = rng.standard_normal((G, D)).astype(np.float32)
    eps = (10.0 ** rng.uniform(-7, -4, size=(copies, G, 1))).astype(np.float32)
    eps[0] = 0.0
    C = (base[None] * (1 + eps)).reshape(1, copies * G, D)
    x = base[rng.integers(0, G, size=N)] + 1e-3 * rng.standard_normal((N, D)).astype(np.float32)
    ids, res, rec, fb = run_sharded(x, C, 2)
    rep = check(x, C, ids, res, rec)
    print("sharded near ties", rep, "fallbacks", fb.tolist())
    assert fb.sum() > 0


def test_empty_batch_and_argument_errors():
    C = torch.randn(2, 64, 64, device="cuda")
    tok = ShardedTokenizer.local(C, 2)
    ids, res, fb = tok.encode(torch.empty((0, 64), device="cuda"))
    assert ids.shape == (0, 2)
    with pytest.raises(ValueError):
        ShardedTokenizer.local(C, 2, sizes=[10, 10])
    with pytest.raises(ValueError):
        ShardedTokenizer.local(torch.randn(1, 64, 64, device="cuda"), 17)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _ipc_worker(rank, world, port, x, C, out_dir):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    torch.cuda.set_device(0)
    try:
        sizes = split_codebook(C.shape[1], world)
        k0 = sum(sizes[:rank])
        shard = torch.from_numpy(np.ascontiguousarray(C[:, k0:k0 + sizes[rank]])).cuda()
        tok = ShardedTokenizer.from_group(shard)
        ids, res, fb = tok.encode(torch.from_numpy(x).cuda(), residual=True)
        torch.cuda.synchronize()
        np.save(os.path.join(out_dir, f"ids{rank}.npy"), ids.cpu().numpy())
        np.save(os.path.join(out_dir, f"res{rank}.npy"), res.cpu().numpy())
        tok.close()
    finally:
        dist.destroy_process_group()


def test_two_processes_share_shards_through_ipc(tmp_path):
    import torch.multiprocessing as mp
    rng = np.random.Generator(np.random.PCG64(41))
    L, K, D, N = 3, 1500, 256, 700
    C = (rng.standard_normal((L, K, D)) * (0.5 ** np.arange(L))[:, None, None]).astype(np.float32)
    x = rng.standard_normal((N, D)).astype(np.float32)
    mp.start_processes(_ipc_worker, args=(2, _free_port(), x, C, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    ids = [np.load(tmp_path / f"ids{r}.npy") for r in range(2)]
    res = [np.load(tmp_path / f"res{r}.npy") for r in range(2)]
    assert np.array_equal(ids[0], ids[1]) and np.array_equal(res[0], res[1]), "replicas diverged"
    rec = mvt.Tokenizer(dev(C, "f32")).decode(torch.from_numpy(ids[0]).cuda()).cpu().numpy()
    check(x, C, ids[0], res[0], rec)
    assert np.array_equal(ids[0], one_gpu_ids(x, C))
