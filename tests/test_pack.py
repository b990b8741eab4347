"""Packing pretokenized image sequences for data-parallel ranks.

CPU: the library's host balance (rvq_balance_sequences) assigns exactly like the pinned oracle.
GPU: the id-cache gather (rvq_gather_sequences) packs exactly numpy's concatenation of the cached
rows, and flags bad selections through the status word.
"""
import numpy as np
import pytest

import multimodal_visual_tokenization_b200 as mvt
import oracle
import workloads


def test_balance_equals_oracle():
    rng = np.random.Generator(np.random.PCG64(41))
    for _ in range(300):
        S = int(rng.integers(0, 400))
        world = int(rng.integers(1, 17))
        lengths = rng.integers(0, 9217, size=S)
        code, owner, load = mvt.rvq_balance_sequences(lengths, world)
        want_owner, want_load = oracle.balance(lengths, world)
        assert code == 0
        assert np.array_equal(owner, want_owner) and np.array_equal(load, want_load)


def test_balance_of_the_packed_batch():
    g = workloads.generate("packed")
    lengths = np.diff(g["offsets"])
    for world in (2, 4, 8):
        code, owner, load = mvt.rvq_balance_sequences(lengths, world)
        assert code == 0 and load.sum() == lengths.sum()
        # longest-first bound against the trivial lower bound max(mean, longest)
        lb = max(lengths.sum() / world, lengths.max())
        assert load.max() <= (4.0 / 3.0) * lb + 1, (world, load, lb)


def test_balance_argument_checks():
    assert mvt.rvq_balance_sequences([3, -1], 2)[0] == -1
    assert mvt.rvq_balance_sequences([3, 1], 0)[0] == -1


torch = pytest.importorskip("torch")


def _gather(cache, offsets, select, out_offsets):
    L = cache.shape[1]
    dev = torch.device("cuda")
    ct = torch.from_numpy(np.ascontiguousarray(cache, np.int32)).to(dev)
    co = torch.from_numpy(np.ascontiguousarray(offsets, np.int64)).to(dev)
    se = torch.from_numpy(np.ascontiguousarray(select, np.int64)).to(dev)
    oo = torch.from_numpy(np.ascontiguousarray(out_offsets, np.int64)).to(dev)
    out = torch.full((int(out_offsets[-1]), L), -7, dtype=torch.int32, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    assert mvt.rvq_gather_sequences(ct, L, co, len(offsets) - 1, se, len(select), oo, out, st) == 0
    torch.cuda.synchronize()
    return out.cpu().numpy(), int(st.item())


@pytest.mark.gpu
@pytest.mark.parametrize("L", [8, 3])   # 3: rows not 16-byte multiples, 4-byte copies
def test_gather_matches_concatenation(L):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    rng = np.random.Generator(np.random.PCG64(42 + L))
    lengths = rng.integers(0, 700, size=90)
    offsets = np.concatenate([[0], np.cumsum(lengths)])
    cache = rng.integers(0, 16384, size=(offsets[-1], L)).astype(np.int32)
    code, owner, load = mvt.rvq_balance_sequences(lengths, 4)
    select = np.nonzero(owner == 1)[0]
    out_offsets = np.concatenate([[0], np.cumsum(lengths[select])])
    got, st = _gather(cache, offsets, select, out_offsets)
    want = np.concatenate([cache[offsets[s]:offsets[s + 1]] for s in select]) if len(select) else np.zeros((0, L))
    assert st == 0 and np.array_equal(got, want)


@pytest.mark.gpu
def test_gather_flags_bad_selection():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    cache = np.arange(40, dtype=np.int32).reshape(20, 2)
    offsets = np.array([0, 5, 12, 20])
    got, st = _gather(cache, offsets, np.array([2, 7]), np.array([0, 8, 10]))
    assert st == -1
    assert np.array_equal(got[:8], cache[12:20])           # the valid sequence is still packed
    got, st = _gather(cache, offsets, np.array([0]), np.array([0, 4]))   # span differs from the cache
    assert st == -1
