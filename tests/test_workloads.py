"""Seeded synthetic inputs: determinism, shapes, storage types and recipe statistics."""
import numpy as np

import workloads


def test_deterministic_and_batches_differ():
    a = workloads.generate("tiny")
    b = workloads.generate("tiny")
    c = workloads.generate("tiny", batch=1)
    assert np.array_equal(a["x"], b["x"]) and np.array_equal(a["codebooks"], b["codebooks"])
    assert np.array_equal(a["codebooks"], c["codebooks"])
    assert not np.array_equal(a["x"], c["x"])


def test_tiny_recipe():
    g = workloads.generate("tiny")
    s = g["spec"]
    assert (s.N, s.D, s.L, s.K) == (256, 64, 2, 256)
    assert g["x"].shape == (256, 64) and g["codebooks"].shape == (2, 256, 64)
    assert (g["codebooks"][:, 0] == 0).all()
    std = g["codebooks"][:, 1:].reshape(2, -1).std(1)
    assert np.allclose(std, [1.0, 0.5], rtol=0.05)
    noise = g["x"] - g["codebooks"][0][g["planted"][:, 0]]
    assert abs(noise.std() - 0.3) < 0.02


def test_bf16_storage():
    g = workloads.generate("image", n_override=64)
    workloads.as_bf16_bits(g["x"])                       # raises if not representable
    bits = workloads.as_bf16_bits(g["x"])
    assert np.array_equal(workloads.bf16_bits_to_f32(bits), g["x"])
    d = workloads.generate("detok", n_override=64)
    workloads.as_bf16_bits(d["codebooks"])


def test_round_bf16_ties_to_even():
    v = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 1.0 + 2 ** -8 + 2 ** -20], np.float32)
    assert workloads.round_bf16(v).tolist() == [1.0, 1.0 + 2 ** -6, -1.0, 1.0 + 2 ** -7]


def test_packed_offsets():
    g = workloads.generate("packed", n_override=5000)
    off = g["offsets"]
    assert len(off) == 65 and off[0] == 0 and off[-1] == g["spec"].N
    assert (np.diff(off) >= 1).all()


def test_detok_zipf_skew():
    d = workloads.generate("detok", n_override=20000)
    ids = d["planted"]
    assert ids.shape == (20000, 8) and ids.min() >= 0 and ids.max() < 16384
    counts = np.bincount(ids[:, 0], minlength=16384)
    # P(rank 1) / P(rank 2) = 2^1.1
    assert counts[0] > 1.6 * counts[1] > 0
    assert counts[0] / 20000 > 0.05
    u = np.bincount(ids[:, 3], minlength=16384)
    assert u.max() < 10


def test_sample_rows_include_boundaries():
    off = np.array([0, 10, 10, 25, 40])
    rows = workloads.sample_rows(40, 5, seed=3, offsets=off)
    for r in (0, 9, 10, 24, 25, 39):
        assert r in rows
    assert len(np.unique(rows)) == len(rows)
