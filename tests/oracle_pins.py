"""Pins that tie the fp64 oracle to facts other than itself.

Each pin takes a loaded oracle library (the real one, or a deliberately broken
build made by the mutation test) and raises AssertionError when the oracle
disagrees with:
  * brute force over all K^L code combinations (greedy = lexicographic minimiser
    of (d_0, id_0, d_1, id_1, ...)),
  * a library nearest-neighbour search (scipy cdist + argmin) when L = 1,
  * closed forms (K = 1; codebook = the features; planted codewords with a wide
    margin; integer-valued decode),
  * invariants (recon + residual == x; residual norms never grow when every level
    holds a zero codeword; exact ties go to the lowest index),
  * the hand-worked example in tests/golden/rvq_toy_2d.txt,
and the gradient of the embedding e[n] = sum_l E_l[ids[n,l]] (the decode gather-sum with
learned tables) with:
  * the adjoint identity <decode(ids, E), G> = <E, backward(ids, G)> (decode pinned above),
  * a permutation of ids per level (each gradient row is one input row, exactly),
  * numpy's unbuffered scatter-add (np.add.at) on small inputs,
  * column sums (every input row lands in exactly one row per level) and the magnitude bounds,
and the k-means update of one codebook level with:
  * points that are their own clusters (the codebook becomes the points, exactly),
  * one cluster holding every point (numpy's mean),
  * the Lloyd property: for fixed assignments the update never increases the squared error,
  * numpy group-by means (bincount + add.at), empty clusters keeping their codeword,
and the balance of sequences across data-parallel ranks with:
  * brute force over all assignments on tiny inputs (Graham's bound for the longest-first rule:
    max load <= (4/3 - 1/(3 world)) x the optimum, and never below it),
  * the hand-worked example in tests/golden/lpt_balance.txt,
  * invariants (every sequence owned once, loads add up, equal lengths split evenly).
"""
from __future__ import annotations

import itertools
import os

import numpy as np
from scipy.spatial.distance import cdist

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def brute_force_greedy(x, C):
    """All K^L combinations; returns the lexicographic minimiser of (d_0,id_0,d_1,id_1,...)."""
    x = np.asarray(x, np.float64)
    C = np.asarray(C, np.float64)
    L, K, D = C.shape
    out = np.empty((x.shape[0], L), np.int32)
    for n in range(x.shape[0]):
        best_key = None
        for combo in itertools.product(range(K), repeat=L):
            r = x[n].copy()
            key = []
            for l, k in enumerate(combo):
                diff = r - C[l, k]
                key += [float(np.dot(diff, diff)), k]
                r = diff
            key = tuple(key)
            if best_key is None or key < best_key:
                best_key, best = key, combo
        out[n] = best
    return out


def pin_bruteforce(lib):
    for seed, (N, D, L, K) in enumerate([(24, 3, 2, 5), (16, 8, 3, 4), (32, 2, 2, 8), (8, 5, 3, 7)]):
        rng = _rng(100 + seed)
        C = rng.standard_normal((L, K, D)).astype(np.float32)
        C *= (0.6 ** np.arange(L, dtype=np.float32))[:, None, None]
        x = rng.standard_normal((N, D)).astype(np.float32)
        ids, _, _, _ = oracle.encode(x, C, lib=lib)
        ref = brute_force_greedy(x, C)
        assert np.array_equal(ids, ref), f"brute force mismatch (case {seed})"


def pin_nearest_neighbour_L1(lib):
    rng = _rng(7)
    for N, D, K in [(200, 16, 64), (64, 1, 33), (50, 130, 9)]:
        C = rng.standard_normal((1, K, D)).astype(np.float32)
        x = rng.standard_normal((N, D)).astype(np.float32)
        ids, res, rec, dist = oracle.encode(x, C, lib=lib)
        dm = cdist(x.astype(np.float64), C[0].astype(np.float64), "sqeuclidean")
        assert np.array_equal(ids[:, 0], np.argmin(dm, axis=1)), "L=1 is not plain nearest neighbour"
        assert np.allclose(dist[:, 0], dm.min(axis=1), rtol=1e-12, atol=1e-12)
        assert np.allclose(rec, C[0][ids[:, 0]], rtol=0, atol=0)


def pin_single_codeword(lib):
    rng = _rng(8)
    C = rng.standard_normal((3, 1, 6)).astype(np.float32)
    x = rng.standard_normal((10, 6)).astype(np.float32)
    ids, res, rec, dist = oracle.encode(x, C, lib=lib)
    assert (ids == 0).all()
    expect_res = x.astype(np.float64) - C[0, 0] - C[1, 0] - C[2, 0]
    assert np.allclose(res, expect_res, rtol=1e-15, atol=1e-15)
    assert np.allclose(rec, C[:, 0].astype(np.float64).sum(0), rtol=1e-15, atol=1e-15)


def pin_codebook_equals_features(lib):
    rng = _rng(9)
    x = rng.standard_normal((40, 12)).astype(np.float32)
    perm = rng.permutation(40)
    C = x[perm][None]                     # codeword perm^-1(n) is row n exactly
    ids, res, rec, dist = oracle.encode(x, C, lib=lib)
    inv = np.argsort(perm)
    assert np.array_equal(ids[:, 0], inv)
    assert (dist == 0).all() and (res == 0).all()


def pin_ties_lowest_index(lib):
    rng = _rng(10)
    base = rng.standard_normal((6, 4)).astype(np.float32)
    C = np.concatenate([base, base, base])[None]        # every codeword appears 3 times
    C = C[:, rng.permutation(18)]
    x = rng.standard_normal((30, 4)).astype(np.float32)
    ids, _, _, _ = oracle.encode(x, C, lib=lib)
    for n in range(30):
        same = np.where((C[0] == C[0][ids[n, 0]]).all(axis=1))[0]
        assert ids[n, 0] == same.min(), "exact tie not broken to the lowest index"
    # an exact geometric tie: x equidistant from two distinct codewords
    C2 = np.array([[[3, 0], [-1, 0], [1, 0]]], np.float32)
    x2 = np.array([[0, 0], [2, 0]], np.float32)            # d=(9,1,1) and (1,9,1)
    ids2, _, _, _ = oracle.encode(x2, C2, lib=lib)
    assert ids2[:, 0].tolist() == [1, 0]


def pin_invariants(lib):
    g = workloads.generate("tiny")
    x, C = g["x"], g["codebooks"]
    ids, res, rec, dist = oracle.encode(x, C, lib=lib)
    xd = x.astype(np.float64)
    err = np.abs(rec + res - xd).max() / np.abs(xd).max()
    assert err <= 1e-12, f"recon + residual != x ({err})"
    # every level has a zero codeword, so ||r_{l+1}||^2 = dist[l] <= ||r_l||^2
    prev = (xd ** 2).sum(1)
    for l in range(C.shape[0]):
        assert (dist[:, l] <= prev * (1 + 1e-15)).all(), "residual norm grew"
        prev = dist[:, l]
    assert np.allclose(dist[:, -1], (res ** 2).sum(1), rtol=1e-12)
    # the recon of the chosen ids is the decode of those ids
    assert np.allclose(oracle.decode(ids, C, lib=lib), rec, rtol=0, atol=1e-12)


def pin_planted(lib):
    # level-0 planted codeword beats any other by ~2*D*1 against noise ~2*sqrt(2*D*sum_rest)
    g = workloads.generate("image", n_override=48)
    x, C, planted = g["x"], g["codebooks"], g["planted"]
    C0 = C[:1]
    ids, _, _, _ = oracle.encode(x, C0, lib=lib)
    assert np.array_equal(ids[:, 0], planted[:, 0]), "planted level-0 codeword not recovered"
    # noiseless round trip (detok recipe, shrunk): decode then re-encode returns the ids
    rng = _rng(11)
    L, K, D = 3, 64, 96
    Cb = workloads.round_bf16(rng.standard_normal((L, K, D)).astype(np.float32)
                              * (0.5 ** np.arange(L, dtype=np.float32))[:, None, None])
    want = rng.integers(0, K, size=(40, L)).astype(np.int32)
    rec = oracle.decode(want, Cb, lib=lib).astype(np.float32)
    got, _, _, _ = oracle.encode(rec, Cb, lib=lib)
    assert np.array_equal(got, want), "round trip ids differ"


def pin_decode_integer(lib):
    rng = _rng(12)
    L, K, D, M = 4, 50, 7, 300
    C = rng.integers(-1000, 1000, size=(L, K, D)).astype(np.float32)
    ids = rng.integers(0, K, size=(M, L)).astype(np.int32)
    out = oracle.decode(ids, C, lib=lib)
    Ci = C.astype(np.int64)
    expect = np.zeros((M, D), np.int64)
    for l in range(L):
        expect += Ci[l][ids[:, l]]
    assert np.array_equal(out, expect.astype(np.float64))
    bad = ids.copy()
    bad[5, 2] = K
    try:
        oracle.decode(bad, C, lib=lib)
    except oracle.OracleError as e:
        assert e.code == -5
    else:
        raise AssertionError("out-of-range id accepted")


def load_golden():
    C = {}
    rows = []
    with open(os.path.join(GOLDEN, "rvq_toy_2d.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("C "):
                _, l, k, a, b = line.split()
                C[(int(l), int(k))] = (float(a), float(b))
            elif line.startswith("X "):
                parts = [p.split() for p in line[2:].split("|")]
                rows.append({"x": [float(v) for v in parts[0]],
                             "ids": [int(v) for v in parts[1][1:]],
                             "dist": [float(v) for v in parts[2][1:]],
                             "residual": [float(v) for v in parts[3][1:]],
                             "recon": [float(v) for v in parts[4][1:]]})
    L = 1 + max(l for l, _ in C)
    K = 1 + max(k for _, k in C)
    cb = np.zeros((L, K, 2), np.float32)
    for (l, k), v in C.items():
        cb[l, k] = v
    return cb, rows


def pin_golden(lib):
    cb, rows = load_golden()
    x = np.array([r["x"] for r in rows], np.float32)
    ids, res, rec, dist = oracle.encode(x, cb, lib=lib)
    assert ids.tolist() == [r["ids"] for r in rows]
    assert dist.tolist() == [r["dist"] for r in rows]
    assert res.tolist() == [r["residual"] for r in rows]
    assert rec.tolist() == [r["recon"] for r in rows]
    assert oracle.decode(ids, cb, lib=lib).tolist() == [r["recon"] for r in rows]


def pin_check_path(lib):
    rng = _rng(13)
    L, K, D, N = 3, 6, 4, 20
    C = rng.standard_normal((L, K, D)).astype(np.float32)
    x = rng.standard_normal((N, D)).astype(np.float32)
    ids = rng.integers(0, K, size=(N, L)).astype(np.int32)       # an arbitrary path
    rows = np.arange(N)
    out = oracle.check_path(x, C, rows, ids, lib=lib)
    for n in range(N):
        r = x[n].astype(np.float64)
        for l in range(L):
            d = ((r[None, :] - C[l].astype(np.float64)) ** 2).sum(1)
            a = int(np.argmin(d))
            assert out["argmin"][n, l] == a
            assert np.isclose(out["best"][n, l], d[a], rtol=1e-13)
            assert np.isclose(out["second"][n, l], np.min(np.delete(d, a)), rtol=1e-13)
            assert np.isclose(out["chosen"][n, l], d[ids[n, l]], rtol=1e-13)
            r = r - C[l, ids[n, l]]
    # distances() is the level-0 distance vector
    d0 = oracle.distances(x[0].astype(np.float64), C[0], lib=lib)
    assert np.allclose(d0, cdist(x[:1].astype(np.float64), C[0].astype(np.float64), "sqeuclidean")[0],
                       rtol=1e-13)


def _embed_case(seed, N, L, K, H, skew=False):
    rng = _rng(seed)
    if skew:  # a few very popular ids, as with Zipf-distributed level-0 tokens
        ids = np.minimum(rng.zipf(1.3, size=(N, L)) - 1, K - 1).astype(np.int32)
    else:
        ids = rng.integers(0, K, size=(N, L)).astype(np.int32)
    g = rng.standard_normal((N, H)).astype(np.float32)
    return ids, g


def pin_embed_adjoint(lib):
    for seed, (N, L, K, H, skew) in enumerate([(300, 3, 17, 24, False), (500, 2, 64, 8, True),
                                               (40, 5, 3, 16, False)]):
        ids, g = _embed_case(900 + seed, N, L, K, H, skew)
        E = _rng(950 + seed).standard_normal((L, K, H)).astype(np.float32)
        e = oracle.decode(ids, E, lib=lib)                       # forward (pinned separately)
        grad = oracle.embed_backward(ids, g, K, lib=lib)
        lhs = float(np.sum(e * g.astype(np.float64)))
        rhs = float(np.sum(E.astype(np.float64) * grad))
        assert abs(lhs - rhs) <= 1e-11 * (abs(lhs) + abs(rhs) + 1.0), (lhs, rhs)


def pin_embed_permutation(lib):
    rng = _rng(960)
    L, K, H = 3, 50, 12
    ids = np.stack([rng.permutation(K) for _ in range(L)], axis=1).astype(np.int32)  # N = K
    g = rng.standard_normal((K, H)).astype(np.float32)
    grad = oracle.embed_backward(ids, g, K, lib=lib)
    for l in range(L):
        assert np.array_equal(grad[l, ids[:, l]], g.astype(np.float64))


def pin_embed_add_at(lib):
    for seed, (N, L, K, H, skew) in enumerate([(200, 2, 9, 5, True), (64, 4, 31, 7, False)]):
        ids, g = _embed_case(970 + seed, N, L, K, H, skew)
        want = np.zeros((L, K, H))
        for l in range(L):
            np.add.at(want[l], ids[:, l], g.astype(np.float64))
        got = oracle.embed_backward(ids, g, K, lib=lib)
        assert np.allclose(got, want, rtol=1e-13, atol=1e-13)


def pin_embed_sums_and_bounds(lib):
    ids, g = _embed_case(980, 400, 3, 20, 9, True)
    grad, count, absum = oracle.embed_backward(ids, g, 20, bounds=True, lib=lib)
    col = g.astype(np.float64).sum(axis=0)
    for l in range(3):
        assert np.allclose(grad[l].sum(axis=0), col, rtol=1e-12, atol=1e-12)
        assert count[l].sum() == 400
        assert np.array_equal(count[l], np.bincount(ids[:, l], minlength=20))
    assert np.all(absum >= np.abs(grad) - 1e-12)
    assert np.all(grad[count == 0] == 0.0)


def pin_kmeans_own_clusters(lib):
    rng = _rng(990)
    N, D = 40, 6
    p = rng.standard_normal((N, D)).astype(np.float32)
    ids = rng.permutation(N).astype(np.int32)
    old = rng.standard_normal((N, D)).astype(np.float32)
    new, count = oracle.codebook_update(p, ids, old, lib=lib)
    assert np.array_equal(count, np.ones(N, np.int64))
    assert np.array_equal(new[ids], p.astype(np.float64))


def pin_kmeans_single_cluster(lib):
    rng = _rng(991)
    p = rng.standard_normal((500, 9)).astype(np.float32)
    old = rng.standard_normal((4, 9)).astype(np.float32)
    new, count = oracle.codebook_update(p, np.full(500, 2, np.int32), old, lib=lib)
    assert np.allclose(new[2], p.astype(np.float64).mean(axis=0), rtol=1e-13, atol=1e-15)
    assert np.array_equal(new[[0, 1, 3]], old[[0, 1, 3]].astype(np.float64))
    assert count.tolist() == [0, 0, 500, 0]


def pin_kmeans_lloyd_step(lib):
    rng = _rng(992)
    N, D, K = 2000, 5, 30
    p = rng.standard_normal((N, D)).astype(np.float32)
    old = rng.standard_normal((K, D)).astype(np.float32)
    ids, _, _, _ = oracle.encode(p, old[None], lib=lib)          # nearest codeword of each point
    ids = ids[:, 0]
    new, count = oracle.codebook_update(p, ids, old, lib=lib)
    pd = p.astype(np.float64)
    sse_old = float(((pd - old.astype(np.float64)[ids]) ** 2).sum())
    sse_new = float(((pd - new[ids]) ** 2).sum())
    assert sse_new <= sse_old * (1 + 1e-12), (sse_new, sse_old)
    # and no other codeword set does better for these assignments: perturbing one mean hurts
    k = int(np.argmax(count))
    moved = new.copy()
    moved[k] += 1e-3
    assert float(((pd - moved[ids]) ** 2).sum()) > sse_new


def pin_kmeans_groupby(lib):
    rng = _rng(993)
    N, D, K = 3000, 7, 64
    p = rng.standard_normal((N, D)).astype(np.float32)
    ids = np.minimum(rng.zipf(1.2, size=N) - 1, K - 9).astype(np.int32)   # skewed; the last 8 stay empty
    old = rng.standard_normal((K, D)).astype(np.float32)
    new, count = oracle.codebook_update(p, ids, old, lib=lib)
    c = np.bincount(ids, minlength=K)
    sums = np.zeros((K, D))
    np.add.at(sums, ids, p.astype(np.float64))
    want = np.where(c[:, None] > 0, sums / np.maximum(c, 1)[:, None], old.astype(np.float64))
    assert np.array_equal(count, c)
    assert (c == 0).any()
    assert np.allclose(new, want, rtol=1e-13, atol=1e-15)


def pin_balance_bruteforce(lib):
    rng = _rng(994)
    for _ in range(40):
        S = int(rng.integers(1, 8))
        world = int(rng.integers(1, 4))
        lengths = rng.integers(0, 50, size=S)
        owner, load = oracle.balance(lengths, world, lib=lib)
        assert owner.min() >= 0 and owner.max() < world
        assert np.array_equal(load, np.bincount(owner, weights=lengths, minlength=world).astype(np.int64))
        best = min(max(np.bincount(np.array(a), weights=lengths, minlength=world))
                   for a in itertools.product(range(world), repeat=S))
        assert best <= load.max() <= (4.0 / 3.0 - 1.0 / (3 * world)) * best + 1e-9, (lengths, world, load, best)


def pin_balance_golden(lib):
    vals = {}
    with open(os.path.join(GOLDEN, "lpt_balance.txt")) as f:
        for ln in f:
            if ln.strip() and not ln.startswith("#"):
                k, *v = ln.split()
                vals[k] = [int(t) for t in v]
    owner, load = oracle.balance(vals["lengths"], vals["world"][0], lib=lib)
    assert owner.tolist() == vals["owner"] and load.tolist() == vals["load"]


def pin_balance_invariants(lib):
    owner, load = oracle.balance(np.full(100, 37), 8, lib=lib)
    assert load.max() - load.min() <= 37 and load.sum() == 3700
    owner, load = oracle.balance(np.arange(500), 1, lib=lib)
    assert (owner == 0).all() and load.tolist() == [sum(range(500))]


ALL_PINS = [pin_bruteforce, pin_nearest_neighbour_L1, pin_single_codeword,
            pin_codebook_equals_features, pin_ties_lowest_index, pin_invariants, pin_planted,
            pin_decode_integer, pin_golden, pin_check_path, pin_embed_adjoint, pin_embed_permutation,
            pin_embed_add_at, pin_embed_sums_and_bounds, pin_kmeans_own_clusters, pin_kmeans_single_cluster,
            pin_kmeans_lloyd_step, pin_kmeans_groupby, pin_balance_bruteforce, pin_balance_golden,
            pin_balance_invariants]
