"""CUDA path (through the C ABI) against the fp64 oracle, element by element.

Small workloads are compared on every row; the large ones (packed, offline, the detok
re-encode) on seeded samples of LARGE_SAMPLE rows (first and last rows and every image's first
and last row included) plus properties checked on every row; the detok decode on every row.
The id rule and tolerances are in tests/parity.py.
"""
import numpy as np
import pytest

import workloads
from tests import parity

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU hosts, run only with a GPU
    pytest.skip("needs a CUDA device", allow_module_level=True)

import multimodal_visual_tokenization_b200 as mvt  # noqa: E402

LARGE_SAMPLE = 16384  # rows compared with the oracle on each large workload


def dev(a, dtype):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype == "bf16":
        t = t.to(torch.bfloat16)
    return t.cuda()


def run_encode(x, C, f_dtype="f32", cb_dtype="f32", offsets=None):
    tok = mvt.Tokenizer(dev(C, cb_dtype))
    fb = torch.zeros(C.shape[0], dtype=torch.int32, device="cuda")
    off = None if offsets is None else torch.from_numpy(offsets).cuda()
    ids, res, rec = tok.encode(dev(x, f_dtype), offsets=off, residual=True, recon=True, fallbacks=fb)
    torch.cuda.synchronize()
    return tok, ids.cpu().numpy(), res.cpu().numpy(), rec.cpu().numpy(), fb.cpu().numpy()


def full_check(x, C, ids, res, rec, rows=None):
    rows = np.arange(x.shape[0]) if rows is None else rows
    rep = parity.check_ids(x, C, rows, ids)
    rep.update(parity.check_recon(x, C, rows, ids, rec, res))
    parity.check_all_rows(x, ids, C.shape[1], rec, res)
    return rep


def test_tiny_all_rows():
    g = workloads.generate("tiny")
    _, ids, res, rec, fb = run_encode(g["x"], g["codebooks"])
    rep = full_check(g["x"], g["codebooks"], ids, res, rec)
    assert rep["exact"] == rep["row_levels"]
    assert (ids[:, 0] == g["planted"][:, 0]).all()


def test_image_sampled():
    g = workloads.generate("image")
    x, C = g["x"], g["codebooks"]
    _, ids, res, rec, fb = run_encode(x, C, "bf16", "f32")
    rows = workloads.sample_rows(len(x), 192, seed=1)
    rep = full_check(x, C, ids, res, rec, rows)
    print("image", rep, "fallbacks", fb.tolist())
    assert (ids[:, 0] == g["planted"][:, 0]).all()         # planted level 0, every row


def test_image_small_all_rows():
    g = workloads.generate("image", n_override=300)
    x, C = g["x"], g["codebooks"]
    _, ids, res, rec, fb = run_encode(x, C, "bf16", "f32")
    rep = full_check(x, C, ids, res, rec)
    assert rep["rows_equal_free_running"] == rep["rows"]


def test_packed_sampled():
    g = workloads.generate("packed")
    x, C, off = g["x"], g["codebooks"], g["offsets"]
    _, ids, res, rec, fb = run_encode(x, C, "bf16", "f32", offsets=off)
    rows = workloads.sample_rows(len(x), LARGE_SAMPLE, seed=2, offsets=off)
    assert np.isin(off[:-1], rows).all() and np.isin(off[1:] - 1, rows).all()
    rep = full_check(x, C, ids, res, rec, rows)
    print("packed", rep, "fallbacks", fb.tolist())
    assert rep["rows"] >= LARGE_SAMPLE
    assert (ids[:, 0] == g["planted"][:, 0]).all()


def test_packed_short_batch_pairs():
    """A 16352-row packed batch runs as CTA pairs with several chunks per 256-row unit (so every
    row merges several candidate lists written by a pair): sampled rows and every image boundary
    against the oracle."""
    g = workloads.generate("packed", n_override=16384)
    x, C, off = g["x"], g["codebooks"], g["offsets"]
    _, ids, res, rec, fb = run_encode(x, C, "bf16", "f32", offsets=off)
    rows = workloads.sample_rows(len(x), 4096, seed=12, offsets=off)
    rep = full_check(x, C, ids, res, rec, rows)
    print("packed short", len(x), rep, "fallbacks", fb.tolist())
    assert (ids[:, 0] == g["planted"][:, 0]).all()


def test_offline_sampled():
    g = workloads.generate("offline")
    x, C = g["x"], g["codebooks"]
    _, ids, res, rec, fb = run_encode(x, C, "bf16", "f32")
    rows = workloads.sample_rows(len(x), LARGE_SAMPLE, seed=3)
    rep = full_check(x, C, ids, res, rec, rows)
    print("offline", rep, "fallbacks", fb.tolist())
    assert rep["rows"] >= LARGE_SAMPLE
    assert (ids[:, 0] == g["planted"][:, 0]).mean() > 0.999   # mixture centre recovered


@pytest.mark.parametrize("D,L,K", [(1024, 3, 700), (256, 2, 1500)])
def test_pairs_ragged_last_unit(D, L, K):
    """A batch long enough for CTA pairs with an odd number of 128-row tiles (at D = 1024 the last
    pair's second tile holds no rows; D = 256 runs single CTAs) and a ragged last codeword tile:
    sampled rows plus every row of the last two row tiles against the oracle, properties on all
    rows."""
    N = 65636
    rng = np.random.Generator(np.random.PCG64(4242))
    C = np.stack([rng.standard_normal((K, D), dtype=np.float32) * np.float32(0.5 ** l) for l in range(L)])
    planted = rng.integers(0, K, size=(N, L)).astype(np.int32)
    x = sum(C[l][planted[:, l]] for l in range(L)) + rng.standard_normal((N, D), dtype=np.float32) * np.float32(0.05)
    x = workloads.round_bf16(x)
    _, ids, res, rec, fb = run_encode(x, C, "bf16", "f32")
    rows = np.union1d(workloads.sample_rows(N, 4096, seed=9), np.arange(N - 100 - 128, N))
    rep = full_check(x, C, ids, res, rec, rows)
    print("pairs ragged", rep, "fallbacks", fb.tolist())
    assert (ids[:, 0] == planted[:, 0]).all()


def test_detok_decode_and_round_trip():
    g = workloads.generate("detok")
    C, want = g["codebooks"], g["planted"]
    tok = mvt.Tokenizer(dev(C, "bf16"))
    ids_d = torch.from_numpy(want).cuda()
    rec = tok.decode(ids_d)
    torch.cuda.synchronize()
    rec_h = rec.cpu().numpy()
    # decode: every row against the oracle's fp64 sum, in chunks (bounded host memory)
    worst = 0.0
    for a in range(0, len(want), 1 << 16):
        rows = np.arange(a, min(len(want), a + (1 << 16)))
        worst = max(worst, parity.check_recon(None, C, rows, want, recon_gpu=rec_h)["recon_rel_l2_max"])
    print("detok decode: all", len(want), "rows, max rel L2", worst)
    # re-encode the fp32 reconstruction: the planted ids must come back on every row
    fb = torch.zeros(C.shape[0], dtype=torch.int32, device="cuda")
    ids, res, rec2 = tok.encode(rec, residual=True, recon=True, fallbacks=fb)
    torch.cuda.synchronize()
    ids_h = ids.cpu().numpy()
    assert np.array_equal(ids_h, want), f"{int((ids_h != want).any(1).sum())} rows differ"
    srows = workloads.sample_rows(len(want), LARGE_SAMPLE, seed=5)
    rep = parity.check_ids(rec_h, C, srows, ids_h)
    rep.update(parity.check_recon(rec_h, C, srows, ids_h, rec2.cpu().numpy(), res.cpu().numpy()))
    print("detok re-encode", rep, "fallbacks", fb.tolist())
    assert rep["rows"] >= LARGE_SAMPLE


EDGE = [
    # N, D, L, K, f_dtype, cb_dtype
    (1, 64, 2, 16, "f32", "f32"),
    (1000, 256, 3, 700, "f32", "f32"),      # all-levels kernel: fp32 features, ragged N and K
    (300, 1024, 1, 300, "f32", "f32"),      # all-levels kernel, one level
    (129, 1024, 3, 257, "bf16", "bf16"),    # all-levels kernel, two row tiles
    (2, 256, 4, 5000, "bf16", "f32"),       # all-levels kernel, one row tile
    (300, 256, 20, 64, "f32", "f32"),       # all-levels kernel, 20 levels
    (150, 1024, 64, 16, "bf16", "bf16"),    # all-levels kernel, the maximum 64 levels, K < 16
    (127, 64, 3, 300, "f32", "f32"),
    (129, 128, 2, 257, "bf16", "f32"),
    (300, 256, 2, 1, "f32", "f32"),
    (513, 1024, 2, 512, "bf16", "bf16"),
    (200, 64, 4, 4096, "f32", "bf16"),
    (1000, 192, 3, 1000, "bf16", "f32"),
    (4100, 64, 2, 33, "f32", "f32"),
    (130, 4096, 2, 300, "bf16", "f32"),     # the widest rows the encode takes (streamed, per level)
    (40, 4096, 1, 17, "f32", "bf16"),
]


@pytest.mark.parametrize("N,D,L,K,fd,cd", EDGE)
def test_edge_shapes(N, D, L, K, fd, cd):
    rng = np.random.Generator(np.random.PCG64([N, D, L, K]))
    scale = 0.5 ** np.minimum(np.arange(L), 10).astype(np.float32)  # deep levels stay well inside fp32/bf16
    C = rng.standard_normal((L, K, D)).astype(np.float32) * scale[:, None, None]
    x = rng.standard_normal((N, D)).astype(np.float32)
    if cd == "bf16":
        C = workloads.round_bf16(C)
    if fd == "bf16":
        x = workloads.round_bf16(x)
    _, ids, res, rec, fb = run_encode(x, C, fd, cd)
    full_check(x, C, ids, res, rec)


def test_duplicate_and_zero_codebooks():
    rng = np.random.Generator(np.random.PCG64(21))
    base = rng.standard_normal((40, 64)).astype(np.float32)
    C = np.stack([np.concatenate([base, base, base]), np.zeros((120, 64), np.float32)])
    x = rng.standard_normal((500, 64)).astype(np.float32)
    _, ids, res, rec, fb = run_encode(x, C)
    assert (ids[:, 0] < 40).all(), "duplicate codewords must resolve to the lowest index"
    assert (ids[:, 1] == 0).all(), "all-zero level must pick codeword 0"
    full_check(x, C, ids, res, rec)


def test_codebook_equals_features():
    rng = np.random.Generator(np.random.PCG64(22))
    x = rng.standard_normal((600, 128)).astype(np.float32)
    perm = rng.permutation(600)
    C = x[perm][None]
    _, ids, res, rec, fb = run_encode(x, C)
    assert np.array_equal(ids[:, 0], np.argsort(perm))
    assert np.abs(res).max() == 0.0


@pytest.mark.parametrize("copies", [2, 16])
def test_near_ties_use_exact_rescoring(copies):
    """Groups of codewords 1e-7..1e-4 apart (relative): bf16 scores cannot order them.  Pairs
    must be settled by exact rescoring of the candidate list; groups of 16 overflow the top-8
    list, fail the certificate and must be settled by the exact full scan."""
    rng = np.random.Generator(np.random.PCG64(23 + copies))
    D, G, N = 256, 32, 400
    base = rng.standard_normal((G, D)).astype(np.float32)
    eps = (10.0 ** rng.uniform(-7, -4, size=(copies, G, 1))).astype(np.float32)
    eps[0] = 0.0
    C = (base[None] * (1 + eps)).reshape(1, copies * G, D)
    pick = rng.integers(0, G, size=N)
    x = base[pick] + 1e-3 * rng.standard_normal((N, D)).astype(np.float32)
    _, ids, res, rec, fb = run_encode(x, C)
    rep = full_check(x, C, ids, res, rec)
    print("near ties", copies, rep, "fallbacks", fb.tolist())
    if copies > 8:
        assert fb.sum() > 0


@pytest.mark.parametrize("copies", [2, 16])
def test_near_ties_wide_rows(copies):
    """The same near-tie groups at D = 1024 (the all-levels kernel): groups of 16 overflow the
    candidate lists, so their rows take the exact scan split into codeword slices."""
    rng = np.random.Generator(np.random.PCG64(123 + copies))
    D, G, N, L = 1024, 16, 300, 2
    base = rng.standard_normal((G, D)).astype(np.float32)
    eps = (10.0 ** rng.uniform(-7, -4, size=(copies, G, 1))).astype(np.float32)
    eps[0] = 0.0
    lvl0 = (base[None] * (1 + eps)).reshape(copies * G, D)
    lvl1 = 0.1 * rng.standard_normal((copies * G, D)).astype(np.float32)
    C = np.stack([lvl0, lvl1])
    pick = rng.integers(0, G, size=N)
    x = workloads.round_bf16(base[pick] + 1e-3 * rng.standard_normal((N, D)).astype(np.float32))
    _, ids, res, rec, fb = run_encode(x, C, "bf16", "f32")
    rep = full_check(x, C, ids, res, rec)
    print("wide near ties", copies, rep, "fallbacks", fb.tolist())
    if copies > 8:
        assert fb[0] > 0


def test_exact_queue_overflow_wide_rows():
    """More uncertifiable rows than the all-levels kernel queues for sliced exact scans: the rest
    are scanned whole by the warp that found them."""
    rng = np.random.Generator(np.random.PCG64(131))
    D, G, copies, N = 1024, 32, 16, 1300
    base = rng.standard_normal((G, D)).astype(np.float32)
    eps = (10.0 ** rng.uniform(-7, -5, size=(copies, G, 1))).astype(np.float32)
    eps[0] = 0.0
    C = (base[None] * (1 + eps)).reshape(1, copies * G, D)
    x = workloads.round_bf16(base[rng.integers(0, G, size=N)] + 1e-4 * rng.standard_normal((N, D)).astype(np.float32))
    _, ids, res, rec, fb = run_encode(x, C, "bf16", "f32")
    full_check(x, C, ids, res, rec)
    print("queue overflow fallbacks", fb.tolist())
    assert fb[0] > 1024


def test_per_level_path_matches_oracle():
    """RVQ_PERSISTENT=0 (fresh process): every level as its own GEMM + certificate launches."""
    import os
    import subprocess
    import sys
    code = (
        "import numpy as np, torch, workloads\n"
        "from tests import parity, test_gpu_parity as t\n"
        "g = workloads.generate('image', n_override=700)\n"
        "_, ids, res, rec, fb = t.run_encode(g['x'], g['codebooks'], 'bf16', 'f32')\n"
        "t.full_check(g['x'], g['codebooks'], ids, res, rec)\n"
        "print('per-level ok')\n")
    env = dict(os.environ, RVQ_PERSISTENT="0")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, "-c", code], env=env, cwd=root, capture_output=True, text=True,
                         timeout=600)
    assert out.returncode == 0 and "per-level ok" in out.stdout, out.stdout[-2000:] + out.stderr[-2000:]


def test_decode_out_of_range_sets_status():
    C = np.random.Generator(np.random.PCG64(24)).standard_normal((2, 10, 64)).astype(np.float32)
    tok = mvt.Tokenizer(dev(C, "f32"))
    ids = torch.zeros((5, 2), dtype=torch.int32, device="cuda")
    ids[3, 1] = 10
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rec = tok.decode(ids, status=st, check=False)
    torch.cuda.synchronize()
    assert int(st.item()) == -5
    want = np.array(C[0, 0] + C[1, 0], np.float32)
    assert np.allclose(rec[0].cpu().numpy(), want)
    assert np.allclose(rec[3].cpu().numpy(), C[0, 0])      # bad level contributes nothing


def test_bad_offsets_set_status():
    rng = np.random.Generator(np.random.PCG64(25))
    C = rng.standard_normal((1, 32, 64)).astype(np.float32)
    x = rng.standard_normal((50, 64)).astype(np.float32)
    tok = mvt.Tokenizer(dev(C, "f32"))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    off = torch.tensor([0, 30, 20, 50], dtype=torch.int64, device="cuda")
    tok.encode(dev(x, "f32"), offsets=off, status=st, check=False)
    torch.cuda.synchronize()
    assert int(st.item()) == -1


def test_bad_offsets_set_status_all_levels_kernel():
    """The all-levels kernel checks the packed-batch offsets too (D = 1024)."""
    rng = np.random.Generator(np.random.PCG64(125))
    C = rng.standard_normal((2, 300, 1024)).astype(np.float32)
    x = rng.standard_normal((200, 1024)).astype(np.float32)
    tok = mvt.Tokenizer(dev(C, "f32"))
    assert mvt.rvq_encode_levels_per_launch(200, 1024, 2, 300) == (0, 2)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    off = torch.tensor([0, 120, 90, 200], dtype=torch.int64, device="cuda")
    tok.encode(dev(x, "f32"), offsets=off, status=st, check=False)
    torch.cuda.synchronize()
    assert int(st.item()) == -1


def test_bounded_waits_give_up():
    """A wait on an mbarrier phase and on a counter that nothing completes ends after its limit
    with RVQ_ERR_TIMEOUT in the status word, and the context stays usable."""
    import time
    ctr = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    assert mvt.rvq_selftest_wait_timeout(ctr, st, 50_000) == 0
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert int(st.item()) == -6, mvt.rvq_status_str(int(st.item()))
    assert 0.045 < dt < 5.0, dt
    g = workloads.generate("tiny")
    _, ids, res, rec, fb = run_encode(g["x"], g["codebooks"])
    full_check(g["x"], g["codebooks"], ids, res, rec)


def test_empty_batch_is_noop():
    C = np.random.Generator(np.random.PCG64(26)).standard_normal((2, 16, 64)).astype(np.float32)
    tok = mvt.Tokenizer(dev(C, "f32"))
    ids, _, _ = tok.encode(torch.empty((0, 64), device="cuda"))
    assert ids.shape == (0, 2)


def test_norms_and_stats():
    g = workloads.generate("image", n_override=8)
    C = g["codebooks"]
    tok = mvt.Tokenizer(dev(C, "f32"))
    torch.cuda.synchronize()
    n = tok.norms.cpu().numpy().astype(np.float64)
    want = (C.astype(np.float64) ** 2).sum(-1)
    D = C.shape[2]
    assert np.allclose(n, want, rtol=(D // 32 + 2) * 2 ** -24, atol=0)   # fp32 lane sums of D/32 squares
    op = tok.operand.float().cpu().numpy()
    assert np.array_equal(op, workloads.round_bf16(C))
    st = tok.level_stats.cpu().numpy()
    cn = np.sqrt(want).max(1)
    assert (st[:, 0] >= cn * (1 - 1e-6)).all() and (st[:, 0] <= cn * (1 + 1e-5)).all()
    assert (st[:, 3] >= want.max(1) * (1 - 1e-6)).all()
    err = np.sqrt(((C.astype(np.float64) - op) ** 2).sum(-1)).max(1)
    assert (st[:, 1] >= err * (1 - 1e-5)).all() and (st[:, 1] <= err * (1 + 1e-4)).all()


def test_launch_count_and_profile_hooks():
    g = workloads.generate("tiny")
    tok = mvt.Tokenizer(dev(g["codebooks"], "f32"))
    x = dev(g["x"], "f32")
    before = mvt.rvq_launch_count()
    assert mvt.rvq_profile_enable(True) == 0
    tok.encode(x)
    code, n, ms = mvt.rvq_profile_read()
    mvt.rvq_profile_enable(False)
    assert code == 0 and n == g["spec"].L and ms > 0
    assert mvt.rvq_launch_count() - before == 1 + 3 * g["spec"].L


def test_levels_per_launch_query():
    """D in (128, 256] or (512, 1024] runs all levels in one launch; other widths launch per level."""
    assert mvt.rvq_encode_levels_per_launch(4096, 1024, 4, 8192) == (0, 4)
    assert mvt.rvq_encode_levels_per_launch(4096, 768, 3, 1000) == (0, 3)
    assert mvt.rvq_encode_levels_per_launch(4096, 256, 4, 8192) == (0, 4)
    assert mvt.rvq_encode_levels_per_launch(4096, 128, 4, 8192) == (0, 1)
    assert mvt.rvq_encode_levels_per_launch(4096, 512, 4, 8192) == (0, 1)
    assert mvt.rvq_encode_levels_per_launch(4096, 2048, 4, 8192) == (0, 1)
    g = workloads.generate("image", n_override=300)
    tok = mvt.Tokenizer(dev(g["codebooks"], "f32"))
    x = dev(g["x"], "bf16")
    assert mvt.rvq_profile_enable(True) == 0
    tok.encode(x)
    code, n, ms = mvt.rvq_profile_read()
    mvt.rvq_profile_enable(False)
    assert code == 0 and n == g["spec"].L and ms > 0


def test_wide_features_use_streaming_rows():
    """D > 1024 takes the path that materialises the fp32 residual and streams rows."""
    rng = np.random.Generator(np.random.PCG64(27))
    L, K, D, N = 3, 300, 2048, 200
    C = rng.standard_normal((L, K, D)).astype(np.float32) * (0.5 ** np.arange(L, dtype=np.float32))[:, None, None]
    x = workloads.round_bf16(C[0][rng.integers(0, K, N)] + 0.1 * rng.standard_normal((N, D)).astype(np.float32))
    _, ids, res, rec, fb = run_encode(x, C, "bf16", "f32")
    full_check(x, C, ids, res, rec)


def test_fewer_codewords_than_list_entries():
    rng = np.random.Generator(np.random.PCG64(28))
    for K in (1, 3, 7):
        C = rng.standard_normal((2, K, 64)).astype(np.float32)
        x = rng.standard_normal((150, 64)).astype(np.float32)
        _, ids, res, rec, fb = run_encode(x, C)
        full_check(x, C, ids, res, rec)


def test_decode_many_levels_generic_path():
    """More than 16 levels uses the runtime-level decode kernel."""
    rng = np.random.Generator(np.random.PCG64(29))
    L, K, D, N = 20, 37, 96, 333
    C = workloads.round_bf16(rng.standard_normal((L, K, D)).astype(np.float32))
    ids = rng.integers(0, K, size=(N, L)).astype(np.int32)
    for dt in ("f32", "bf16"):
        tok = mvt.Tokenizer(dev(C, dt))
        rec = tok.decode(torch.from_numpy(ids).cuda())
        torch.cuda.synchronize()
        parity.check_recon(None, C, np.arange(N), ids, recon_gpu=rec.cpu().numpy())


@pytest.mark.parametrize("N,L,K,D", [
    (3001, 8, 500, 512),     # ragged token count, two 256-column slices
    (1, 1, 7, 256),          # one token, one level (a gather of four rows, three of them padding)
    (777, 3, 64, 768),       # L not a multiple of four
    (4100, 16, 33, 256),     # the deepest level count the fixed decode handles
])
def test_bf16_decode_whole_slices(N, L, K, D):
    """bf16 codebooks with D % 256 == 0: every row against the oracle, and an id outside [0, K)
    sets the status and drops that level only."""
    rng = np.random.Generator(np.random.PCG64([N, L, K, D]))
    C = workloads.round_bf16(rng.standard_normal((L, K, D)).astype(np.float32))
    ids = rng.integers(0, K, size=(N, L)).astype(np.int32)
    tok = mvt.Tokenizer(dev(C, "bf16"))
    rec = tok.decode(torch.from_numpy(ids).cuda())
    torch.cuda.synchronize()
    parity.check_recon(None, C, np.arange(N), ids, recon_gpu=rec.cpu().numpy())
    bad = ids.copy()
    bad[N // 2, L - 1] = K
    bad[0, 0] = -1
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rec2 = tok.decode(torch.from_numpy(bad).cuda(), status=st, check=False).cpu().numpy()
    assert int(st.item()) == -5
    keep = (bad >= 0) & (bad < K)
    for n in (0, N // 2):
        want = sum(C[l, bad[n, l]].astype(np.float64) for l in range(L) if keep[n, l])
        want = np.zeros(D) if isinstance(want, int) else want
        assert np.allclose(rec2[n], want, rtol=1e-5, atol=1e-5)
    others = np.ones(N, bool)
    others[[0, N // 2]] = False
    assert np.array_equal(rec2[others], rec.cpu().numpy()[others])


@pytest.mark.parametrize("L,K,D,dt", [
    (4, 65536, 256, "f32"),   # 128-column slices would hold 128 MiB of codebook: two rows per warp
    (8, 65536, 128, "f32"),   # four rows per warp (32-column slices)
    (8, 65536, 256, "bf16"),  # four rows per warp, 16-byte bf16 gathers
    (12, 32768, 132, "bf16"),  # D % 8 != 0: 8-byte gathers, two rows per warp
])
def test_decode_narrow_slices(L, K, D, dt):
    """Codebooks whose live columns outgrow L2 are decoded in narrower slices with several rows per
    warp: every row against the oracle at ragged counts (fewer rows than a warp holds included),
    and out-of-range ids in rows held by different lane groups set the status and drop only
    their own level.  Called through rvq_decode itself (D % 64 != 0 is a decode-only width)."""
    rng = np.random.Generator(np.random.PCG64([L, K, D, 11]))
    C = rng.standard_normal((L, K, D), dtype=np.float32)
    if dt == "bf16":
        C = workloads.round_bf16(C)
    Cd = dev(C, dt)
    code = mvt.RVQ_BF16 if dt == "bf16" else mvt.RVQ_F32

    def decode(ids):
        N = ids.shape[0]
        rec = torch.empty((N, D), dtype=torch.float32, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        assert mvt.rvq_decode(torch.from_numpy(ids).cuda(), N, L, Cd, code, K, D, rec, st) == 0
        torch.cuda.synchronize()
        return rec.cpu().numpy(), int(st.item())

    for N in (1, 3, 5003):
        ids = rng.integers(0, K, size=(N, L)).astype(np.int32)
        rec, st = decode(ids)
        assert st == 0
        parity.check_recon(None, C, np.arange(N), ids, recon_gpu=rec)
    bad = ids.copy()
    hit = [1, 2, N - 1]
    bad[1, L - 1] = K
    bad[2, 0] = -1
    bad[N - 1, L // 2] = 1 << 30
    rec2, st = decode(bad)
    assert st == -5
    keep = (bad >= 0) & (bad < K)
    for n in hit:
        want = sum(C[l, bad[n, l]].astype(np.float64) for l in range(L) if keep[n, l])
        assert np.allclose(rec2[n], want, rtol=1e-5, atol=1e-5)
    others = np.ones(N, bool)
    others[hit] = False
    assert np.array_equal(rec2[others], rec[others])
