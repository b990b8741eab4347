"""k-means update of one codebook level on the GPU (rvq_codebook_update) against the fp64 oracle.

The cluster sums are fp32 atomics in no fixed order; with c points of total magnitude
A = sum |p| the fp32 sum is within (c - 1) * 2^-24 * A of the exact one, and dividing it by c
(exact count, one rounding) keeps the mean within 2^-24 * A / c * (c - 1) + 2^-24 * |mean|
<= 2^-24 * A of the exact mean; the test allows that bound (+1%).  Empty clusters must keep
their codeword exactly.
"""
import numpy as np
import pytest

import oracle

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import multimodal_visual_tokenization_b200 as mvt  # noqa: E402

U = 2.0 ** -24


def gpu_update(p, ids, old, inplace=False):
    N, D = p.shape
    K = old.shape[0]
    pt = torch.from_numpy(np.ascontiguousarray(p, np.float32)).cuda()
    it = torch.from_numpy(np.ascontiguousarray(ids, np.int32)).cuda()
    ot = torch.from_numpy(np.ascontiguousarray(old, np.float32)).cuda()
    nt = ot if inplace else torch.empty_like(ot)
    sums = torch.empty_like(ot)
    counts = torch.empty(K, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = mvt.rvq_codebook_update(pt, it, N, D, K, ot, nt, sums, counts, st)
    torch.cuda.synchronize()
    assert rc == 0, mvt.rvq_status_str(rc)
    return nt.cpu().numpy().astype(np.float64), counts.cpu().numpy(), int(st.item())


def check(p, ids, old, inplace=False):
    new, counts, st = gpu_update(p, ids, old, inplace)
    want, count, absum = oracle.codebook_update(p, ids, old, bounds=True)
    assert np.array_equal(counts, count)
    empty = count == 0
    assert np.array_equal(new[empty], old[empty].astype(np.float64))
    tol = 1.01 * U * absum[~empty]
    err = np.abs(new[~empty] - want[~empty])
    assert (err <= tol).all(), (float(err.max()), float(tol.min()))
    return st


def _case(seed, N, D, K, zipf=None, gap=0):
    rng = np.random.Generator(np.random.PCG64(seed))
    p = rng.standard_normal((N, D)).astype(np.float32)
    hi = K - 1 - gap
    ids = (np.minimum(rng.zipf(zipf, size=N) - 1, hi) if zipf else rng.integers(0, hi + 1, size=N)).astype(np.int32)
    old = rng.standard_normal((K, D)).astype(np.float32)
    return p, ids, old


@pytest.mark.parametrize("N,D,K,zipf,gap", [
    (5000, 64, 100, None, 10),     # uniform, last 10 clusters empty
    (20000, 256, 1000, 1.1, 0),    # skewed: one cluster with thousands of points
    (333, 100, 64, None, 0),       # D not a multiple of 128
    (1, 4, 3, None, 0),
])
def test_codebook_update_matches_oracle(N, D, K, zipf, gap):
    p, ids, old = _case(N + D + K, N, D, K, zipf, gap)
    assert check(p, ids, old) == 0


def test_codebook_update_in_place_and_empty_batch():
    p, ids, old = _case(7, 3000, 32, 50, None, 5)
    assert check(p, ids, old, inplace=True) == 0
    new, counts, st = gpu_update(np.zeros((0, 32), np.float32), np.zeros(0, np.int32), old)
    assert np.array_equal(new, old.astype(np.float64)) and counts.sum() == 0 and st == 0


def test_codebook_update_bad_id_sets_status():
    p, ids, old = _case(8, 400, 16, 20)
    ids[5] = 20
    new, counts, st = gpu_update(p, ids, old)
    assert st == -5 and counts.sum() == 399


def test_lloyd_iteration_on_gpu_lowers_the_error():
    """encode (one level) -> update: the squared error of the points to their codewords drops."""
    rng = np.random.Generator(np.random.PCG64(9))
    centres = rng.standard_normal((64, 256)).astype(np.float32)
    x = (centres[rng.integers(0, 64, size=8000)] + 0.3 * rng.standard_normal((8000, 256))).astype(np.float32)
    C = rng.standard_normal((1, 256, 256)).astype(np.float32)
    tok = mvt.Tokenizer(torch.from_numpy(C).cuda())
    xt = torch.from_numpy(x).cuda()
    ids, res, _ = tok.encode(xt, residual=True)
    torch.cuda.synchronize()
    sse0 = float((res.double() ** 2).sum())
    new, counts, st = gpu_update(x, ids[:, 0].contiguous().cpu().numpy(), C[0])
    assert st == 0
    idn = ids[:, 0].cpu().numpy()
    sse1 = float(((x.astype(np.float64) - new[idn]) ** 2).sum())
    assert sse1 < sse0
