"""Gradient of the visual-token embedding e[n] = sum_l E_l[ids[n,l]] on the GPU (rvq_embed_backward
with fp32 atomics, rvq_embed_backward_sorted by sorted segments) against the fp64 oracle, element
by element.

fp32 atomics add a destination row's terms in no fixed order, so the GPU result may differ from
the exact sum by rounding: for c terms (the initial value counted as one more) recursive fp32
summation in any order stays within (c - 1) * 2^-24 * sum |terms| of it; the test allows that
bound (+1%) per element, using the oracle's per-row counts and magnitude sums.
"""
import numpy as np
import pytest

import oracle
import workloads

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import multimodal_visual_tokenization_b200 as mvt  # noqa: E402

U = 2.0 ** -24


def run_backward(ids, g, K, grad0=None, sort=False, raw=False):
    N, L = ids.shape
    H = g.shape[1]
    gt = torch.from_numpy(np.ascontiguousarray(g, np.float32)).cuda()
    it = torch.from_numpy(np.ascontiguousarray(ids, np.int32)).cuda()
    out = (torch.zeros((L, K, H), dtype=torch.float32, device="cuda") if grad0 is None
           else torch.from_numpy(np.ascontiguousarray(grad0, np.float32)).cuda())
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    if sort:
        code, nbytes = mvt.rvq_embed_backward_workspace_size(N, L, K, H)
        assert code == 0
        ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device="cuda")
        rc = mvt.rvq_embed_backward_sorted(it, N, L, K, H, gt, out, ws, nbytes, st)
    else:
        rc = mvt.rvq_embed_backward(it, N, L, K, H, gt, out, st)
    torch.cuda.synchronize()
    assert rc == 0, mvt.rvq_status_str(rc)
    got = out.cpu().numpy()
    return (got if raw else got.astype(np.float64)), int(st.item())


def check(ids, g, K, grad0=None, sort=False):
    got, st = run_backward(ids, g, K, grad0, sort)
    want, count, absum = oracle.embed_backward(ids, g, K, bounds=True)
    terms = count[:, :, None].astype(np.float64)
    if grad0 is not None:
        want = want + grad0.astype(np.float64)
        absum = absum + np.abs(grad0.astype(np.float64))
        terms = terms + 1.0
    tol = 1.01 * np.maximum(terms - 1.0, 0.0) * U * absum
    err = np.abs(got - want)
    bad = err > tol
    assert not bad.any(), (int(bad.sum()), float(err[bad].max()), float(tol[bad].min()))
    return st, float((err / np.maximum(absum, 1e-30)).max())


def _case(seed, N, L, K, H, zipf=None):
    rng = np.random.Generator(np.random.PCG64(seed))
    if zipf:
        ids = np.minimum(rng.zipf(zipf, size=(N, L)) - 1, K - 1).astype(np.int32)
    else:
        ids = rng.integers(0, K, size=(N, L)).astype(np.int32)
    g = rng.standard_normal((N, H)).astype(np.float32)
    return ids, g


@pytest.mark.parametrize("sort", [False, True])
@pytest.mark.parametrize("N,L,K,H,zipf", [
    (3000, 4, 50, 96, None),      # one slice, lanes 24..31 idle
    (20000, 8, 512, 256, 1.1),    # popular ids: thousands of terms per row (sorted: pieces of 256)
    (777, 3, 1000, 100, None),    # H not a multiple of 128 (25 fp32x4 columns)
    (500, 40, 64, 128, None),     # more than 32 levels
    (1, 2, 7, 4, None),           # a single row
    (40000, 2, 49151, 20, 1.05),  # sorted: the largest K, many empty ids, two column slices
    (70000, 3, 300, 8, None),     # sorted: several histogram chunks, ragged last chunk
    (5000, 3, 300, 1100, 1.1),    # sorted: two 1024-column passes per segment, the second ragged
    (3000, 2, 200, 2048, None),   # sorted: two full passes
])
def test_embed_backward_matches_oracle(N, L, K, H, zipf, sort):
    ids, g = _case(N * 7 + L, N, L, K, H, zipf)
    st, rel = check(ids, g, K, sort=sort)
    assert st == 0
    print("embed backward", "sorted" if sort else "atomic", (N, L, K, H), "max |err| / sum|terms|", rel)


@pytest.mark.parametrize("sort", [False, True])
def test_embed_backward_accumulates_into_existing_gradient(sort):
    ids, g = _case(31, 4000, 2, 300, 64)
    grad0 = np.random.Generator(np.random.PCG64(32)).standard_normal((2, 300, 64)).astype(np.float32)
    st, _ = check(ids, g, 300, grad0, sort=sort)
    assert st == 0


def test_sorted_backward_is_deterministic():
    """Zipf ids (hot ids cut into pieces) and one id taking every token of a level: two calls give
    bit-identical gradients, both within the oracle's bound."""
    ids, g = _case(36, 30000, 3, 700, 48, 1.1)
    ids[:, 2] = 5                       # one segment of 30000 tokens: 118 pieces
    a, st = run_backward(ids, g, 700, sort=True, raw=True)
    b, _ = run_backward(ids, g, 700, sort=True, raw=True)
    assert st == 0 and np.array_equal(a, b)
    check(ids, g, 700, sort=True)


@pytest.mark.parametrize("sort", [False, True])
def test_embed_backward_bad_id_sets_status_and_skips(sort):
    ids, g = _case(33, 600, 3, 80, 32)
    ids[17, 1] = 80   # out of range
    ids[400, 2] = -3
    got, st = run_backward(ids, g, 80, sort=sort)
    assert st == -5
    keep = ids.copy()
    mask = (keep < 0) | (keep >= 80)
    # the oracle skips the same entries: compare with the bad ones removed from the sums
    want = np.zeros((3, 80, 32))
    for l in range(3):
        ok = ~mask[:, l]
        np.add.at(want[l], keep[ok, l], g[ok].astype(np.float64))
    assert np.allclose(got, want, rtol=1e-5, atol=1e-4)


def test_embedding_forward_is_decode_and_adjoint_holds():
    """Forward e = rvq_decode(ids, E); <e, G> equals <E, backward(ids, G)> up to fp32 rounding."""
    ids, G = _case(34, 5000, 4, 200, 128, 1.2)
    E = np.random.Generator(np.random.PCG64(35)).standard_normal((4, 200, 128)).astype(np.float32)
    tok = mvt.Tokenizer(torch.from_numpy(E).cuda())
    e = tok.decode(torch.from_numpy(ids).cuda()).cpu().numpy().astype(np.float64)
    grad, st = run_backward(ids, G, 200)
    assert st == 0
    lhs = float(np.sum(e * G))
    rhs = float(np.sum(E.astype(np.float64) * grad))
    assert abs(lhs - rhs) <= 1e-4 * (np.sum(np.abs(e * G)) + 1.0), (lhs, rhs)


def test_sorted_backward_workspace_checks():
    ids = torch.zeros((10, 2), dtype=torch.int32, device="cuda")
    g = torch.zeros((10, 16), dtype=torch.float32, device="cuda")
    out = torch.zeros((2, 8, 16), dtype=torch.float32, device="cuda")
    code, nbytes = mvt.rvq_embed_backward_workspace_size(10, 2, 8, 16)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    assert mvt.rvq_embed_backward_sorted(ids, 10, 2, 8, 16, g, out, ws, nbytes - 256) == -3
    assert mvt.rvq_embed_backward_sorted(ids, 10, 2, 49152, 16, g, out, ws, nbytes) == -2
