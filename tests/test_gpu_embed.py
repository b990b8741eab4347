"""Gradient of the visual-token embedding e[n] = sum_l E_l[ids[n,l]] on the GPU
(rvq_embed_backward) against the fp64 oracle, element by element.

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


def run_backward(ids, g, K, grad0=None):
    N, L = ids.shape
    H = g.shape[1]
    gt = torch.from_numpy(np.ascontiguousarray(g, np.float32)).cuda()
    it = torch.from_numpy(np.ascontiguousarray(ids, np.int32)).cuda()
    out = (torch.zeros((L, K, H), dtype=torch.float32, device="cuda") if grad0 is None
           else torch.from_numpy(np.ascontiguousarray(grad0, np.float32)).cuda())
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = mvt.rvq_embed_backward(it, N, L, K, H, gt, out, st)
    torch.cuda.synchronize()
    assert rc == 0, mvt.rvq_status_str(rc)
    return out.cpu().numpy().astype(np.float64), int(st.item())


def check(ids, g, K, grad0=None):
    got, st = run_backward(ids, g, K, grad0)
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


@pytest.mark.parametrize("N,L,K,H,zipf", [
    (3000, 4, 50, 96, None),      # one slice, lanes 24..31 idle
    (20000, 8, 512, 256, 1.1),    # popular ids: thousands of terms per row
    (777, 3, 1000, 100, None),    # H not a multiple of 128 (25 fp32x4 columns)
    (500, 40, 64, 128, None),     # more than 32 levels
    (1, 2, 7, 4, None),           # a single row
])
def test_embed_backward_matches_oracle(N, L, K, H, zipf):
    ids, g = _case(N * 7 + L, N, L, K, H, zipf)
    st, rel = check(ids, g, K)
    assert st == 0
    print("embed backward", (N, L, K, H), "max |err| / sum|terms|", rel)


def test_embed_backward_accumulates_into_existing_gradient():
    ids, g = _case(31, 4000, 2, 300, 64)
    grad0 = np.random.Generator(np.random.PCG64(32)).standard_normal((2, 300, 64)).astype(np.float32)
    st, _ = check(ids, g, 300, grad0)
    assert st == 0


def test_embed_backward_bad_id_sets_status_and_skips():
    ids, g = _case(33, 600, 3, 80, 32)
    ids[17, 1] = 80   # out of range
    ids[400, 2] = -3
    got, st = run_backward(ids, g, 80)
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
