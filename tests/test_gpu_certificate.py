"""The certificate's hardware model, measured on the B200.

The encode accepts a row without an exact scan of all K codewords when its bf16 candidate
scores leave no doubt, using a bound E on |d~ - (||r-c||^2 - ||r||^2)| that assumes the tensor
core forms bf16 products exactly and adds them into an fp32 accumulator with at most one rounding
per addition.  Here every candidate score the kernels left in the workspace (the 8 lowest d~ per
row, 128-row tile and slot, of the last level encoded; rvq_encode_candidate_layout says where)
is compared with the exact value from the stored operands in fp64, and must lie within E
computed in fp64 from the row's residual and the level's codebook maxima.  The maximum of
|err| / E is printed.
"""
import numpy as np
import pytest

import workloads

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import multimodal_visual_tokenization_b200 as mvt  # noqa: E402


def error_bound(rx, ry, C, D):
    """E per row for level codebook C [K, D] (fp32 stored values): rx = ||r - bf16(r)||, ry = ||bf16(r)||."""
    c = C.astype(np.float64)
    cq = workloads.round_bf16(C).astype(np.float64)
    cmax = np.sqrt((c * c).sum(1)).max()
    dcmax = np.sqrt(((c - cq) ** 2).sum(1)).max()
    cqmax = np.sqrt((cq * cq).sum(1)).max()
    nmax = (c * c).sum(1).max() * (1 + 2.0 ** -23)  # fl32(||c||^2) <= that
    gamma = (D + 32) * 2.0 ** -22
    norm_err = (D // 32 + 2) * 2.0 ** -24
    e = norm_err * nmax + 2 * (rx * cmax + ry * dcmax) + 2 * gamma * (ry * cqmax + 0.51 * nmax) + 2.0 ** -23 * nmax
    return 1.01 * e


def measure(x, C, f_dtype, rows):
    """Encode x with codebooks C (fp32 [L, K, D]) in a workspace this test keeps, then compare the
    last level's candidate scores of `rows` with the exact values.  Returns (max |err|/E, entries)."""
    N, D = x.shape
    L, K, _ = C.shape
    tok = mvt.Tokenizer(torch.from_numpy(C).cuda())
    xd = torch.from_numpy(x).cuda()
    if f_dtype == "bf16":
        xd = xd.to(torch.bfloat16)
    code, nbytes = mvt.rvq_encode_workspace_size(N, D, L, K)
    assert code == 0
    ws = torch.full((nbytes,), 0xFF, dtype=torch.uint8, device="cuda")  # empty slots read as id -1
    ids = torch.empty((N, L), dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    code = mvt.rvq_encode(xd, mvt._dtype_code(xd), N, D, tok.codebooks, tok.cb_dtype, tok.operand, tok.norms,
                          tok.level_stats, L, K, None, 0, ids, None, None, None, ws, nbytes, status)
    assert code == 0, mvt.rvq_status_str(code)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    code, off, slots = mvt.rvq_encode_candidate_layout(N, D, L, K)
    assert code == 0 and slots >= 1
    RT = (N + 127) // 128
    raw = ws[off:off + RT * slots * 128 * 8 * 8].cpu().numpy()
    d_t = raw.view(np.float32).reshape(RT, slots, 128, 8, 2)[..., 0]
    id_t = raw.view(np.int32).reshape(RT, slots, 128, 8, 2)[..., 1]
    ids_h = ids.cpu().numpy()
    # the fp32 residual of the last level, exactly as the kernels form it: r -= C_l[id] in fp32
    r = x[rows].astype(np.float32)
    for j in range(L - 1):
        r = (r - C[j][ids_h[rows, j]]).astype(np.float32)
    rq = workloads.round_bf16(r).astype(np.float64)
    r64 = r.astype(np.float64)
    rx = np.sqrt(((r64 - rq) ** 2).sum(1))
    ry = np.sqrt((rq * rq).sum(1))
    Cl = C[L - 1]
    E = error_bound(rx, ry, Cl, D)
    c64 = Cl.astype(np.float64)
    exact = (c64 * c64).sum(1)[None, :] - 2.0 * (r64 @ c64.T)  # ||r-c||^2 - ||r||^2, fp64
    worst, entries, found = 0.0, 0, 0
    for j, n in enumerate(rows):
        d = d_t[n // 128, :, n % 128].reshape(-1)
        k = id_t[n // 128, :, n % 128].reshape(-1)
        ok = (k >= 0) & (k < K)
        assert ok.sum() >= min(8, K), f"row {n}: only {int(ok.sum())} candidates"
        err = np.abs(d[ok].astype(np.float64) - exact[j, k[ok]])
        ratio = float(err.max() / E[j])
        assert ratio <= 1.0, f"row {n}: |d~ - exact| = {err.max():.4g} above the bound {E[j]:.4g}"
        found += int(ids_h[n, L - 1]) in set(k[ok].tolist())
        worst = max(worst, ratio)
        entries += int(ok.sum())
    # the chosen codeword is normally among the candidates (only rows settled by the exact scan of
    # all K codewords may have chosen one the lists dropped)
    assert found >= 0.99 * len(rows), f"chosen id among the candidates in only {found} of {len(rows)} rows"
    return worst, entries


def test_bound_holds_on_packed_shaped_rows():
    """All-levels kernel, D = 1024, K = 16384: level-2 candidates of packed-batch features."""
    g = workloads.generate("packed", n_override=4096)
    x, C = g["x"], np.ascontiguousarray(g["codebooks"][:3])
    rows = workloads.sample_rows(len(x), 384, seed=31)
    worst, entries = measure(x, C, "bf16", rows)
    print(f"packed-shaped: {entries} candidate scores, max |err|/E = {worst:.3g}")


def test_bound_holds_with_cta_pairs():
    """All-levels kernel run as CTA pairs (66000 rows at D = 1024): the M = 256 MMAs
    of a pair must meet the same bound; rows from both CTAs of a pair are sampled."""
    g = workloads.generate("packed", n_override=66000)
    x, C = g["x"], np.ascontiguousarray(g["codebooks"][:3])
    rows = workloads.sample_rows(len(x), 384, seed=35)
    assert (((rows // 128) % 2) == 1).any() and (((rows // 128) % 2) == 0).any()
    worst, entries = measure(x, C, "bf16", rows)
    print(f"packed-shaped, CTA pairs: {entries} candidate scores, max |err|/E = {worst:.3g}")


def test_bound_holds_on_offline_shaped_rows():
    """All-levels kernel, D = 256, K = 65536: level-1 candidates of mixture features."""
    g = workloads.generate("offline", n_override=8192)
    x, C = g["x"], np.ascontiguousarray(g["codebooks"][:2])
    rows = workloads.sample_rows(len(x), 384, seed=32)
    worst, entries = measure(x, C, "bf16", rows)
    print(f"offline-shaped: {entries} candidate scores, max |err|/E = {worst:.3g}")


def test_bound_holds_in_the_per_level_kernel():
    """Per-level distance GEMM (D = 512), fp32 features: level-1 candidates."""
    rng = np.random.Generator(np.random.PCG64(33))
    L, K, D, N = 2, 4096, 512, 2048
    C = rng.standard_normal((L, K, D)).astype(np.float32) * np.array([1.0, 0.5], np.float32)[:, None, None]
    x = (C[0][rng.integers(0, K, N)] + 0.5 * rng.standard_normal((N, D))).astype(np.float32)
    assert mvt.rvq_encode_levels_per_launch(N, D, L, K) == (0, 1)
    worst, entries = measure(x, C, "f32", workloads.sample_rows(N, 384, seed=34))
    print(f"per-level D=512: {entries} candidate scores, max |err|/E = {worst:.3g}")
