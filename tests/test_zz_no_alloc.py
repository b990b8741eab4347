"""rvq_encode_noalloc: the encode entry point for callers that cannot allocate device memory
(a framework that owns every device byte through its own pool, a serving loop that must not
call cudaMalloc because it can synchronize the device, a plugin host that offers no
workspace).  Its scratch is the library's own statically sized device array.

Checked through the C ABI against rvq_encode with a caller workspace, on two calls in a row
(the shared scratch keeps the first call's contents when the second starts), with the
tolerances the parity tests use: ids equal, residual and recon within REL_L2.  Kept in a file
that pytest collects last; it passes alone in a fresh process and after the other tests.
"""
import numpy as np
import pytest

import workloads
from tests.parity import REL_L2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import multimodal_visual_tokenization_b200 as mvt  # noqa: E402


def _features(batch, n):
    g = workloads.generate("image", batch=batch, n_override=n)
    return g, torch.from_numpy(g["x"]).to(torch.bfloat16).cuda()


def _rel_l2(a, b):
    a = a.double()
    b = b.double()
    return float(((a - b).norm(dim=1) / b.norm(dim=1).clamp_min(1e-30)).max())


def test_noalloc_matches_workspace_encode_on_two_calls():
    n = 1024
    g, _ = _features(0, n)
    tok = mvt.Tokenizer(torch.from_numpy(g["codebooks"]).cuda())
    code, need = mvt.rvq_encode_workspace_size(n, tok.D, tok.L, tok.K)
    assert code == 0 and need <= mvt.RVQ_NOALLOC_SCRATCH_BYTES
    for batch in (0, 1):
        _, x = _features(batch, n)
        ids_ref, res_ref, rec_ref = tok.encode(x, residual=True, recon=True)
        ids = torch.full((n, tok.L), -1, dtype=torch.int32, device="cuda")
        res = torch.empty((n, tok.D), dtype=torch.float32, device="cuda")
        rec = torch.empty((n, tok.D), dtype=torch.float32, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        code = mvt.rvq_encode_noalloc(x, mvt.RVQ_BF16, n, tok.D, tok.codebooks, tok.cb_dtype, tok.operand,
                                      tok.norms, tok.level_stats, tok.L, tok.K, None, 0, ids, res, rec, None,
                                      status)
        assert code == 0, mvt.rvq_status_str(code)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(ids, ids_ref), f"call {batch}: ids differ"
        assert _rel_l2(res, res_ref) <= REL_L2
        assert _rel_l2(rec, rec_ref) <= REL_L2


def test_noalloc_rejects_sizes_beyond_the_scratch():
    g, _ = _features(0, 16)
    tok = mvt.Tokenizer(torch.from_numpy(g["codebooks"]).cuda())
    n = 1 << 16  # needs far more than the static scratch
    code, need = mvt.rvq_encode_workspace_size(n, tok.D, tok.L, tok.K)
    assert code == 0 and need > mvt.RVQ_NOALLOC_SCRATCH_BYTES
    before = mvt.rvq_launch_count()
    code = mvt.rvq_encode_noalloc(16, mvt.RVQ_BF16, n, tok.D, tok.codebooks, tok.cb_dtype, tok.operand, tok.norms,
                                  tok.level_stats, tok.L, tok.K, None, 0, 16, None, None, None, None)
    assert code == -3  # RVQ_ERR_WORKSPACE, rejected before anything is enqueued
    assert mvt.rvq_launch_count() == before
