"""rvq_encode_noalloc: the encode entry point for callers that cannot allocate device memory
(a framework that owns every device byte through its own pool, a serving loop that must not
call cudaMalloc because it can synchronize the device, a plugin host that offers no
workspace).  Its scratch is the library's own statically sized device array.

Checked through the C ABI against rvq_encode with a caller workspace, on two calls in a row
(the shared scratch keeps the first call's contents when the second starts), with the
tolerances the parity tests use: ids equal, residual and recon within REL_L2; the ids are also
checked against the fp64 oracle with the parity rule.  Two shapes: image-shaped bf16 features
(all levels in one launch) and fp32 features at D = 512 (one launch per level, whose counters
and operand rows are re-initialised by other kernels).  Kept in a file that pytest collects
last; it passes alone in a fresh process and after the other tests.
"""
import numpy as np
import pytest

import workloads
from tests import parity
from tests.parity import REL_L2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import multimodal_visual_tokenization_b200 as mvt  # noqa: E402


def _image_case(batch, n):
    g = workloads.generate("image", batch=batch, n_override=n)
    return g["codebooks"], g["x"], "bf16"


def _per_level_case(batch, n):
    rng = np.random.Generator(np.random.PCG64([77, batch]))
    L, K, D = 3, 700, 512
    C = np.random.Generator(np.random.PCG64(77)).standard_normal((L, K, D)).astype(np.float32)
    C *= (0.5 ** np.arange(L, dtype=np.float32))[:, None, None]
    x = (C[0][rng.integers(0, K, n)] + 0.3 * rng.standard_normal((n, D))).astype(np.float32)
    return C, x, "f32"


def _rel_l2(a, b):
    a = a.double()
    b = b.double()
    return float(((a - b).norm(dim=1) / b.norm(dim=1).clamp_min(1e-30)).max())


@pytest.mark.parametrize("make,n,levels_per_launch", [(_image_case, 1024, "all"), (_per_level_case, 600, 1)])
def test_noalloc_matches_workspace_encode_on_two_calls(make, n, levels_per_launch):
    C, _, _ = make(0, n)
    tok = mvt.Tokenizer(torch.from_numpy(C).cuda())
    code, need = mvt.rvq_encode_workspace_size(n, tok.D, tok.L, tok.K)
    assert code == 0 and need <= mvt.RVQ_NOALLOC_SCRATCH_BYTES
    code, lpl = mvt.rvq_encode_levels_per_launch(n, tok.D, tok.L, tok.K)
    assert code == 0 and lpl == (tok.L if levels_per_launch == "all" else levels_per_launch)
    for batch in (0, 1):
        _, xh, fd = make(batch, n)
        x = torch.from_numpy(xh).cuda()
        if fd == "bf16":
            x = x.to(torch.bfloat16)
        ids_ref, res_ref, rec_ref = tok.encode(x, residual=True, recon=True)
        ids = torch.full((n, tok.L), -1, dtype=torch.int32, device="cuda")
        res = torch.empty((n, tok.D), dtype=torch.float32, device="cuda")
        rec = torch.empty((n, tok.D), dtype=torch.float32, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        code = mvt.rvq_encode_noalloc(x, mvt._dtype_code(x), n, tok.D, tok.codebooks, tok.cb_dtype, tok.operand,
                                      tok.norms, tok.level_stats, tok.L, tok.K, None, 0, ids, res, rec, None,
                                      status)
        assert code == 0, mvt.rvq_status_str(code)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(ids, ids_ref), f"call {batch}: ids differ"
        assert _rel_l2(res, res_ref) <= REL_L2
        assert _rel_l2(rec, rec_ref) <= REL_L2
        rows = workloads.sample_rows(n, 64, seed=batch)
        parity.check_ids(xh, C, rows, ids.cpu().numpy())


def test_noalloc_rejects_sizes_beyond_the_scratch():
    C, _, _ = _image_case(0, 16)
    tok = mvt.Tokenizer(torch.from_numpy(C).cuda())
    n = 1 << 16  # needs far more than the static scratch
    code, need = mvt.rvq_encode_workspace_size(n, tok.D, tok.L, tok.K)
    assert code == 0 and need > mvt.RVQ_NOALLOC_SCRATCH_BYTES
    before = mvt.rvq_launch_count()
    code = mvt.rvq_encode_noalloc(16, mvt.RVQ_BF16, n, tok.D, tok.codebooks, tok.cb_dtype, tok.operand, tok.norms,
                                  tok.level_stats, tok.L, tok.K, None, 0, 16, None, None, None, None)
    assert code == -3  # RVQ_ERR_WORKSPACE, rejected before anything is enqueued
    assert mvt.rvq_launch_count() == before
