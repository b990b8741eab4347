"""Comparison of the CUDA path's outputs with the fp64 oracle.

Rule for ids (greedy RVQ has one correct answer per level except at exact ties, and a
legitimate near-tie can send two encoders down different residual paths):
  * the oracle, driven by the GPU's own ids, forms every level's full distance vector
    (teacher forcing: the residual at level l is x minus the GPU's codewords of levels < l);
  * the GPU id must be that vector's argmin (lowest index on ties), except where the
    oracle's best-vs-second gap is below REL_GAP relative, and there the GPU's chosen
    distance must be within REL_GAP relative of the minimum (an exact 0 minimum needs 0).
  * the free-running oracle ids are also compared; rows that differ must have taken an
    exemption at the first level where they differ.  A row whose every level matched the
    teacher-forced argmin is on the free-running path by construction (same residual, same
    argmin, level by level, in the same fp64 arithmetic), so only rows with an exemption are
    re-encoded free-running.
Reconstructions: ||recon_gpu - recon_oracle(ids_gpu)|| <= REL_L2 * ||recon_oracle|| per row,
and the residual within REL_L2 * ||x|| of x - recon_oracle(ids_gpu).  fp32 accumulation of
L <= 16 codewords carries a relative error of a few 1e-7, so 1e-5 has ample headroom.
"""
from __future__ import annotations

import numpy as np

import oracle

REL_GAP = 1e-6
REL_L2 = 1e-5


def check_ids(x, C, rows, ids_gpu, threads=0):
    """Returns a report dict; raises AssertionError on a violation."""
    rows = np.asarray(rows, np.int64)
    g = np.ascontiguousarray(ids_gpu[rows], np.int32)
    K = C.shape[1]
    assert g.min() >= 0 and g.max() < K, "GPU id outside [0, K)"
    tf = oracle.check_path(x, C, rows, g, threads=threads)
    match = g == tf["argmin"]
    best, second, chosen = tf["best"], tf["second"], tf["chosen"]
    denom = np.maximum(best, 1e-30)
    near_tie = (second - best) / denom < REL_GAP
    close = np.where(best == 0, chosen == 0, chosen <= best * (1 + REL_GAP))
    exempt = ~match & near_tie & close
    bad = ~match & ~exempt
    if bad.any():
        j, l = np.argwhere(bad)[0]
        raise AssertionError(
            f"row {rows[j]} level {l}: gpu id {g[j, l]} (d={chosen[j, l]!r}) but oracle argmin "
            f"{tf['argmin'][j, l]} (d={best[j, l]!r}, second={second[j, l]!r}); "
            f"{int(bad.sum())} violations in {bad.size} row-levels")
    differ = np.zeros_like(g, dtype=bool)
    touched = np.where(exempt.any(axis=1))[0]
    if touched.size:
        free, _, _, _ = oracle.encode(x, C, rows=rows[touched], threads=threads)
        differ[touched] = free != g[touched]
    first_diff_ok = True
    for j in np.where(differ.any(axis=1))[0]:
        l = int(np.argmax(differ[j]))
        first_diff_ok &= bool(exempt[j, l])
    assert first_diff_ok, "GPU left the oracle's path at a level without a near-tie"
    return {"row_levels": int(g.size), "exact": int(match.sum()), "exempt": int(exempt.sum()),
            "rows_equal_free_running": int((~differ.any(axis=1)).sum()), "rows": int(len(rows))}


def check_recon(x, C, rows, ids_gpu, recon_gpu=None, residual_gpu=None, threads=0):
    rows = np.asarray(rows, np.int64)
    ids = np.ascontiguousarray(ids_gpu[rows], np.int32)
    ref = oracle.decode(ids, C, threads=threads)
    out = {}
    if recon_gpu is not None:
        rg = np.asarray(recon_gpu[rows], np.float64)
        err = np.linalg.norm(rg - ref, axis=1) / np.maximum(np.linalg.norm(ref, axis=1), 1e-30)
        assert (err <= REL_L2).all(), f"recon rel L2 {err.max():.3g} > {REL_L2}"
        out["recon_rel_l2_max"] = float(err.max())
    if residual_gpu is not None and x is not None:
        xs = np.asarray(x[rows], np.float64)
        want = xs - ref
        rg = np.asarray(residual_gpu[rows], np.float64)
        err = np.linalg.norm(rg - want, axis=1) / np.maximum(np.linalg.norm(xs, axis=1), 1e-30)
        assert (err <= REL_L2).all(), f"residual rel L2 {err.max():.3g} > {REL_L2}"
        out["residual_rel_l2_max"] = float(err.max())
    return out


def check_all_rows(x, ids_gpu, K, recon_gpu=None, residual_gpu=None):
    """Properties that hold at any size, checked on every row."""
    assert ids_gpu.min() >= 0 and ids_gpu.max() < K
    if recon_gpu is not None and residual_gpu is not None and x is not None:
        s = recon_gpu.astype(np.float64) + residual_gpu.astype(np.float64)
        err = np.linalg.norm(s - x, axis=1) / np.maximum(np.linalg.norm(x, axis=1), 1e-30)
        assert (err <= REL_L2).all(), f"recon + residual != x: {err.max():.3g}"
        return float(err.max())
    return None
