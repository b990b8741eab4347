"""The fp64 oracle against brute force, library routines, closed forms and invariants."""
import os
import shutil
import subprocess
import tempfile

import pytest

import oracle
from tests import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(oracle.load())


# Plausible mistakes planted in a copy of the oracle source; each must trip a pin.
MUTANTS = {
    "distance_sign": ("double t = r[i] - (double)c[i];", "double t = r[i] + (double)c[i];"),
    "ties_highest": ("if (d < bd) {", "if (d <= bd) {"),
    "residual_sign": ("r[i] = r[i] - (double)c[i];\n                    acc",
                      "r[i] = r[i] + (double)c[i];\n                    acc"),
    "always_level0": ("const float *C_l = C + (size_t)l * K * D;\n                double bd;",
                      "const float *C_l = C;\n                double bd;"),
    "recon_drops_term": ("acc[i] = acc[i] + (double)c[i];", "acc[i] = (double)c[i];"),
    "decode_transposed": ("const float *c = C + ((size_t)l * K + (size_t)id) * D;",
                          "const float *c = C + ((size_t)id * L + (size_t)l) * D;"),
    "skip_first_codeword": ("for (int k = 1; k < K; ++k) {\n        double d = sq_dist(r, C_l + (size_t)k * D, D);",
                            "bd = 1e300;\n    for (int k = 1; k < K; ++k) {\n        double d = sq_dist(r, C_l + (size_t)k * D, D);"),
    "square_dropped": ("s += t * t;", "s += t;"),
    "embed_overwrites": ("for (int i = 0; i < H; ++i) dst[i] = dst[i] + (double)src[i];",
                         "for (int i = 0; i < H; ++i) dst[i] = (double)src[i];"),
    "embed_level0_ids": ("int32_t id = ids[(size_t)n * L + l];", "int32_t id = ids[(size_t)n * L];"),
    "embed_transposed": ("double *dst = grad + ((size_t)l * K + (size_t)id) * H;",
                         "double *dst = grad + ((size_t)id * L + (size_t)l) * H;"),
    "kmeans_no_divide": ("for (int i = 0; i < D; ++i) s[i] = s[i] / (double)count[k];",
                         "for (int i = 0; i < D; ++i) s[i] = s[i];"),
    "kmeans_empty_zero": ("for (int i = 0; i < D; ++i) s[i] = (double)old_cb[(size_t)k * D + i];",
                          "for (int i = 0; i < D; ++i) s[i] = 0.0;"),
    "kmeans_skips_first_row": ("for (int64_t n = 0; n < N; ++n) {\n        int32_t id = ids[n];",
                               "for (int64_t n = 1; n < N; ++n) {\n        int32_t id = ids[n];"),
    "balance_most_loaded": ("if (load[r] < load[best]) best = r;", "if (load[r] > load[best]) best = r;"),
    "balance_increasing": ("while (j >= 0 && lengths[order[j]] < lengths[v]) {",
                           "while (j >= 0 && lengths[order[j]] > lengths[v]) {"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    old, new = MUTANTS[name]
    src = open(os.path.join(os.path.dirname(oracle.__file__), "rvq_oracle.c")).read()
    assert src.count(old) >= 1, f"mutation anchor missing for {name}"
    tmp = tempfile.mkdtemp(prefix="oracle_mutant_")
    try:
        msrc = os.path.join(tmp, "m.c")
        with open(msrc, "w") as f:
            f.write(src.replace(old, new, 1))
        mlib = oracle.build(src=msrc, out=os.path.join(tmp, "m.so"), force=True)
        lib = oracle.load(mlib)
        caught = []
        for pin in oracle_pins.ALL_PINS:
            try:
                pin(lib)
            except (AssertionError, oracle.OracleError):
                caught.append(pin.__name__)
        assert caught, f"mutant {name} passed every pin"
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
