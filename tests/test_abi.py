"""librvq.so loads, exports every entry point include/rvq.h declares, and rejects bad
arguments on the host before touching the GPU (no compute calls here)."""
import ctypes
import os
import re

import pytest

import multimodal_visual_tokenization_b200 as mvt
from multimodal_visual_tokenization_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"RVQ_API\s+[\w\s\*]*?\b(rvq_\w+)\s*\(", src)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return mvt.load()


def test_header_declares_the_abi():
    names = declared_symbols()
    assert set(mvt.EXPORTS) == set(names), names


def test_every_declared_symbol_is_exported(lib):
    raw = ctypes.CDLL(mvt.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(raw, name), f"{name} not exported"


def test_binding_names_match(lib):
    for name in declared_symbols():
        assert callable(getattr(mvt, name)), name


def test_status_strings(lib):
    for code, name in mvt.STATUS.items():
        assert mvt.rvq_status_str(code).startswith(name)
    assert "unknown" in mvt.rvq_status_str(12345)


def test_host_argument_checks(lib):
    L = lib
    # null codebooks / bad dtype / unsupported D: rejected before any CUDA call
    assert L.rvq_build_norms(None, 0, 2, 8, 64, None, None, None, None) == -1
    assert L.rvq_build_norms(16, 7, 2, 8, 64, 16, 16, 16, None) == -1
    assert L.rvq_build_norms(16, 0, 2, 8, 40, 16, 16, 16, None) == -2
    assert L.rvq_build_norms(16, 0, 2, 8, 64, 16, 16, None, None) == -1      # fp32 needs operand copy
    assert L.rvq_decode(16, 0, 2, 16, 0, 8, 64, 16, None, None) == 0        # N = 0: no-op
    assert L.rvq_decode(None, 5, 2, 16, 0, 8, 64, 16, None, None) == -1
    assert L.rvq_decode(16, 5, 2, 16, 0, 8, 66, 16, None, None) == -2        # D % 4
    assert L.rvq_decode(16, 5, 65, 16, 0, 8, 64, 16, None, None) == -2       # L > 64
    enc = L.rvq_encode
    args = [16, 0, 0, 64, 16, 0, 16, 16, 16, 2, 8, None, 0, 16, None, None, None, 256, 1 << 20, None, None]
    assert enc(*args) == 0                                                   # N = 0: no-op
    bad_d = list(args); bad_d[2] = 5; bad_d[3] = 96
    assert enc(*bad_d) == -2                                                 # D % 64
    bad_off = list(args); bad_off[2] = 5; bad_off[12] = 3
    assert enc(*bad_off) == -1                                               # B without offsets
    no_ws = list(args); no_ws[2] = 5; no_ws[17] = None
    assert enc(*no_ws) == -3
    mis = list(args); mis[2] = 5; mis[0] = 18
    assert enc(*mis) == -1                                                   # misaligned features
    lv = ctypes.c_int32(0)
    assert L.rvq_encode_levels_per_launch(100, 1024, 4, 8192, None) == -1    # no output
    assert L.rvq_encode_levels_per_launch(100, 1000, 4, 8192, ctypes.byref(lv)) == -2   # D % 64
    assert L.rvq_encode_levels_per_launch(100, 1024, 65, 8192, ctypes.byref(lv)) == -2  # L > 64
    eb = L.rvq_embed_backward
    assert eb(16, 0, 2, 8, 64, 16, 16, None, None) == 0                        # N = 0: no-op
    assert eb(None, 5, 2, 8, 64, 16, 16, None, None) == -1                     # no ids
    assert eb(16, 5, 65, 8, 64, 16, 16, None, None) == -2                      # L > 64
    assert eb(16, 5, 2, 8, 6, 16, 16, None, None) == -2                        # H % 4
    assert eb(16, 5, 2, 8, 64, 24, 16, None, None) == -1                       # misaligned grad_out
    cu = L.rvq_codebook_update
    assert cu(16, 16, 5, 6, 8, 16, 16, 16, 16, None, None) == -2               # D % 4
    assert cu(16, 16, 5, 64, 8, None, 16, 16, 16, None, None) == -1            # no old codebook
    assert cu(24, 16, 5, 64, 8, 16, 16, 16, 16, None, None) == -1              # misaligned points
    assert L.rvq_gather_sequences(16, 0, 16, 1, 16, 1, 16, 16, None, None) == -1   # L < 1
    assert L.rvq_gather_sequences(16, 8, 16, 1, 16, 0, 16, 16, None, None) == 0    # M = 0: no-op
    assert L.rvq_gather_sequences(None, 8, 16, 1, 16, 1, 16, 16, None, None) == -1 # no cache
    assert L.rvq_selftest_wait_timeout(None, 16, 1000, None) == -1               # no counter
    assert L.rvq_selftest_wait_timeout(16, 16, 0, None) == -1                  # limit out of range


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError):
        mvt._lib_backup = mvt._lib
        try:
            mvt._lib = None
            mvt.load(str(tmp_path / "nope.so"))
        finally:
            mvt._lib = mvt._lib_backup
