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
    off, slots = ctypes.c_size_t(0), ctypes.c_int32(0)
    assert L.rvq_encode_candidate_layout(100, 1024, 4, 8192, None, ctypes.byref(slots)) == -1
    assert L.rvq_encode_candidate_layout(-1, 1024, 4, 8192, ctypes.byref(off), ctypes.byref(slots)) == -1
    assert L.rvq_encode_candidate_layout(100, 96, 4, 8192, ctypes.byref(off), ctypes.byref(slots)) == -2
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
    sz = ctypes.c_size_t(0)
    assert L.rvq_shard_workspace_size(100, 1024, 4096, None) == -1             # no output
    assert L.rvq_shard_workspace_size(100, 2048, 4096, ctypes.byref(sz)) == -2  # D > 1024
    assert L.rvq_shard_workspace_size(100, 96, 4096, ctypes.byref(sz)) == -2   # D % 64
    sel = L.rvq_shard_select
    sargs = [16, 0, 0, 64, 16, 0, 16, 16, 16, 2, 8, 0, 0, None, 16, None, 256, 1 << 20, None, None]
    assert sel(*sargs) == 0                                                    # N = 0: no-op
    s1 = list(sargs); s1[12] = 2
    assert sel(*s1) == -1                                                      # level l >= L
    s2 = list(sargs); s2[2] = 5; s2[6] = None
    assert sel(*s2) == -1                                                      # fp32 shard needs operand copy
    s3 = list(sargs); s3[2] = 5; s3[3] = 2048
    assert sel(*s3) == -2                                                      # D > 1024
    s4 = list(sargs); s4[2] = 5; s4[16] = None
    assert sel(*s4) == -3                                                      # no workspace
    s5 = list(sargs); s5[2] = 5; s5[14] = 24
    assert sel(*s5) == -1                                                      # misaligned sel
    s6 = list(sargs); s6[11] = -1
    assert sel(*s6) == -1                                                      # negative first id
    app = L.rvq_shard_apply
    vp2 = (ctypes.c_void_p * 2)(16, 32)
    k2 = (ctypes.c_int * 2)(8, 8)
    aargs = [16, 0, 0, 64, 16, 2, vp2, 0, k2, 2, 0, 16, None, 256, 1 << 20, None, None]
    assert app(*aargs) == 0                                                    # N = 0: no-op
    a1 = list(aargs); a1[5] = 0
    assert app(*a1) == -1                                                      # no shards
    a2 = list(aargs); a2[5] = 17
    assert app(*a2) == -2                                                      # above RVQ_MAX_SHARDS
    a3 = list(aargs); a3[8] = (ctypes.c_int * 2)(8, 0)
    assert app(*a3) == -1                                                      # empty shard
    a4 = list(aargs); a4[6] = (ctypes.c_void_p * 2)(16, 40)
    assert app(*a4) == -1                                                      # misaligned peer pointer
    a5 = list(aargs); a5[2] = 5; a5[14] = 100
    assert app(*a5) == -3                                                      # workspace below the row state
    a6 = list(aargs); a6[10] = 2
    assert app(*a6) == -1                                                      # level l >= L
    off = ctypes.c_size_t(0)
    h = ctypes.create_string_buffer(mvt.RVQ_IPC_HANDLE_BYTES)
    assert L.rvq_ipc_export(None, h, ctypes.byref(off)) == -1
    assert L.rvq_ipc_import(None, 0, ctypes.byref(ctypes.c_void_p())) == -1
    assert L.rvq_ipc_close(None, 0) == -1
    assert L.rvq_embed_backward_workspace_size(10, 2, 8, 16, None) == -1
    assert L.rvq_embed_backward_workspace_size(10, 2, 49152, 16, ctypes.byref(sz)) == -2     # K too large
    assert L.rvq_embed_backward_workspace_size(10, 2, 8, 18, ctypes.byref(sz)) == -2         # H % 4
    assert L.rvq_embed_backward_workspace_size(10, 2, 8, 16, ctypes.byref(sz)) == 0 and sz.value > 0
    ebs = L.rvq_embed_backward_sorted
    assert ebs(16, 0, 2, 8, 16, 16, 16, None, 0, None, None) == 0                           # N = 0: no-op
    assert ebs(None, 5, 2, 8, 16, 16, 16, 256, 1 << 20, None, None) == -1                   # no ids
    assert ebs(16, 5, 2, 8, 16, 16, 16, None, 0, None, None) == -3                          # no workspace
    assert ebs(16, 5, 2, 8, 16, 16, 16, 256, 100, None, None) == -3                         # too small


@pytest.mark.parametrize("L,K,D,dt,want_rpw,want_cols", [
    (8, 16384, 1024, "bf16", 1, 256),   # detok: 8 x 16384 x 256 bf16 columns = 64 MiB live
    (8, 16384, 1024, "f32", 1, 128),    # packed: 64 MiB
    (4, 8192, 1024, "f32", 1, 128),     # image: 16 MiB
    (4, 65536, 256, "f32", 2, 64),      # offline: 128 MiB at 128 columns, 64 MiB at 64
    (8, 65536, 128, "f32", 4, 32),      # 256 MiB -> 128 -> 64 MiB
    (8, 65536, 256, "bf16", 4, 64),     # bf16, 16-byte gathers
    (12, 32768, 132, "bf16", 2, 64),    # D % 8 != 0: 8-byte gathers; 12 levels fit 16 lanes, not 8
    (16, 65536, 256, "f32", 2, 64),     # 16 levels: at most two rows per warp
    (20, 65536, 256, "f32", 1, 128),    # more than 16 levels: the generic kernel, one row per warp
    (1, 7, 256, "bf16", 1, 256),
])
def test_decode_slice_plan(lib, L, K, D, dt, want_rpw, want_cols):
    """The rows-per-warp choice of rvq_decode: the widest slice whose live codebook columns
    (L * K * columns * element size) stay within 64 MiB, as narrow as a row's ids allow."""
    code, rpw, cols = mvt.rvq_decode_slice_plan(L, K, D, mvt.RVQ_BF16 if dt == "bf16" else mvt.RVQ_F32)
    assert code == 0 and (rpw, cols) == (want_rpw, want_cols)
    el = 2 if dt == "bf16" else 4
    if L <= 16:
        lanes = 32 // rpw
        assert L <= lanes
        live = L * K * cols * el
        narrower_allowed = rpw < 4 and L <= lanes // 2
        assert live <= 64 << 20 or not narrower_allowed
        if rpw > 1:  # one step wider would have exceeded the budget
            assert L * K * (cols * 2) * el > 64 << 20


def test_decode_slice_plan_argument_checks(lib):
    i32 = ctypes.c_int32
    a, b = i32(0), i32(0)
    assert lib.rvq_decode_slice_plan(8, 16384, 1024, 1, None, ctypes.byref(b)) == -1
    assert lib.rvq_decode_slice_plan(0, 16384, 1024, 1, ctypes.byref(a), ctypes.byref(b)) == -1
    assert lib.rvq_decode_slice_plan(8, 16384, 1024, 7, ctypes.byref(a), ctypes.byref(b)) == -1
    assert lib.rvq_decode_slice_plan(8, 16384, 1022, 1, ctypes.byref(a), ctypes.byref(b)) == -2
    assert lib.rvq_decode_slice_plan(65, 16384, 1024, 1, ctypes.byref(a), ctypes.byref(b)) == -2


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    """No CPU fallback: without librvq.so the binding raises instead of running anything else."""
    monkeypatch.setattr(mvt, "_lib", None)
    monkeypatch.setattr(mvt, "LIB_PATH", str(tmp_path / "nope.so"))
    with pytest.raises(RuntimeError):
        mvt.load()
