"""Python binding of librvq.so: residual vector quantization (RVQ) of visual features
into multi-level discrete token ids and the gather-sum decode, on one B200 (sm_100a).

The functions named ``rvq_*`` mirror the C ABI in include/rvq.h one to one: they only
marshal arguments (torch tensors -> device pointers, dtype codes, the current CUDA stream)
and return the library's status.  Every step of the computation runs in the library's
CUDA kernels; there is no Python or CPU fallback, and loading fails loudly when the
library is missing.

``Tokenizer`` is the convenience layer a user calls: it holds a fixed codebook set with
its prepared norms/operand copy (the pages' "fixed tokenizer"), and its ``encode`` /
``decode`` allocate outputs with torch and call the C entry points.

Usage (one GPU)::

    tok = Tokenizer(codebooks)                 # [L, K, D] float32 or bfloat16, on the GPU
    ids, residual, recon = tok.encode(x, residual=True, recon=True)   # x [N, D]
    feats = tok.decode(ids)                    # [N, D] float32 = sum_l C_l[ids[:, l]]

Other entry points:
* ``rvq_embed_backward`` (fp32 atomics) / ``rvq_embed_backward_sorted`` (bit-reproducible, with a
  workspace): gradient of an embedding e[n] = sum_l E_l[ids[n, l]] with respect to its tables.
* ``rvq_codebook_update``: one k-means step of a codebook level.
* ``rvq_balance_sequences`` / ``rvq_gather_sequences``: packing id sequences for data-parallel
  ranks.
* ``sharded.ShardedTokenizer``: the codebook axis split over the ranks of a process group.
* Queries and measurement hooks: ``rvq_encode_levels_per_launch``, ``rvq_encode_candidate_layout``,
  ``rvq_decode_slice_plan``, ``rvq_launch_count``, ``rvq_profile_enable`` / ``rvq_profile_read``.
"""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "librvq.so")

RVQ_F32, RVQ_BF16 = 0, 1
RVQ_LEVEL_STATS = 4
STATUS = {0: "RVQ_OK", -1: "RVQ_ERR_ARG", -2: "RVQ_ERR_UNSUPPORTED", -3: "RVQ_ERR_WORKSPACE",
          -4: "RVQ_ERR_CUDA", -5: "RVQ_ERR_ID_RANGE", -6: "RVQ_ERR_TIMEOUT"}

EXPORTS = ("rvq_build_norms", "rvq_encode_workspace_size", "rvq_encode", "rvq_decode",
           "rvq_status_str", "rvq_launch_count", "rvq_profile_enable", "rvq_profile_read",
           "rvq_encode_levels_per_launch", "rvq_selftest_wait_timeout", "rvq_embed_backward",
           "rvq_codebook_update", "rvq_balance_sequences", "rvq_gather_sequences",
           "rvq_encode_noalloc", "rvq_shard_workspace_size", "rvq_shard_select", "rvq_shard_apply",
           "rvq_ipc_export", "rvq_ipc_import", "rvq_ipc_close", "rvq_embed_backward_workspace_size",
           "rvq_embed_backward_sorted", "rvq_encode_candidate_layout", "rvq_decode_slice_plan")
RVQ_MAX_SHARDS = 16
RVQ_IPC_HANDLE_BYTES = 64
RVQ_NOALLOC_SCRATCH_BYTES = 32 << 20

_lib = None
_lock = threading.Lock()


class RVQError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        super().__init__(f"{what}: {STATUS.get(code, code)}" if what else STATUS.get(code, str(code)))
        self.code = code


def load():
    """Load librvq.so (built in-tree by `python -m multimodal_visual_tokenization_b200._build`)."""
    global _lib
    path = LIB_PATH
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(f"librvq.so not found at {path}; build it with "
                               "`python -m multimodal_visual_tokenization_b200._build`")
        lib = ctypes.CDLL(path)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
        lib.rvq_build_norms.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp]
        lib.rvq_encode_workspace_size.argtypes = [i64, i32, i32, i32, ctypes.POINTER(sz)]
        lib.rvq_encode.argtypes = [vp, i32, i64, i32, vp, i32, vp, vp, vp, i32, i32, vp, i64,
                                   vp, vp, vp, vp, vp, sz, vp, vp]
        lib.rvq_decode.argtypes = [vp, i64, i32, vp, i32, i32, i32, vp, vp, vp]
        lib.rvq_encode_noalloc.argtypes = [vp, i32, i64, i32, vp, i32, vp, vp, vp, i32, i32, vp, i64,
                                           vp, vp, vp, vp, vp, vp]
        lib.rvq_status_str.argtypes = [i32]
        lib.rvq_status_str.restype = ctypes.c_char_p
        lib.rvq_launch_count.argtypes = []
        lib.rvq_launch_count.restype = ctypes.c_int64
        lib.rvq_profile_enable.argtypes = [i32]
        lib.rvq_profile_read.argtypes = [ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_double)]
        lib.rvq_encode_levels_per_launch.argtypes = [i64, i32, i32, i32, ctypes.POINTER(i32)]
        lib.rvq_encode_candidate_layout.argtypes = [i64, i32, i32, i32, ctypes.POINTER(sz), ctypes.POINTER(i32)]
        lib.rvq_decode_slice_plan.argtypes = [i32, i32, i32, i32, ctypes.POINTER(i32), ctypes.POINTER(i32)]
        lib.rvq_selftest_wait_timeout.argtypes = [vp, vp, i64, vp]
        lib.rvq_embed_backward.argtypes = [vp, i64, i32, i32, i32, vp, vp, vp, vp]
        lib.rvq_codebook_update.argtypes = [vp, vp, i64, i32, i32, vp, vp, vp, vp, vp, vp]
        lib.rvq_balance_sequences.argtypes = [vp, i64, i32, vp, vp]
        lib.rvq_gather_sequences.argtypes = [vp, i32, vp, i64, vp, i64, vp, vp, vp, vp]
        lib.rvq_shard_workspace_size.argtypes = [i64, i32, i32, ctypes.POINTER(sz)]
        lib.rvq_shard_select.argtypes = [vp, i32, i64, i32, vp, i32, vp, vp, vp, i32, i32, i64, i32, vp,
                                         vp, vp, vp, sz, vp, vp]
        lib.rvq_shard_apply.argtypes = [vp, i32, i64, i32, vp, i32, ctypes.POINTER(vp), i32,
                                        ctypes.POINTER(i32), i32, i32, vp, vp, vp, sz, vp, vp]
        lib.rvq_ipc_export.argtypes = [vp, vp, ctypes.POINTER(sz)]
        lib.rvq_ipc_import.argtypes = [vp, sz, ctypes.POINTER(vp)]
        lib.rvq_ipc_close.argtypes = [vp, sz]
        lib.rvq_embed_backward_workspace_size.argtypes = [i64, i32, i32, i32, ctypes.POINTER(sz)]
        lib.rvq_embed_backward_sorted.argtypes = [vp, i64, i32, i32, i32, vp, vp, vp, sz, vp, vp]
        for fn in ("rvq_build_norms", "rvq_encode_workspace_size", "rvq_encode", "rvq_decode",
                   "rvq_profile_enable", "rvq_profile_read", "rvq_encode_noalloc",
                   "rvq_encode_levels_per_launch", "rvq_selftest_wait_timeout", "rvq_embed_backward",
                   "rvq_codebook_update", "rvq_balance_sequences", "rvq_gather_sequences",
                   "rvq_shard_workspace_size", "rvq_shard_select", "rvq_shard_apply", "rvq_ipc_export",
                   "rvq_ipc_import", "rvq_ipc_close", "rvq_embed_backward_workspace_size",
                   "rvq_embed_backward_sorted", "rvq_encode_candidate_layout", "rvq_decode_slice_plan"):
            getattr(lib, fn).restype = ctypes.c_int
        _lib = lib
        return lib


# ------------------------------------------------------------------ marshalling helpers

def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _dtype_code(t):
    import torch
    if t.dtype == torch.float32:
        return RVQ_F32
    if t.dtype == torch.bfloat16:
        return RVQ_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; expected float32 or bfloat16")


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _check(code, what):
    if code != 0:
        raise RVQError(code, what)
    return code


# ------------------------------------------------------------------ the C ABI, one to one

def rvq_build_norms(codebooks, cb_dtype, L, K, D, norms, level_stats, cb_operand, stream=None):
    return load().rvq_build_norms(_ptr(codebooks), cb_dtype, L, K, D, _ptr(norms), _ptr(level_stats),
                                  _ptr(cb_operand), _stream(stream))


def rvq_encode_workspace_size(N, D, L, K):
    out = ctypes.c_size_t(0)
    code = load().rvq_encode_workspace_size(N, D, L, K, ctypes.byref(out))
    return code, out.value


def rvq_encode(features, f_dtype, N, D, codebooks, cb_dtype, cb_operand, norms, level_stats, L, K,
               offsets, B, ids, residual, recon, fallbacks, workspace, workspace_bytes, status,
               stream=None):
    return load().rvq_encode(_ptr(features), f_dtype, N, D, _ptr(codebooks), cb_dtype, _ptr(cb_operand),
                             _ptr(norms), _ptr(level_stats), L, K, _ptr(offsets), B, _ptr(ids),
                             _ptr(residual), _ptr(recon), _ptr(fallbacks), _ptr(workspace),
                             workspace_bytes, _ptr(status), _stream(stream))


def rvq_encode_noalloc(features, f_dtype, N, D, codebooks, cb_dtype, cb_operand, norms, level_stats, L, K,
                       offsets, B, ids, residual, recon, fallbacks, status, stream=None):
    """rvq_encode without a workspace argument, for callers that cannot allocate device memory:
    the library's own statically sized scratch array (RVQ_NOALLOC_SCRATCH_BYTES) is used."""
    return load().rvq_encode_noalloc(_ptr(features), f_dtype, N, D, _ptr(codebooks), cb_dtype,
                                     _ptr(cb_operand), _ptr(norms), _ptr(level_stats), L, K, _ptr(offsets),
                                     B, _ptr(ids), _ptr(residual), _ptr(recon), _ptr(fallbacks),
                                     _ptr(status), _stream(stream))


def rvq_decode(ids, N, L, codebooks, cb_dtype, K, D, recon, status, stream=None):
    return load().rvq_decode(_ptr(ids), N, L, _ptr(codebooks), cb_dtype, K, D, _ptr(recon), _ptr(status),
                             _stream(stream))


def rvq_status_str(status):
    return load().rvq_status_str(status).decode()


def rvq_launch_count():
    return load().rvq_launch_count()


def rvq_profile_enable(enable):
    return load().rvq_profile_enable(1 if enable else 0)


def rvq_profile_read():
    n = ctypes.c_int64(0)
    ms = ctypes.c_double(0.0)
    code = load().rvq_profile_read(ctypes.byref(n), ctypes.byref(ms))
    return code, n.value, ms.value


def rvq_encode_levels_per_launch(N, D, L, K):
    lv = ctypes.c_int32(0)
    code = load().rvq_encode_levels_per_launch(int(N), int(D), int(L), int(K), ctypes.byref(lv))
    return code, lv.value


def rvq_encode_candidate_layout(N, D, L, K):
    """-> (status, byte offset of the candidate lists in the encode workspace, slots per row tile)."""
    off = ctypes.c_size_t(0)
    slots = ctypes.c_int32(0)
    code = load().rvq_encode_candidate_layout(int(N), int(D), int(L), int(K), ctypes.byref(off), ctypes.byref(slots))
    return code, off.value, slots.value


def rvq_decode_slice_plan(L, K, D, cb_dtype):
    """-> (status, rows per warp, columns per slice) that rvq_decode uses for this shape."""
    rpw = ctypes.c_int32(0)
    cols = ctypes.c_int32(0)
    code = load().rvq_decode_slice_plan(int(L), int(K), int(D), int(cb_dtype), ctypes.byref(rpw), ctypes.byref(cols))
    return code, rpw.value, cols.value


def rvq_embed_backward(ids, N, L, K, H, grad_out, grad_tables, status=None, stream=None):
    return load().rvq_embed_backward(_ptr(ids), int(N), int(L), int(K), int(H), _ptr(grad_out), _ptr(grad_tables),
                                     _ptr(status), _stream(stream))


def rvq_embed_backward_workspace_size(N, L, K, H):
    out = ctypes.c_size_t(0)
    code = load().rvq_embed_backward_workspace_size(N, L, K, H, ctypes.byref(out))
    return code, out.value


def rvq_embed_backward_sorted(ids, N, L, K, H, grad_out, grad_tables, workspace, workspace_bytes, status=None,
                              stream=None):
    return load().rvq_embed_backward_sorted(_ptr(ids), N, L, K, H, _ptr(grad_out), _ptr(grad_tables),
                                            _ptr(workspace), workspace_bytes, _ptr(status), _stream(stream))


def rvq_codebook_update(points, ids, N, D, K, old_codebook, new_codebook, sums, counts, status=None, stream=None):
    return load().rvq_codebook_update(_ptr(points), _ptr(ids), int(N), int(D), int(K), _ptr(old_codebook),
                                      _ptr(new_codebook), _ptr(sums), _ptr(counts), _ptr(status), _stream(stream))


def rvq_balance_sequences(lengths, world):
    """Host call: lengths is a sequence of token counts; returns (code, owner [S] int32, load [world] int64)."""
    import numpy as np
    lengths = np.ascontiguousarray(lengths, dtype=np.int64)
    owner = np.empty(lengths.shape[0], np.int32)
    load_ = np.empty(int(world), np.int64)
    code = load().rvq_balance_sequences(lengths.ctypes.data if lengths.size else None, lengths.shape[0], int(world),
                                        owner.ctypes.data, load_.ctypes.data)
    return code, owner, load_


def rvq_gather_sequences(cache_ids, L, cache_offsets, S, select, M, out_offsets, out_ids, status=None, stream=None):
    return load().rvq_gather_sequences(_ptr(cache_ids), int(L), _ptr(cache_offsets), int(S), _ptr(select), int(M),
                                       _ptr(out_offsets), _ptr(out_ids), _ptr(status), _stream(stream))


def rvq_shard_workspace_size(N, D, K_shard):
    out = ctypes.c_size_t(0)
    code = load().rvq_shard_workspace_size(N, D, K_shard, ctypes.byref(out))
    return code, out.value


def rvq_shard_select(features, f_dtype, N, D, shard_codebooks, cb_dtype, shard_operand, shard_norms, shard_stats,
                     L, K_shard, k0, l, residual, sel, fallbacks, workspace, workspace_bytes, status=None,
                     stream=None):
    return load().rvq_shard_select(_ptr(features), f_dtype, N, D, _ptr(shard_codebooks), cb_dtype,
                                   _ptr(shard_operand), _ptr(shard_norms), _ptr(shard_stats), L, K_shard, k0, l,
                                   _ptr(residual), _ptr(sel), _ptr(fallbacks), _ptr(workspace), workspace_bytes,
                                   _ptr(status), _stream(stream))


def rvq_shard_apply(features, f_dtype, N, D, sel_all, W, shard_codebooks, cb_dtype, shard_K, L, l, ids, residual,
                    workspace, workspace_bytes, status=None, stream=None):
    """shard_codebooks: W device pointers (ints or tensors); shard_K: W codeword counts (host)."""
    ptrs = (ctypes.c_void_p * max(W, 1))(*[_ptr(p) for p in shard_codebooks])
    ks = (ctypes.c_int * max(W, 1))(*[int(k) for k in shard_K])
    return load().rvq_shard_apply(_ptr(features), f_dtype, N, D, _ptr(sel_all), W, ptrs, cb_dtype, ks, L, l,
                                  _ptr(ids), _ptr(residual), _ptr(workspace), workspace_bytes, _ptr(status),
                                  _stream(stream))


def rvq_ipc_export(ptr):
    """-> (status, handle bytes, offset) of the device allocation holding ptr."""
    h = ctypes.create_string_buffer(RVQ_IPC_HANDLE_BYTES)
    off = ctypes.c_size_t(0)
    code = load().rvq_ipc_export(_ptr(ptr), h, ctypes.byref(off))
    return code, h.raw, off.value


def rvq_ipc_import(handle, offset):
    """-> (status, device pointer as int) mapping another process's allocation."""
    if len(handle) != RVQ_IPC_HANDLE_BYTES:
        raise ValueError("IPC handle must be RVQ_IPC_HANDLE_BYTES bytes")
    h = ctypes.create_string_buffer(bytes(handle), RVQ_IPC_HANDLE_BYTES)
    out = ctypes.c_void_p(None)
    code = load().rvq_ipc_import(h, int(offset), ctypes.byref(out))
    return code, (out.value or 0)


def rvq_ipc_close(ptr, offset):
    return load().rvq_ipc_close(_ptr(ptr), int(offset))


def rvq_selftest_wait_timeout(counter, status, limit_us, stream=None):
    return load().rvq_selftest_wait_timeout(_ptr(counter), _ptr(status), int(limit_us), _stream(stream))


# ------------------------------------------------------------------ convenience layer

class Tokenizer:
    """A fixed RVQ codebook set resident on the GPU, with its prepared norms / operand copy.

    codebooks: torch tensor [L, K, D] (float32 or bfloat16) on a CUDA device.
    """

    def __init__(self, codebooks, stream=None):
        import torch
        if not codebooks.is_cuda or codebooks.dim() != 3:
            raise ValueError("codebooks must be a CUDA tensor [L, K, D]")
        self.codebooks = codebooks.contiguous()
        self.L, self.K, self.D = (int(v) for v in self.codebooks.shape)
        self.cb_dtype = _dtype_code(self.codebooks)
        dev = self.codebooks.device
        self.norms = torch.empty((self.L, self.K), dtype=torch.float32, device=dev)
        self.level_stats = torch.empty((self.L, RVQ_LEVEL_STATS), dtype=torch.float32, device=dev)
        self.operand = (torch.empty_like(self.codebooks, dtype=torch.bfloat16)
                        if self.cb_dtype == RVQ_F32 else None)
        self._ws = None
        self.prepare(stream)

    def prepare(self, stream=None):
        """(Re)compute norms, level statistics and the bf16 operand copy (rvq_build_norms)."""
        _check(rvq_build_norms(self.codebooks, self.cb_dtype, self.L, self.K, self.D, self.norms,
                               self.level_stats, self.operand, stream), "rvq_build_norms")

    def workspace(self, N):
        import torch
        code, nbytes = rvq_encode_workspace_size(N, self.D, self.L, self.K)
        _check(code, "rvq_encode_workspace_size")
        if self._ws is None or self._ws.numel() < nbytes:
            self._ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=self.codebooks.device)
        return self._ws, nbytes

    def encode(self, features, offsets=None, residual=False, recon=False, out=None, status=None,
               fallbacks=None, stream=None, check=True):
        """Greedy RVQ of features [N, D] -> ids [N, L] int32 (+ residual / recon fp32 [N, D])."""
        import torch
        N, D = (int(v) for v in features.shape)
        if D != self.D:
            raise ValueError("feature width differs from the codebooks")
        dev = self.codebooks.device
        o = dict(out or {})
        ids = o.get("ids")
        if ids is None:
            ids = torch.empty((N, self.L), dtype=torch.int32, device=dev)
        res = o.get("residual")
        if residual and res is None:
            res = torch.empty((N, D), dtype=torch.float32, device=dev)
        rec = o.get("recon")
        if recon and rec is None:
            rec = torch.empty((N, D), dtype=torch.float32, device=dev)
        own_status = status is None and check
        if own_status:
            status = torch.zeros(1, dtype=torch.int32, device=dev)
        ws, nbytes = self.workspace(N)
        B = 0 if offsets is None else int(offsets.numel()) - 1
        _check(rvq_encode(features, _dtype_code(features), N, D, self.codebooks, self.cb_dtype,
                          self.operand, self.norms, self.level_stats, self.L, self.K, offsets, B,
                          ids, res if residual else None, rec if recon else None, fallbacks, ws,
                          ws.numel(), status, stream), "rvq_encode")
        if own_status:
            code = int(status.item())
            if code != 0:
                raise RVQError(code, "rvq_encode (device)")
        return ids, (res if residual else None), (rec if recon else None)

    def decode(self, ids, out=None, status=None, stream=None, check=True):
        """recon[n] = sum_l C_l[ids[n, l]] (fp32)."""
        import torch
        N, L = (int(v) for v in ids.shape)
        if L != self.L:
            raise ValueError("ids have a different number of levels")
        rec = out if out is not None else torch.empty((N, self.D), dtype=torch.float32,
                                                      device=self.codebooks.device)
        own_status = status is None and check
        if own_status:
            status = torch.zeros(1, dtype=torch.int32, device=self.codebooks.device)
        _check(rvq_decode(ids, N, L, self.codebooks, self.cb_dtype, self.K, self.D, rec, status, stream),
               "rvq_decode")
        if own_status:
            code = int(status.item())
            if code != 0:
                raise RVQError(code, "rvq_decode (device)")
        return rec
